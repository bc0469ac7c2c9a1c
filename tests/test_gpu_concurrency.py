"""Calls from several host threads on several streams at once: the library's
host state (tensor-map encoder, per-device set-up) is shared, every call is
independent, and all outputs match the oracle."""
import threading

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from scale_factor_layout_b200 import _binding as B  # noqa: E402
from scale_factor_layout_b200 import synth  # noqa: E402
from gpu_util import DeviceCase  # noqa: E402

pytestmark = pytest.mark.gpu


def test_threads_and_streams(mxlib, orc):
    cases = [synth.m_skinny(), synth.m_wide(), synth.k_groups(), synth.m_tiny(),
             synth.strided(synth.k_groups(), 5), synth.k_sweep_point(3, 5)]
    dcs = [DeviceCase(c) for c in cases]
    torch.cuda.synchronize()
    errors = []

    def worker(dc):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for _ in range(5):
                    st = dc.run(stream=s.cuda_stream)
                    if st != B.MX_OK:
                        errors.append((dc.case.name, st, B.mx_last_cuda_error()))
            s.synchronize()
        except Exception as exc:  # noqa: BLE001
            errors.append((dc.case.name, repr(exc)))

    threads = [threading.Thread(target=worker, args=(dc,)) for dc in dcs]
    for t in threads:
        t.start()
    for t in threads:
        t.join(120)
    assert not errors, errors
    torch.cuda.synchronize()
    for dc in dcs:
        c = dc.case
        assert np.array_equal(dc.output(), orc.rearrange(c.dim, c.scales, c.ends)), c.name


def test_fresh_thread_legacy_stream(mxlib, orc):
    """A host thread whose first CUDA work is a library call on the legacy
    stream (no torch call in that thread): the tensor-map paths must work."""
    cases = [synth.m_wide(), synth.k_groups(), synth.m_skinny()]
    dcs = [DeviceCase(c) for c in cases]
    torch.cuda.synchronize()
    results = []

    def worker(dc):
        results.append((dc.case.name, dc.run(stream=0), B.mx_last_cuda_error()))

    for dc in dcs:
        t = threading.Thread(target=worker, args=(dc,))
        t.start()
        t.join(60)
    assert all(st == B.MX_OK for _, st, _ in results), results
    torch.cuda.synchronize()
    for dc in dcs:
        c = dc.case
        assert np.array_equal(dc.output(), orc.rearrange(c.dim, c.scales, c.ends)), c.name


def test_fresh_thread_inverse(mxlib, orc):
    """The inverse from a host thread whose first CUDA work is the library call
    (the M-groups path encodes an output tensor map, a driver call that needs
    the device's context current in that thread)."""
    cases = [synth.m_wide(), synth.k_groups(), synth.m_skinny()]
    prepared = []
    for c in cases:
        blocked_np = orc.rearrange(c.dim, c.scales, c.ends)
        blocked = torch.from_numpy(blocked_np).cuda()
        ends = torch.from_numpy(np.ascontiguousarray(c.ends, dtype=np.int32)).cuda()
        out = torch.full((c.rows, c.cols), 0xEE, dtype=torch.uint8, device="cuda")
        prepared.append((c, blocked_np, blocked, ends, out))
    torch.cuda.synchronize()
    results = []

    def worker(c, blocked, ends, out):
        fn = B.mx_unrearrange_m_groups if c.dim == synth.DIM_M else B.mx_unrearrange_k_groups
        st = fn(blocked.data_ptr(), c.rows, c.cols, ends.data_ptr(), len(c.ends), out.data_ptr(), c.cols, 0)
        results.append((c.name, st, B.mx_last_cuda_error()))

    for c, _, blocked, ends, out in prepared:
        t = threading.Thread(target=worker, args=(c, blocked, ends, out))
        t.start()
        t.join(60)
    assert all(st == B.MX_OK for _, st, _ in results), results
    torch.cuda.synchronize()
    for c, blocked_np, _, _, out in prepared:
        assert np.array_equal(out.cpu().numpy(), orc.inverse(c.dim, blocked_np, c.rows, c.cols, c.ends)), c.name
