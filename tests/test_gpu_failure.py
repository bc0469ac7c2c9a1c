"""Failure detection on the GPU without a fault: a bounded pipeline wait on a
barrier that nothing arrives at gives up, raises the device flag, and the
context stays usable for ordinary calls."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from scale_factor_layout_b200 import _binding as B  # noqa: E402
from scale_factor_layout_b200 import synth  # noqa: E402
from gpu_util import DeviceCase  # noqa: E402

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_flags(mxlib, orc):
    torch.cuda.synchronize()
    B.mx_device_flags(clear=True)
    assert B.mx_selftest_bounded_wait(1 << 20, torch.cuda.current_stream().cuda_stream) == B.MX_OK
    torch.cuda.synchronize()
    assert B.mx_device_flags(clear=True) & 1, "timeout flag not raised"
    assert B.mx_device_flags() == 0, "flags not cleared"
    # the context still works
    c = synth.m_tiny()
    dc = DeviceCase(c)
    assert dc.run() == B.MX_OK
    torch.cuda.synchronize()
    assert np.array_equal(dc.output(), orc.rearrange(c.dim, c.scales, c.ends))


def test_selftest_rejects_bad_limits(mxlib):
    assert B.mx_selftest_bounded_wait(0) == B.MX_ERR_INVALID_ARG
    assert B.mx_selftest_bounded_wait((1 << 32) + 1) == B.MX_ERR_INVALID_ARG
