"""Inputs and outputs larger than 2 GiB (byte offsets past 2^31) on the GPU.

The oracle cannot hold whole outputs this large in a test's time, so the
input is an analytic byte pattern made on the device, and the output is
checked at sampled positions (random ones, every byte around offset 2^31, the
first and last 64 KiB) that the oracle decodes one by one into the input
element they hold, or padding.  The inverse is checked on sampled rows against
the same pattern (covered elements come back, uncovered ones are zero)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import scale_factor_layout_b200 as mxs  # noqa: E402
from scale_factor_layout_b200 import _binding as B  # noqa: E402
from scale_factor_layout_b200 import synth  # noqa: E402

pytestmark = pytest.mark.gpu
SENTINEL = 0xEE


def _pattern(i, j):
    """Byte at element (i, j): never 0, so padding is told apart from data."""
    return (i * 131 + j * 7) % 251 + 1


def _make_input(rows, cols, device):
    s = torch.empty((rows, cols), dtype=torch.uint8, device=device)
    j = torch.arange(cols, device=device, dtype=torch.int64)[None, :]
    step = max(1, (1 << 26) // cols)
    for r0 in range(0, rows, step):
        i = torch.arange(r0, min(rows, r0 + step), device=device, dtype=torch.int64)[:, None]
        s[r0:r0 + i.shape[0]] = _pattern(i, j).to(torch.uint8)
    return s


def _sample_positions(size, rng):
    pos = [rng.integers(0, size, size=2_000_000, dtype=np.int64),
           np.arange(max(0, (1 << 31) - 65536), min(size, (1 << 31) + 65536), dtype=np.int64),
           np.arange(0, min(size, 65536), dtype=np.int64),
           np.arange(max(0, size - 65536), size, dtype=np.int64)]
    return np.unique(np.concatenate(pos))


@pytest.mark.parametrize("dim,rows,cols", [(synth.DIM_M, 1_000_077, 2304), (synth.DIM_K, 65_613, 36_032)])
def test_beyond_2gib(mxlib, orc, dim, rows, cols):
    dev = torch.device("cuda", 0)
    rng = np.random.default_rng(4300 + dim)
    total = rows if dim == synth.DIM_M else cols
    ends = np.append(np.sort(rng.choice(np.arange(1, total), size=7, replace=False)), total).astype(np.int32)
    scales = _make_input(rows, cols, dev)
    ends_d = torch.from_numpy(ends).to(dev)
    size = mxs.mx_rearranged_size(dim, rows, cols, len(ends))
    assert size > (1 << 31) + (1 << 20)
    out = torch.full((size,), SENTINEL, dtype=torch.uint8, device=dev)
    fn = B.mx_rearrange_m_groups if dim == synth.DIM_M else B.mx_rearrange_k_groups
    st = fn(scales.data_ptr(), rows, cols, cols, ends_d.data_ptr(), len(ends), out.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
    assert st == B.MX_OK, B.status_string(st)
    assert B.mx_select_path(dim, scales.data_ptr(), rows, cols, cols) == B.MX_PATH_TMA

    pos = _sample_positions(size, rng)
    got = out[torch.from_numpy(pos).to(dev)].cpu().numpy()
    r, c = orc.decode_at(dim, rows, cols, ends, pos)
    want = np.where(r < 0, 0, _pattern(r, c)).astype(np.uint8)
    bad = np.flatnonzero(got != want)
    assert len(bad) == 0, f"{len(bad)} of {len(pos)} sampled bytes differ, first at {pos[bad[:5]]}"

    # inverse back to row-major; sampled rows against the pattern
    back = torch.full((rows, cols), SENTINEL, dtype=torch.uint8, device=dev)
    ifn = B.mx_unrearrange_m_groups if dim == synth.DIM_M else B.mx_unrearrange_k_groups
    st = ifn(out.data_ptr(), rows, cols, ends_d.data_ptr(), len(ends), back.data_ptr(), cols,
             torch.cuda.current_stream().cuda_stream)
    assert st == B.MX_OK, B.status_string(st)
    sample_rows = np.unique(np.concatenate([rng.integers(0, rows, size=200), [0, rows - 1],
                                            np.arange(max(0, rows - 130), rows)]))
    got_rows = back[torch.from_numpy(sample_rows).to(dev)].cpu().numpy().astype(np.int64)
    i = sample_rows[:, None].astype(np.int64)
    j = np.arange(cols, dtype=np.int64)[None, :]
    want_rows = _pattern(i, j)
    used = int(ends[-1])
    if dim == synth.DIM_M:
        want_rows = np.where(i < used, want_rows, 0)
    else:
        want_rows = np.where(j < used, want_rows, 0)
    assert np.array_equal(got_rows, want_rows)
    del out, back, scales
    torch.cuda.empty_cache()
