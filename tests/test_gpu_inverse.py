"""GPU parity of the inverse rearrange (blocked -> row-major) and of the padded
group starts, against the CPU oracle; round trips through both directions."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import scale_factor_layout_b200 as mxs  # noqa: E402
from scale_factor_layout_b200 import _binding as B  # noqa: E402
from scale_factor_layout_b200 import synth  # noqa: E402

pytestmark = pytest.mark.gpu
SENTINEL = 0xEE


def _inverse_check(case, orc, out_pad=0, misalign=0, blocked_np=None):
    """Blocked input from the oracle (or given); run the GPU inverse into a
    strided, possibly misaligned row-major buffer pre-filled with a sentinel."""
    rows, cols, dim = case.rows, case.cols, case.dim
    if blocked_np is None:
        blocked_np = orc.rearrange(dim, case.scales, case.ends)
    blocked = torch.from_numpy(blocked_np).cuda()
    ends = torch.from_numpy(np.ascontiguousarray(case.ends, dtype=np.int32)).cuda()
    stride = cols + out_pad
    nbytes = rows * stride + misalign + 64
    buf = torch.full((nbytes,), SENTINEL, dtype=torch.uint8, device="cuda")
    ptr = buf.data_ptr() + misalign
    fn = B.mx_unrearrange_m_groups if dim == synth.DIM_M else B.mx_unrearrange_k_groups
    st = fn(blocked.data_ptr(), rows, cols, ends.data_ptr(), len(case.ends), ptr, stride,
            torch.cuda.current_stream().cuda_stream)
    assert st == B.MX_OK, B.status_string(st)
    torch.cuda.synchronize()
    host = buf.cpu().numpy()
    assert (host[:misalign] == SENTINEL).all() and (host[misalign + rows * stride:] == SENTINEL).all()
    view = host[misalign: misalign + rows * stride].reshape(rows, stride) if rows else np.zeros((0, stride), np.uint8)
    want = orc.inverse(dim, blocked_np, rows, cols, case.ends)
    if not np.array_equal(view[:, :cols], want):
        bad = np.argwhere(view[:, :cols] != want)
        raise AssertionError(f"{case.name}: {len(bad)} elements differ, first {bad[:5].tolist()}")
    assert (view[:, cols:] == SENTINEL).all(), "row-stride gap bytes were written"


@pytest.mark.parametrize("name", list(synth.NAMED))
def test_inverse_workloads(mxlib, orc, name):
    _inverse_check(synth.NAMED[name](), orc)


@pytest.mark.parametrize("name,pad,misalign", [("m_tiny", 5, 3), ("m_wide", 16, 0), ("k_groups", 3, 1),
                                               ("m_skinny", 4, 4), ("k_groups", 0, 8)])
def test_inverse_strided_misaligned_out(mxlib, orc, name, pad, misalign):
    _inverse_check(synth.NAMED[name](), orc, out_pad=pad, misalign=misalign)


@pytest.mark.parametrize("misalign", range(16))
def test_inverse_every_chunk_offset(mxlib, orc, misalign):
    """Row strides that are multiples of 16 with the output base at every
    offset within a 16-byte chunk: each row of an item then starts at the same
    offset, and every head and tail mask of a partial chunk occurs (K groups
    start at arbitrary columns; M rows wider than one 128-column item)."""
    rng = np.random.default_rng(4100 + misalign)
    rows, cols = 300, 700
    scales = rng.integers(1, 255, size=(rows, cols), dtype=np.uint8)
    cuts = np.sort(rng.choice(np.arange(1, cols), size=7, replace=False))
    k_case = synth.Case("shiftK", synth.DIM_K, scales, np.append(cuts, cols).astype(np.int32), 0)
    _inverse_check(k_case, orc, out_pad=(-cols) % 16 + 16, misalign=misalign)
    m_scales = rng.integers(1, 255, size=(rows, 150), dtype=np.uint8)
    m_case = synth.Case("shiftM", synth.DIM_M, m_scales, np.array([0, 77, 200, 200, 300], np.int32), 0)
    _inverse_check(m_case, orc, out_pad=(-150) % 16, misalign=misalign)


@pytest.mark.parametrize("misalign", [0, 1, 5, 11, 13, 15])
def test_inverse_narrow_k_groups(mxlib, orc, misalign):
    """K groups of 0..24 columns, so that seam chunks hold bytes of up to three
    groups and every branch of the seam rule runs: seams written whole by the
    later group, seams left to masked copies because the earlier group is
    narrower than the seam offset, because its columns spread over five tiles,
    or because the later group does not fill the chunk; empty groups between."""
    rng = np.random.default_rng(4200 + misalign)
    rows, G = 260, 64
    widths = rng.integers(0, 25, size=G)
    widths[rng.random(G) < 0.2] = 0
    cols = int(widths.sum()) + 7          # the last 7 columns are not covered by any group
    scales = rng.integers(1, 255, size=(rows, cols), dtype=np.uint8)
    case = synth.Case("narrowK", synth.DIM_K, scales, np.cumsum(widths).astype(np.int32), 0)
    _inverse_check(case, orc, out_pad=(-cols) % 16 + 16, misalign=misalign)


@pytest.mark.parametrize("seed", range(12))
def test_inverse_k_output_boxes(mxlib, orc, seed):
    """Groups along K into a 16-byte aligned output with a row stride that is a
    multiple of 16: the kernel that writes 128 x 128 boxes of the output with
    tensor stores.  Widths from 16 to 1100 columns (a last chunk cut by the
    width, boxes narrower than 128), groups from one column wide to wider than
    a box (so boxes hold one to many pieces, beyond what a stage takes), empty
    groups, columns no group covers, and rows that end inside a row band."""
    rng = np.random.default_rng(4600 + seed)
    rows = int(rng.integers(1, 700))
    cols = int(rng.choice([16, 17, 40, 127, 128, 129, 300, 512, 1100, int(rng.integers(16, 1200))]))
    G = int(rng.integers(1, 65))
    narrow = seed % 3 == 0
    widths = rng.integers(0, 12 if narrow else 2 * cols // G + 2, size=G)
    widths[rng.random(G) < 0.15] = 0
    while widths.sum() > cols:
        widths[int(rng.integers(0, G))] //= 2
    scales = rng.integers(1, 255, size=(rows, cols), dtype=np.uint8)
    case = synth.Case("boxK", synth.DIM_K, scales, np.cumsum(widths).astype(np.int32), 0)
    for pad in ((-cols) % 16, (-cols) % 16 + 16):
        _inverse_check(case, orc, out_pad=pad, misalign=0)


@pytest.mark.parametrize("unit", [1, 4, 16, 128])
def test_inverse_k_boxes_seam_alignment(mxlib, orc, unit):
    """Output boxes whose group seams all fall on multiples of `unit` columns:
    with 16 and 128 every 16-column output chunk lies inside one group and
    starts on a tile boundary (the path with no shift and no seam merge); with
    4 the seams sit on tiles but inside chunks; with 1 anywhere.  The last 48
    columns belong to no group when the groups cover only whole units."""
    rng = np.random.default_rng(4700 + unit)
    rows, cols = 389, 1072
    covered = cols - cols % unit if unit > 1 else cols
    widths = synth.split_units(rng, covered, 8, unit)
    scales = rng.integers(1, 255, size=(rows, cols), dtype=np.uint8)
    case = synth.Case(f"seams{unit}K", synth.DIM_K, scales, np.cumsum(widths).astype(np.int32), 0)
    for pad in (0, 16):
        _inverse_check(case, orc, out_pad=pad, misalign=0)


def test_inverse_ignores_padding_values(mxlib, orc):
    """Padding bytes of the blocked buffer (and its tail) filled with garbage
    change nothing: the inverse reads whole tiles but writes only real data."""
    rng = np.random.default_rng(4400)
    cases = [synth.m_tiny(), synth.k_sweep_point(2, 3), synth.random_small(601), synth.random_small(777)]
    rows, cols = 300, 700
    cuts = np.sort(rng.choice(np.arange(1, cols), size=7, replace=False))
    cases.append(synth.Case("padK", synth.DIM_K, rng.integers(1, 255, size=(rows, cols), dtype=np.uint8),
                            np.append(cuts, cols).astype(np.int32), 0))
    for case in cases:
        blocked = orc.rearrange(case.dim, case.scales, case.ends)
        r, _ = orc.decode_at(case.dim, case.rows, case.cols, case.ends, np.arange(blocked.size, dtype=np.int64))
        dirty = blocked.copy()
        pad = r < 0
        dirty[pad] = rng.integers(1, 256, size=int(pad.sum()), dtype=np.uint8)
        for pad_out, misalign in ((0, 0), ((-case.cols) % 16 + 16, 3)):
            _inverse_check(case, orc, out_pad=pad_out, misalign=misalign, blocked_np=dirty)


def test_inverse_sweep_subset(mxlib, orc):
    for i_rows in range(len(synth.SWEEP_ROWS)):
        for i_k in (0, 3, 6):
            _inverse_check(synth.k_sweep_point(i_rows, i_k), orc)


@pytest.mark.parametrize("chunk", range(4))
def test_inverse_random_small(mxlib, orc, chunk):
    for seed in range(500 + chunk * 50, 500 + chunk * 50 + 50):
        c = synth.random_small(seed)
        _inverse_check(c, orc, out_pad=seed % 7, misalign=seed % 5)


def test_inverse_clamped_and_uncovered(mxlib, orc):
    base = synth.m_tiny()
    for ends in ([500, 300, 2000, 900], [0, 0, 0, 500], [100, 200, 300, 400]):
        _inverse_check(synth.Case("clampM", synth.DIM_M, base.scales, np.asarray(ends, np.int32), 0), orc)
        _inverse_check(synth.Case("clampK", synth.DIM_K, base.scales, np.asarray(ends, np.int32) // 20, 0), orc)


def test_round_trip_on_gpu(mxlib, orc):
    """forward then inverse on the GPU returns the covered input exactly."""
    for c in (synth.m_wide(), synth.k_groups(), synth.m_skinny()):
        s = torch.from_numpy(np.ascontiguousarray(c.scales)).cuda()
        e = torch.from_numpy(c.ends).cuda()
        blocked = mxs.rearrange(c.dim, s, e)
        back = mxs.unrearrange(c.dim, blocked, c.rows, c.cols, e)
        torch.cuda.synchronize()
        assert torch.equal(back, s)


def test_padded_group_starts(mxlib, orc):
    rng = np.random.default_rng(17)
    for _ in range(60):
        dim = int(rng.integers(0, 2))
        rows, cols, G = int(rng.integers(0, 20000)), int(rng.integers(1, 5000)), int(rng.integers(1, 65))
        T = rows if dim == synth.DIM_M else cols
        ends = rng.integers(-10, T + 50, size=G).astype(np.int32)
        if rng.random() < 0.5:
            ends = np.sort(ends)
        got = mxs.padded_group_starts(dim, rows, cols, torch.from_numpy(ends).cuda()).cpu().numpy()
        want = orc.padded_group_starts(dim, rows, cols, ends)
        assert np.array_equal(got.astype(np.int64), want), (dim, rows, cols, ends)


def test_inverse_graph_capture(mxlib, orc):
    """The inverse calls (output boxes along K, tensor-store boxes along M)
    captured in one CUDA graph and replayed; group ends rewritten in place
    between replays are read on the device by the next replay."""
    rng = np.random.default_rng(4800)
    cases = [synth.k_groups(), synth.m_wide()]
    blocked, ends_d, outs = [], [], []
    for c in cases:
        e = torch.from_numpy(np.ascontiguousarray(c.ends, dtype=np.int32)).cuda()
        blocked.append(torch.from_numpy(orc.rearrange(c.dim, c.scales, c.ends)).cuda())
        ends_d.append(e)
        outs.append(torch.empty((c.rows, c.cols), dtype=torch.uint8, device="cuda"))

    def call(i, stream):
        c = cases[i]
        fn = B.mx_unrearrange_m_groups if c.dim == synth.DIM_M else B.mx_unrearrange_k_groups
        st = fn(blocked[i].data_ptr(), c.rows, c.cols, ends_d[i].data_ptr(), len(c.ends), outs[i].data_ptr(),
                c.cols, stream)
        assert st == B.MX_OK, B.status_string(st)

    s = torch.cuda.Stream()
    for i in range(len(cases)):     # first calls set kernel attributes, outside capture
        call(i, s.cuda_stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(len(cases)):
                call(i, s.cuda_stream)
    for rep in range(3):
        if rep == 2:
            # other group ends, the same blocked buffers read under them
            c = cases[0]
            new = synth.ends_from_sizes(synth.split_distinct_cuts(rng, c.cols, len(c.ends)))
            ends_d[0].copy_(torch.from_numpy(new))
            cases[0] = synth.Case(c.name, c.dim, c.scales, new, c.seed)
        for o in outs:
            o.fill_(0x5A)
        g.replay()
        torch.cuda.synchronize()
        for i, c in enumerate(cases):
            want = orc.inverse(c.dim, blocked[i].cpu().numpy(), c.rows, c.cols, c.ends)
            assert np.array_equal(outs[i].cpu().numpy(), want), (rep, c.name)
    del g
