"""GPU parity: the CUDA path through the C ABI against the CPU oracle, byte for
byte, on the seeded workloads (full size), forced kernel paths, strided and
misaligned inputs, a randomized sweep of small shapes, clamped offsets,
maximum group counts, and CUDA-graph capture."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from scale_factor_layout_b200 import _binding as B  # noqa: E402
from scale_factor_layout_b200 import synth  # noqa: E402
from gpu_util import DeviceCase  # noqa: E402

pytestmark = pytest.mark.gpu


def _check(case, orc, path="auto", misalign=0):
    dc = DeviceCase(case, misalign=misalign)
    st = dc.run(path)
    assert st == B.MX_OK, f"{case.name} path={path}: {B.status_string(st)}"
    torch.cuda.synchronize()
    got = dc.output()
    want = orc.rearrange(case.dim, case.scales, case.ends)
    if not np.array_equal(got, want):
        bad = np.flatnonzero(got != want)
        raise AssertionError(f"{case.name} path={path} misalign={misalign}: {len(bad)} bytes differ, "
                             f"first at {bad[:8]} got {got[bad[:8]]} want {want[bad[:8]]}")
    return dc


@pytest.fixture(scope="module")
def cases():
    return {name: make() for name, make in synth.NAMED.items()}


@pytest.mark.parametrize("name", list(synth.NAMED))
def test_workloads_auto(mxlib, orc, cases, name):
    _check(cases[name], orc)


def flat_ok(c, ptr):
    return (c.dim == synth.DIM_M and ptr % 16 == 0 and c.row_stride % 4 == 0 and c.cols % 4 == 0
            and c.row_stride <= 256 and c.rows >= 1 and c.cols >= 1)


@pytest.mark.parametrize("name,path", [
    ("m_tiny", "flat"), ("m_tiny", "word"), ("m_tiny", "byte"),
    ("m_skinny", "flat"), ("m_skinny", "word"), ("m_skinny", "byte"),
    ("m_wide", "tma"), ("m_wide", "flat"), ("m_wide", "word"), ("m_wide", "byte"),
    ("k_groups", "tma"), ("k_groups", "word"), ("k_groups", "byte"),
])
def test_workloads_forced_path(mxlib, orc, cases, name, path):
    _check(cases[name], orc, path)


@pytest.mark.parametrize("rows,cols", [(262144, 44), (600000, 44), (700000, 60), (40000, 100), (40000, 252)])
def test_flat_instances(mxlib, orc, rows, cols):
    """The flat-row kernel's instances at the sizes where each is chosen:
    4 warps with direct stores (up to two waves of items: 262144 rows) and
    with staged bulk stores (more: 600000 and 700000 rows), and 8 warps with
    direct stores for rows of 65-256 padded columns; the row stride is the
    column count (a multiple of 4, not of 16)."""
    rng = np.random.default_rng(5100 + cols + rows)
    scales = rng.integers(1, 255, size=(rows, cols), dtype=np.uint8)
    sizes = synth.split_multinomial(rng, rows, 8)
    case = synth.Case(f"flat{rows}x{cols}", synth.DIM_M, scales, np.cumsum(sizes).astype(np.int32), 0)
    dc = DeviceCase(case)
    assert B.mx_select_path(case.dim, dc.ptr, case.rows, case.cols, case.row_stride) == B.MX_PATH_FLAT
    _check(case, orc, "auto")


def test_auto_dispatch_choices(mxlib, cases):
    for name, want in (("m_tiny", B.MX_PATH_FLAT), ("m_skinny", B.MX_PATH_FLAT),
                       ("m_wide", B.MX_PATH_TMA), ("k_groups", B.MX_PATH_TMA)):
        c = cases[name]
        dc = DeviceCase(c)
        assert B.mx_select_path(c.dim, dc.ptr, c.rows, c.cols, c.row_stride) == want


@pytest.mark.parametrize("i_rows", range(len(synth.SWEEP_ROWS)))
def test_k_sweep(mxlib, orc, i_rows):
    for i_k in range(len(synth.SWEEP_TOTAL_K)):
        _check(synth.k_sweep_point(i_rows, i_k), orc)


def test_k_groups_large_ragged(mxlib, orc):
    """A 193 MiB K-groups input, whole output compared: rows that end inside
    a row band, 64 groups from a few columns (quads that straddle group
    boundaries) to hundreds wide, empty groups, columns that no group covers,
    and gap bytes between rows."""
    rng = np.random.default_rng(4700)
    rows, cols, G = 16461, 12293, 64
    widths = np.where(rng.random(G) < 0.5, rng.integers(0, 10, size=G), rng.integers(50, 600, size=G))
    widths[rng.random(G) < 0.1] = 0
    while widths.sum() > cols - 37:
        widths[int(rng.integers(0, G))] //= 2
    base = synth.Case("k_large", synth.DIM_K, np.zeros((rows, cols), np.uint8),
                      np.cumsum(widths).astype(np.int32), 4700)
    case = synth.strided(base, (-cols) % 16 + 16)
    assert case.rows * case.cols >= 192 << 20 and case.row_stride % 16 == 0
    _check(case, orc)


@pytest.mark.parametrize("name,pad,path", [
    ("m_wide", 32, "auto"), ("k_groups", 32, "auto"),   # stride still a multiple of 16: TMA with gaps
    ("m_wide", 4, "auto"), ("k_groups", 4, "auto"),     # word path
    ("m_skinny", 4, "auto"), ("m_skinny", 20, "flat"),  # flat path with gaps between rows
    ("m_tiny", 8, "flat"),
    ("m_skinny", 5, "auto"), ("k_groups", 5, "auto"),   # byte path
    ("m_tiny", 19, "auto"),
])
def test_strided(mxlib, orc, cases, name, pad, path):
    _check(synth.strided(cases[name], pad), orc, path)


@pytest.mark.parametrize("misalign", [1, 2, 4, 8, 12])
def test_misaligned_base(mxlib, orc, misalign):
    for c in (synth.m_tiny(), synth.k_sweep_point(1, 3), synth.m_wide()):
        _check(c, orc, misalign=misalign)


def test_arange_pattern(mxlib, orc):
    """Scale bytes arange % 251 (every byte value but four, position-dependent)."""
    for base in (synth.m_wide(), synth.k_groups()):
        vals = (np.arange(base.rows * base.cols) % 251).astype(np.uint8).reshape(base.rows, base.cols)
        c = synth.Case(base.name + "_arange", base.dim, vals, base.ends, base.seed)
        _check(c, orc)


@pytest.mark.parametrize("chunk", range(8))
def test_random_small(mxlib, orc, chunk):
    for seed in range(chunk * 40, chunk * 40 + 40):
        c = synth.random_small(seed)
        paths = ["auto", "byte"]
        dc = DeviceCase(c)
        auto = B.mx_select_path(c.dim, dc.ptr, c.rows, c.cols, c.row_stride)
        if auto in (B.MX_PATH_TMA, B.MX_PATH_FLAT):
            paths.append("word")
        if auto == B.MX_PATH_TMA and flat_ok(c, dc.ptr):
            paths.append("flat")
        for p in paths:
            _check(c, orc, p)


def test_max_groups_and_empty(mxlib, orc):
    rng = np.random.default_rng(7)
    for dim, rows, cols in ((synth.DIM_M, 9000, 96), (synth.DIM_K, 700, 2000), (synth.DIM_M, 300, 20)):
        total = rows if dim == synth.DIM_M else cols
        for pattern in ("random", "all_in_last", "all_in_first", "all_empty", "one_each"):
            if pattern == "random":
                sizes = synth.split_multinomial(rng, total, 64)
            elif pattern == "all_in_last":
                sizes = np.zeros(64, np.int64); sizes[-1] = total
            elif pattern == "all_in_first":
                sizes = np.zeros(64, np.int64); sizes[0] = total
            elif pattern == "all_empty":
                sizes = np.zeros(64, np.int64)
            else:
                sizes = np.ones(64, np.int64); sizes[-1] = total - 63
            s = synth.uniform_scales(rng, rows, cols, 100, 140)
            c = synth.Case(f"g64_{pattern}", dim, s, synth.ends_from_sizes(sizes), 0)
            for p in ("auto", "word") + (("flat",) if flat_ok(c, 0) else ()):
                _check(c, orc, p)


def test_clamped_offsets(mxlib, orc):
    """Offsets past the end, decreasing, or negative are clamped like the oracle."""
    base = synth.m_tiny()
    for ends in ([500, 300, 2000, 900], [-5, 400, 400, 10**9], [1000, 0, 0, 0], [0, 0, 0, 500],
                 [2**31 - 1, 5, 6, 7]):
        c = synth.Case("clamp", synth.DIM_M, base.scales, np.asarray(ends, np.int32), 0)
        _check(c, orc)
        k = synth.Case("clamp_k", synth.DIM_K, base.scales, np.asarray(ends, np.int32) // 20, 0)
        _check(k, orc)


def test_degenerate_shapes(mxlib, orc):
    rng = np.random.default_rng(3)
    for dim, rows, cols in ((synth.DIM_M, 0, 44), (synth.DIM_M, 5, 0), (synth.DIM_K, 5, 0),
                            (synth.DIM_M, 1, 1), (synth.DIM_K, 1, 1), (synth.DIM_K, 129, 3)):
        s = synth.uniform_scales(rng, rows, cols, 100, 140)
        total = rows if dim == synth.DIM_M else cols
        c = synth.Case("degenerate", dim, s, np.asarray([total // 2, total], np.int32), 0)
        if B.mx_rearranged_size(dim, rows, cols, 2) == 0:
            continue
        _check(c, orc)


def test_graph_capture(mxlib, orc):
    """Three calls with different offset buffers captured in one CUDA graph,
    replayed twice; the launch reads the offsets on the device each replay."""
    base = synth.k_groups()
    dc = DeviceCase(base)
    dc.run()  # first call on the device sets kernel attributes, outside capture
    torch.cuda.synchronize()
    rng = np.random.default_rng(9)
    splits = [synth.ends_from_sizes(synth.split_distinct_cuts(rng, base.cols, 8)) for _ in range(3)]
    dev_ends = [torch.from_numpy(e).cuda() for e in splits]
    outs = [torch.empty(dc.size, dtype=torch.uint8, device="cuda") for _ in range(3)]
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for e, o in zip(dev_ends, outs):
                st = B.mx_rearrange_ex(base.dim, dc.ptr, base.rows, base.cols, base.row_stride, e.data_ptr(), 8,
                                       o.data_ptr(), B.MX_PATH_AUTO, s.cuda_stream)
                assert st == B.MX_OK
    for _ in range(2):
        for o in outs:
            o.fill_(0x5A)
        g.replay()
        torch.cuda.synchronize()
        for e, o in zip(splits, outs):
            assert np.array_equal(o.cpu().numpy(), orc.rearrange(base.dim, base.scales, e))
    # new offsets written in place are picked up on the next replay
    new = synth.ends_from_sizes(synth.split_distinct_cuts(rng, base.cols, 8))
    dev_ends[0].copy_(torch.from_numpy(new))
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(outs[0].cpu().numpy(), orc.rearrange(base.dim, base.scales, new))
    del g


def test_torch_wrapper(mxlib, orc):
    import scale_factor_layout_b200 as mxs

    c = synth.m_wide()
    s = torch.from_numpy(np.ascontiguousarray(c.scales)).cuda()
    e = torch.from_numpy(c.ends).cuda()
    out = mxs.rearrange_m_groups(s, e)
    assert np.array_equal(out.cpu().numpy(), orc.rearrange(c.dim, c.scales, c.ends))
    k = synth.k_groups()
    out = mxs.rearrange_k_groups(torch.from_numpy(np.ascontiguousarray(k.scales)).cuda(),
                                 torch.from_numpy(k.ends).cuda())
    assert np.array_equal(out.cpu().numpy(), orc.rearrange(k.dim, k.scales, k.ends))


def test_no_device_flags_raised(mxlib):
    torch.cuda.synchronize()
    assert B.mx_device_flags() == 0
