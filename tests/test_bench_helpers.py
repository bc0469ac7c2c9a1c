"""Host-side helpers of bench.py: the device-code key that ties the DRAM
traffic figures of profiles/ncu_traffic.txt to the kernels they were taken on."""
import os
import shutil

import bench


def _copy_tree(tmp_path):
    dst = tmp_path / "scale_factor_layout_b200" / "csrc"
    dst.mkdir(parents=True)
    src = os.path.join(bench.ROOT, "scale_factor_layout_b200", "csrc")
    for name in ("mx_device.cuh", "mx_rearrange.cu", "mx_inverse.cu"):
        shutil.copy(os.path.join(src, name), dst / name)
    return dst


def _keys(root):
    return bench.kernel_source_sha(root), bench.kernel_source_sha(root, op="inverse")


def test_key_ignores_comments_and_host_code(tmp_path):
    csrc = _copy_tree(tmp_path)
    before = _keys(str(tmp_path))
    p = csrc / "mx_device.cuh"
    p.write_text(p.read_text().replace("namespace mx {", "namespace mx {\n// a comment added\n\n", 1))
    for name in ("mx_rearrange.cu", "mx_inverse.cu"):
        q = csrc / name
        q.write_text(q.read_text() + "\nstatic int host_side_addition = 0;\n")
    assert _keys(str(tmp_path)) == before


def test_key_tracks_each_ops_device_code(tmp_path):
    csrc = _copy_tree(tmp_path)
    fwd, inv = _keys(str(tmp_path))
    q = csrc / "mx_inverse.cu"
    text = q.read_text()
    cut = text.index(bench.HOST_MARKER.decode())
    assert "kInvStages = 2" in text[:cut]
    q.write_text(text[:cut].replace("kInvStages = 2", "kInvStages = 3", 1) + text[cut:])
    assert bench.kernel_source_sha(str(tmp_path)) == fwd
    assert bench.kernel_source_sha(str(tmp_path), op="inverse") != inv
    p = csrc / "mx_device.cuh"     # shared by both ops
    p.write_text(p.read_text().replace("constexpr int kTileRows = 128;", "constexpr int kTileRows = 256;", 1))
    assert bench.kernel_source_sha(str(tmp_path)) != fwd


def test_traffic_lookup_by_op_call_and_key(tmp_path):
    _copy_tree(tmp_path)
    fwd, inv = _keys(str(tmp_path))
    traffic = tmp_path / "traffic.txt"
    traffic.write_text("# header\n"
                       f"op=rearrange call=k_groups bytes_per_launch=111 source_sha={fwd} capture=a.md\n"
                       f"op=inverse call=k_groups bytes_per_launch=222 source_sha={inv} capture=b.md\n"
                       f"op=inverse call=m_wide bytes_per_launch=333 source_sha=0000000000000000 capture=c.md\n")
    root, path = str(tmp_path), str(traffic)
    assert bench.ncu_traffic("k_groups", "rearrange", root, path) == 111
    assert bench.ncu_traffic("k_groups", "inverse", root, path) == 222
    assert bench.ncu_traffic("m_wide", "inverse", root, path) is None      # taken on other kernels
    assert bench.ncu_traffic("m_skinny", "rearrange", root, path) is None  # never captured


def test_algorithmic_bytes_match_the_oracle(orc):
    """The bytes behind the bench's GB/s (real input read, exact padded output
    written, the allocation) agree with the oracle's own counts."""
    from scale_factor_layout_b200 import synth

    cases = [f() for f in synth.NAMED.values()]
    cases += [synth.k_sweep_point(i, k) for i in (0, 3, 6) for k in (0, 5, 9)]
    cases += [synth.random_small(seed) for seed in range(900, 1100)]
    for c in cases:
        b = bench.algorithmic_bytes(c)
        assert b["read"] == orc.read_bytes(c.dim, c.rows, c.cols, c.ends), c.name
        assert b["written"] == orc.written_bytes(c.dim, c.rows, c.cols, c.ends), c.name
        assert b["alloc"] == orc.rearranged_size(c.dim, c.rows, c.cols, len(c.ends)), c.name


def test_traffic_detail_and_roofline_fields(tmp_path):
    """The roofline object carries read and write traffic apart, flags a
    launch whose writes are still in L2 when it ends, and gives the fraction
    of the nominal peak beside the measured one."""
    _copy_tree(tmp_path)
    fwd, _ = _keys(str(tmp_path))
    traffic = tmp_path / "traffic.txt"
    traffic.write_text(f"op=rearrange call=k_groups bytes_per_launch=1068 read=1000 write=68 l2_write=998 "
                       f"source_sha={fwd} capture=a.md\n"
                       f"op=rearrange call=m_wide bytes_per_launch=2000 read=1000 write=1000 "
                       f"source_sha={fwd} capture=b.md\n")
    root, path = str(tmp_path), str(traffic)
    t = bench.ncu_traffic("k_groups", "rearrange", root, path, detail=True)
    assert t == {"read": 1000, "write": 68, "l2_write": 998}
    assert bench.ncu_traffic("m_wide", "rearrange", root, path, detail=True)["l2_write"] is None
    r = bench.roofline_entry("k", "k_groups", 2000, 1e-6, 4000.0, "measured", t)
    assert r["achieved"] == 2.0 and r["frac"] == round(2.0 / 4000.0, 4)
    assert r["frac_of_nominal"] == round(2.0 / bench.NOMINAL_HBM_GBS, 4)
    assert (r["traffic"], r["traffic_read"], r["traffic_write"], r["traffic_l2_write"]) == (1068, 1000, 68, 998)
    assert "traffic_note" in r
    full = bench.roofline_entry("k", "m_wide", 2000, 1e-6, 4000.0, "measured",
                                bench.ncu_traffic("m_wide", "rearrange", root, path, detail=True))
    assert "traffic_note" not in full and "traffic_l2_write" not in full
    assert bench.roofline_entry("k", "x", 2000, 1e-6, 4000.0, "measured", None)["traffic"] is None


def test_timing_graph_sizes():
    """Per-call timing graphs hold at least the minimum launch count; sweep
    graphs hold about 20 ms of work, between 20 and 2000 launches."""
    assert bench.per_launch_launches(20, 2000) == 2000
    assert bench.per_launch_launches(4000, 2000) == 4000
    assert bench.sweep_launches(8192) == 2000
    assert bench.sweep_launches(940_000_000) == 84
    assert bench.sweep_launches(10**12) == 20


def test_oracle_seconds_times_either_op():
    """The sweep's CPU leg times the oracle's rearrange, or its inverse of the
    oracle's own blocked output, on the host (no GPU)."""
    from scale_factor_layout_b200 import synth

    case = synth.k_sweep_point(0, 0)   # 128 x 32 scale columns, G=8
    for op in ("rearrange", "inverse"):
        t, how = bench.oracle_seconds(case, op)
        assert t > 0 and how.startswith("median of 3 runs of ")
