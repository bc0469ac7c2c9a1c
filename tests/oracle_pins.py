"""Pins that tie the CPU oracle to something other than itself.

Each ``pin_*`` takes a loaded oracle library and raises AssertionError on a
mismatch.  They are run against the real oracle by ``test_oracle_pins.py`` and
against copies of the oracle with planted mistakes by
``test_oracle_mutants.py`` (``python tests/oracle_pins.py <lib.so>`` exits
non-zero when any pin fails).

What they compare against:
  * hand-worked positions (golden/hand_positions.txt);
  * the bandwidth tables printed in pytorch/ao #3604 and #4704, which fix the
    K-groups output allocation (golden/page_k_groups_bandwidth.tsv);
  * the layout stated as a chain of numpy index reshapes (brute force);
  * the textbook reduction of one tile to a 4x32 -> 32x4 transpose of 32-bit
    words (numpy ``.T``);
  * the running-max closed form of the offset clamp;
  * invariants: bijection of tagged inputs, zero padding, inverse round trip,
    per-group decomposition, M and K agreeing on a single group.
"""
from __future__ import annotations

import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from scale_factor_layout_b200 import synth  # noqa: E402

M, K = oracle.DIM_M, oracle.DIM_K
GOLDEN = os.path.join(HERE, "golden")


# ---------------------------------------------------------------- references
def ceil_to(x: int, a: int) -> int:
    return -(-x // a) * a


def blocked_reference(mat: np.ndarray) -> np.ndarray:
    """Blocked layout of one padded matrix (rows % 128 == 0, cols % 4 == 0)
    written as index reshapes: tiles of 128 rows x 4 columns in row-block-major
    order; inside a tile, row r = 32*a + b and the bytes run over (b, a, c)."""
    R, C = mat.shape
    t = mat.reshape(R // 128, 128, C // 4, 4)
    t = t.transpose(0, 2, 1, 3)
    t = t.reshape(R // 128, C // 4, 4, 32, 4)
    t = t.transpose(0, 1, 3, 2, 4)
    return np.ascontiguousarray(t).reshape(-1)


def pad_to(mat: np.ndarray, R: int, C: int) -> np.ndarray:
    out = np.zeros((R, C), dtype=mat.dtype)
    out[: mat.shape[0], : mat.shape[1]] = mat
    return out


def clamp_reference(ends, limit: int) -> np.ndarray:
    """Closed form of E'[g] = min(max(E[g], E'[g-1]), T), E'[-1] = 0: a running
    maximum of max(E, 0), capped at T."""
    e = np.maximum(np.asarray(ends, dtype=np.int64), 0)
    return np.minimum(np.maximum.accumulate(e), limit)


def brute_force(dim: int, S: np.ndarray, ends, alloc: int) -> np.ndarray:
    rows, cols = S.shape
    e = clamp_reference(ends, rows if dim == M else cols)
    parts, begin = [], 0
    for end in e:
        end = int(end)
        if dim == M:
            block = S[begin:end, :]
            parts.append(blocked_reference(pad_to(block, ceil_to(end - begin, 128), ceil_to(cols, 4))))
        else:
            block = S[:, begin:end]
            parts.append(blocked_reference(pad_to(block, ceil_to(rows, 128), ceil_to(end - begin, 4))))
        begin = end
    flat = np.concatenate(parts) if parts else np.zeros(0, np.uint8)
    out = np.zeros(alloc, dtype=np.uint8)
    out[: len(flat)] = flat
    return out


def tiny_cases(n: int = 120, seed0: int = 1000):
    for s in range(seed0, seed0 + n):
        yield synth.random_small(s, max_rows=300, max_cols=24, max_groups=6)


# ---------------------------------------------------------------- golden file
def read_hand_positions():
    tiles, cases, cur = [], [], None
    with open(os.path.join(GOLDEN, "hand_positions.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            tok = line.split()
            if tok[0] == "tile":
                tiles.append(tuple(int(x) for x in tok[1:4]))
            elif tok[0] == "case":
                cur = {"name": tok[1], "dim": M if tok[2] == "M" else K, "rows": int(tok[3]),
                       "cols": int(tok[4]), "ends": [int(x) for x in tok[5].split(",")],
                       "at": [], "pad": [], "size": None}
                cases.append(cur)
            elif tok[0] == "at":
                cur["at"].append(tuple(int(x) for x in tok[1:4]))
            elif tok[0] == "pad":
                cur["pad"].append(int(tok[1]))
            elif tok[0] == "size":
                cur["size"] = (int(tok[1]), int(tok[2]))
    return tiles, cases


def read_page_rows():
    rows = []
    with open(os.path.join(GOLDEN, "page_k_groups_bandwidth.tsv")) as f:
        for line in f:
            if line.startswith("#") or line.startswith("source"):
                continue
            src, r, c, g, t, bw = line.rstrip("\n").split("\t")
            rows.append((src, int(r), int(c), int(g), float(t), float(bw)))
    return rows


# ---------------------------------------------------------------- pins
def _one_hot_dest(lib, dim, rows, cols, ends, i, j):
    S = np.zeros((rows, cols), dtype=np.uint8)
    S[i, j] = 7
    out = oracle.rearrange(dim, S, ends, lib=lib)
    nz = np.flatnonzero(out)
    assert len(nz) == 1, f"one-hot ({i},{j}) produced {len(nz)} non-zero bytes"
    return int(nz[0])


def pin_tile_golden(lib):
    tiles, _ = read_hand_positions()
    for dim, ends in ((M, [128]), (K, [4])):
        for r, c, byte in tiles:
            got = _one_hot_dest(lib, dim, 128, 4, ends, r, c)
            assert got == byte, f"dim {dim}: tile ({r},{c}) -> {got}, hand-worked {byte}"
            rr, cc = oracle.decode_at(dim, 128, 4, ends, [byte], lib=lib)
            assert (rr[0], cc[0]) == (r, c), f"decode {byte} -> ({rr[0]},{cc[0]})"


def pin_case_golden(lib):
    _, cases = read_hand_positions()
    rng = np.random.default_rng(5)
    for cs in cases:
        dim, rows, cols, ends = cs["dim"], cs["rows"], cs["cols"], cs["ends"]
        for i, j, byte in cs["at"]:
            got = _one_hot_dest(lib, dim, rows, cols, ends, i, j)
            assert got == byte, f"{cs['name']}: ({i},{j}) -> {got}, hand-worked {byte}"
            dest = oracle.dest_index(dim, rows, cols, ends, lib=lib)
            assert dest[i, j] == byte, f"{cs['name']}: dest_index ({i},{j}) -> {dest[i, j]}"
            rr, cc = oracle.decode_at(dim, rows, cols, ends, [byte], lib=lib)
            assert (rr[0], cc[0]) == (i, j), f"{cs['name']}: decode {byte} -> ({rr[0]},{cc[0]})"
        S = rng.integers(100, 141, size=(rows, cols), dtype=np.uint8)
        out = oracle.rearrange(dim, S, ends, lib=lib)
        for byte in cs["pad"]:
            assert out[byte] == 0, f"{cs['name']}: padding byte {byte} = {out[byte]}"
            rr, cc = oracle.decode_at(dim, rows, cols, ends, [byte], lib=lib)
            assert rr[0] == -1 and cc[0] == -1, f"{cs['name']}: pad byte {byte} decodes to ({rr[0]},{cc[0]})"
        alloc, written = cs["size"]
        assert oracle.rearranged_size(dim, rows, cols, len(ends), lib=lib) == alloc
        assert oracle.written_bytes(dim, rows, cols, ends, lib=lib) == written
        assert len(out) == alloc


def pin_word_transpose(lib):
    """One 128x4 tile is a 4x32 -> 32x4 transpose of 32-bit words: input row r
    (4 bytes) is word r; the tile's output words are that 4x32 word matrix
    transposed."""
    rng = np.random.default_rng(11)
    for dim, ends in ((M, [128]), (K, [4])):
        for _ in range(4):
            S = rng.integers(0, 256, size=(128, 4), dtype=np.uint8)
            out = oracle.rearrange(dim, S, ends, lib=lib)[:512]
            words_in = S.copy().view("<u4").reshape(4, 32)
            words_out = out.copy().view("<u4")
            assert np.array_equal(words_out, words_in.T.reshape(-1)), "tile is not a word transpose"


def pin_reshape_chain(lib):
    for case in tiny_cases():
        S = np.ascontiguousarray(case.scales)
        alloc = oracle.rearranged_size(case.dim, case.rows, case.cols, case.num_groups, lib=lib)
        want = brute_force(case.dim, S, case.ends, alloc)
        got = oracle.rearrange(case.dim, case.scales, case.ends, lib=lib)
        assert np.array_equal(got, want), f"{case.note}: scatter != reshape chain"


def pin_gather_vs_scatter(lib):
    for case in tiny_cases(60, 2000):
        a = oracle.rearrange(case.dim, case.scales, case.ends, lib=lib)
        b = oracle.gather(case.dim, case.scales, case.ends, lib=lib)
        assert np.array_equal(a, b), f"{case.note}: gather != scatter"


def pin_bijection(lib):
    """Tagged inputs (tag = i*cols + j + 1, four byte planes): every covered
    element's tag appears exactly once, at its destination, and every other
    output byte is 0."""
    for case in tiny_cases(60, 3000):
        rows, cols, ends, dim = case.rows, case.cols, case.ends, case.dim
        tags = (np.arange(rows * cols, dtype=np.uint32) + 1).reshape(rows, cols)
        planes = [oracle.rearrange(dim, np.ascontiguousarray(((tags >> (8 * p)) & 0xFF).astype(np.uint8)),
                                   ends, lib=lib) for p in range(4)]
        out = sum(planes[p].astype(np.uint32) << (8 * p) for p in range(4))
        dest = oracle.dest_index(dim, rows, cols, ends, lib=lib)
        covered = dest >= 0
        e = clamp_reference(ends, rows if dim == M else cols)
        used = int(e[-1]) if len(e) else 0
        if dim == M:
            expect_cov = np.zeros((rows, cols), bool)
            expect_cov[:used, :] = True
        else:
            expect_cov = np.zeros((rows, cols), bool)
            expect_cov[:, :used] = True
        assert np.array_equal(covered, expect_cov), f"{case.note}: coverage"
        nz = out[out != 0]
        assert len(nz) == covered.sum(), f"{case.note}: {len(nz)} tags placed for {covered.sum()} elements"
        assert len(np.unique(nz)) == len(nz), f"{case.note}: a tag appears twice"
        assert np.array_equal(np.sort(nz), np.sort(tags[covered])), f"{case.note}: tag set differs"
        assert np.array_equal(out[dest[covered]], tags[covered]), f"{case.note}: tag not at its destination"


def pin_round_trip(lib):
    for case in tiny_cases(60, 4000):
        S = np.ascontiguousarray(case.scales)
        out = oracle.rearrange(case.dim, case.scales, case.ends, lib=lib)
        back = oracle.inverse(case.dim, out, case.rows, case.cols, case.ends, lib=lib)
        dest = oracle.dest_index(case.dim, case.rows, case.cols, case.ends, lib=lib)
        want = np.where(dest >= 0, S, 0)
        assert np.array_equal(back, want), f"{case.note}: inverse does not round-trip"


def pin_clamp(lib):
    rng = np.random.default_rng(21)
    for _ in range(300):
        G = int(rng.integers(1, 65))
        T = int(rng.integers(0, 1000))
        ends = rng.integers(-50, 1100, size=G).astype(np.int32)
        got = oracle.clamp_ends(ends, T, lib=lib)
        assert np.array_equal(got, clamp_reference(ends, T)), "clamp != running-max closed form"


def pin_sizes(lib):
    # closed forms evaluated by hand
    # 44 columns are already whole 4-column tiles; 45 pad to 48
    assert oracle.rearranged_size(M, 1000, 44, 4, lib=lib) == (1000 + 512) * 44
    assert oracle.rearranged_size(M, 1000, 45, 4, lib=lib) == (1000 + 512) * 48
    assert oracle.rearranged_size(M, 0, 44, 4, lib=lib) == 512 * 44
    assert oracle.rearranged_size(M, 5, 1, 1, lib=lib) == 133 * 4
    assert oracle.rearranged_size(K, 7168, 4096, 8, lib=lib) == 7168 * 4128
    assert oracle.rearranged_size(K, 0, 10, 3, lib=lib) == 0
    assert oracle.rearranged_size(K, 1, 1, 1, lib=lib) == 128 * 5
    assert oracle.rearranged_size(M, 1, 1, 0, lib=lib) == -1
    assert oracle.rearranged_size(M, 1, 1, 65, lib=lib) == -1
    # the allocation bounds the exact padded output for every split
    rng = np.random.default_rng(31)
    for _ in range(400):
        dim = int(rng.integers(0, 2))
        rows, cols, G = int(rng.integers(0, 2000)), int(rng.integers(1, 600)), int(rng.integers(1, 65))
        T = rows if dim == M else cols
        ends = np.sort(rng.integers(0, T + 1, size=G)).astype(np.int32)
        w = oracle.written_bytes(dim, rows, cols, ends, lib=lib)
        assert 0 <= w <= oracle.rearranged_size(dim, rows, cols, G, lib=lib)
        # exact padded bytes from the clamped sizes, summed directly
        e = clamp_reference(ends, T)
        sizes = np.diff(np.concatenate([[0], e]))
        if dim == M:
            want = sum(ceil_to(int(n), 128) for n in sizes) * ceil_to(cols, 4)
        else:
            want = ceil_to(rows, 128) * sum(ceil_to(int(n), 4) for n in sizes)
        assert w == want
        assert oracle.read_bytes(dim, rows, cols, ends, lib=lib) == (int(e[-1]) * cols if dim == M else rows * int(e[-1]))


def pin_page_tables(lib):
    """Every K-groups row of the #3604 and #4704 tables satisfies
    GB/s = (rows*cols + allocation) / time within 1.5%; a 3*G column slack
    instead of 4*G misses some rows by more than 8%."""
    worst = 0.0
    for src, rows, cols, G, t_us, gbps in read_page_rows():
        alloc = oracle.rearranged_size(K, rows, cols, G, lib=lib)
        pred = (rows * cols + alloc) / (t_us * 1e-6) / 1e9
        worst = max(worst, abs(pred - gbps) / gbps)
    assert worst < 0.015, f"allocation disagrees with the page tables by {worst:.3%}"


def pin_single_group_m_equals_k(lib):
    rng = np.random.default_rng(41)
    for rows in (128, 256, 384):
        for cols in (4, 8, 20):
            S = rng.integers(0, 256, size=(rows, cols), dtype=np.uint8)
            a = oracle.rearrange(M, S, [rows], lib=lib)[: rows * cols]
            b = oracle.rearrange(K, S, [cols], lib=lib)[: rows * cols]
            assert np.array_equal(a, b), "M and K disagree on one aligned group"
            assert np.array_equal(a, blocked_reference(S)), "single group != blocked matrix"


def pin_group_decomposition(lib):
    """A G-group output is the concatenation of each group's one-group output."""
    for case in tiny_cases(40, 5000):
        S = np.ascontiguousarray(case.scales)
        rows, cols, dim = case.rows, case.cols, case.dim
        full = oracle.rearrange(dim, S, case.ends, lib=lib)
        e = clamp_reference(case.ends, rows if dim == M else cols)
        parts, begin = [], 0
        for end in e:
            end = int(end)
            if dim == M:
                sub = np.ascontiguousarray(S[begin:end, :])
                one = oracle.rearrange(M, sub, [end - begin], lib=lib)
                parts.append(one[: ceil_to(end - begin, 128) * ceil_to(cols, 4)])
            else:
                sub = np.ascontiguousarray(S[:, begin:end])
                one = oracle.rearrange(K, sub, [end - begin], lib=lib) if end > begin else np.zeros(0, np.uint8)
                parts.append(one[: ceil_to(rows, 128) * ceil_to(end - begin, 4)])
            begin = end
        flat = np.concatenate(parts)
        assert np.array_equal(full[: len(flat)], flat), f"{case.note}: not a concatenation of groups"
        assert not full[len(flat):].any(), f"{case.note}: allocation tail not zero"


ALL_PINS = [
    pin_tile_golden, pin_case_golden, pin_word_transpose, pin_reshape_chain, pin_gather_vs_scatter,
    pin_bijection, pin_round_trip, pin_clamp, pin_sizes, pin_page_tables,
    pin_single_group_m_equals_k, pin_group_decomposition,
]


def main(argv):
    lib = oracle.load(argv[1]) if len(argv) > 1 else oracle.load()
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except AssertionError as exc:
            failed.append(f"{pin.__name__}: {exc}")
    for f in failed:
        print("FAILED", f)
    return 1 if failed else 0


if __name__ == "__main__":
    sys.exit(main(sys.argv))
