"""Seeded synthetic inputs: E8M0 scale tensors and group end offsets.

This module draws random numbers and nothing else: it holds none of the
layout's arithmetic, so the CUDA path and the CPU oracle can both be fed from
it.  Shapes follow the workloads of the pytorch/ao pages on MXFP8 MoE
training: the (131072, 44) M-groups case of "fallback cuda kernel for when
input doesn't meet 2d TMA constraints" (Benchmarks), the (7168, 4096)
K-groups case of "add bench script for scale conversion to blocked format
kernels for groups along K", and the M x TotalK powers-of-two sweep of "Add
CuTeDSL MXFP8 K-groups scale rearrange kernel".  Scale bytes are drawn
uniformly from a narrow band around the E8M0 bias (127), which is where the
exponents of unit-variance data land; the layout's cost does not depend on the
values.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

DIM_M = 0
DIM_K = 1

SEED_BASE = 0x5CA1E000
SWEEP_SEED_BASE = 0x5CA1E100
SWEEP_ROWS = (128, 1024, 2048, 4096, 8192, 16384, 28672)
SWEEP_TOTAL_K = tuple(2 ** p for p in range(10, 20))
BLOCK_SIZE = 32  # data elements per E8M0 scale


@dataclass
class Case:
    name: str
    dim: int                    # DIM_M or DIM_K
    scales: np.ndarray          # (rows, cols) uint8 view; rows may be strided
    ends: np.ndarray            # (G,) int32 cumulative group end offsets
    seed: int
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def rows(self) -> int:
        return self.scales.shape[0]

    @property
    def cols(self) -> int:
        return self.scales.shape[1]

    @property
    def row_stride(self) -> int:
        return self.scales.strides[0]

    @property
    def num_groups(self) -> int:
        return len(self.ends)


def uniform_scales(rng: np.random.Generator, rows: int, cols: int, lo: int, hi: int,
                   row_stride: int | None = None, gap_fill: int = 0xFF) -> np.ndarray:
    """(rows, cols) uint8 with values in [lo, hi].  With ``row_stride > cols``
    the bytes between rows hold ``gap_fill`` (a sentinel no real value uses)."""
    stride = cols if row_stride is None else row_stride
    assert stride >= cols
    if stride == cols:
        return rng.integers(lo, hi + 1, size=(rows, cols), dtype=np.uint8)
    buf = np.full((rows, stride), gap_fill, dtype=np.uint8)
    buf[:, :cols] = rng.integers(lo, hi + 1, size=(rows, cols), dtype=np.uint8)
    return buf[:, :cols]


def ends_from_sizes(sizes) -> np.ndarray:
    return np.cumsum(np.asarray(sizes, dtype=np.int64)).astype(np.int32)


def split_distinct_cuts(rng: np.random.Generator, total: int, groups: int) -> np.ndarray:
    """Sizes >= 1 summing to ``total``: groups-1 distinct sorted cut points in [1, total-1]."""
    assert total >= groups
    cuts = np.sort(rng.choice(np.arange(1, total), size=groups - 1, replace=False))
    edges = np.concatenate([[0], cuts, [total]])
    return np.diff(edges)


def split_multinomial(rng: np.random.Generator, total: int, groups: int) -> np.ndarray:
    """Sizes from ``total`` independent uniform draws of a group index."""
    return np.bincount(rng.integers(0, groups, size=total), minlength=groups)


def split_units(rng: np.random.Generator, total: int, groups: int, unit: int) -> np.ndarray:
    """Sizes that are multiples of ``unit``: total/unit units split by groups-1
    sorted uniform cut points (zero-size groups allowed if drawn)."""
    assert total % unit == 0
    n = total // unit
    cuts = np.sort(rng.integers(0, n + 1, size=groups - 1))
    edges = np.concatenate([[0], cuts, [n]])
    return np.diff(edges) * unit


def m_tiny(seed: int = SEED_BASE + 0) -> Case:
    """(1000, 44) M-groups, G=4, one empty group; output pads 44 -> 48 columns."""
    rng = np.random.default_rng(seed)
    s = uniform_scales(rng, 1000, 44, 110, 135)
    nonzero = split_distinct_cuts(rng, 1000, 3)
    empty_at = int(rng.integers(0, 4))
    sizes = np.insert(nonzero, empty_at, 0)
    return Case("m_tiny", DIM_M, s, ends_from_sizes(sizes), seed,
                "M-groups (1000, 44), G=4 with one empty group")


def m_skinny(seed: int = SEED_BASE + 1) -> Case:
    """(131072, 44) M-groups, row stride 44 B (not a multiple of 16 B), G=8."""
    rng = np.random.default_rng(seed)
    s = uniform_scales(rng, 131072, 44, 100, 140)
    sizes = split_multinomial(rng, 131072, 8)
    return Case("m_skinny", DIM_M, s, ends_from_sizes(sizes), seed,
                "M-groups (131072, 44), stride 44 B, G=8 multinomial split")


def m_wide(seed: int = SEED_BASE + 2) -> Case:
    """(131072, 224) M-groups (data K = 7168), G=8, sizes multiples of 32."""
    rng = np.random.default_rng(seed)
    s = uniform_scales(rng, 131072, 224, 100, 140)
    sizes = split_units(rng, 131072, 8, 32)
    return Case("m_wide", DIM_M, s, ends_from_sizes(sizes), seed,
                "M-groups (131072, 224), G=8, sizes multiples of 32")


def k_groups(seed: int = SEED_BASE + 3) -> Case:
    """(7168, 4096) K-groups (data K = 131072), G=8, column widths >= 1."""
    rng = np.random.default_rng(seed)
    s = uniform_scales(rng, 7168, 4096, 100, 140)
    sizes = split_distinct_cuts(rng, 4096, 8)
    return Case("k_groups", DIM_K, s, ends_from_sizes(sizes), seed,
                "K-groups (7168, 4096), G=8, widths >= 1")


def k_sweep_point(i_rows: int, i_k: int) -> Case:
    """One point of the M x TotalK sweep: scales (M, TotalK/32), G=8."""
    rows = SWEEP_ROWS[i_rows]
    total_k = SWEEP_TOTAL_K[i_k]
    cols = total_k // BLOCK_SIZE
    seed = SWEEP_SEED_BASE + 16 * i_rows + i_k
    rng = np.random.default_rng(seed)
    s = uniform_scales(rng, rows, cols, 100, 140)
    sizes = split_distinct_cuts(rng, cols, 8)
    return Case(f"k_sweep_{rows}x{total_k}", DIM_K, s, ends_from_sizes(sizes), seed,
                f"K-groups sweep M={rows} TotalK={total_k}", {"M": rows, "TotalK": total_k})


def sweep_points():
    return [(i, j) for i in range(len(SWEEP_ROWS)) for j in range(len(SWEEP_TOTAL_K))]


NAMED = {"m_tiny": m_tiny, "m_skinny": m_skinny, "m_wide": m_wide, "k_groups": k_groups}


def strided(case: Case, pad: int, seed_offset: int = 0x77) -> Case:
    """The same shape and groups with ``row_stride = cols + pad`` and fresh values;
    the gap bytes are 0xFF."""
    rng = np.random.default_rng(case.seed + seed_offset)
    s = uniform_scales(rng, case.rows, case.cols, 100, 140, row_stride=case.cols + pad)
    return Case(case.name + f"_stride+{pad}", case.dim, s, case.ends.copy(), case.seed + seed_offset,
                case.note + f", row stride cols+{pad}")


def random_small(seed: int, max_rows: int = 700, max_cols: int = 300, max_groups: int = 64) -> Case:
    """A small random case for sweeps: any dim, shape, stride, group count,
    empty groups (including first and last), offsets that may stop short."""
    rng = np.random.default_rng(seed)
    dim = int(rng.integers(0, 2))
    rows = int(rng.integers(0, max_rows + 1))
    cols = int(rng.integers(1, max_cols + 1))
    G = int(rng.integers(1, max_groups + 1))
    stride_kind = int(rng.integers(0, 3))
    if stride_kind == 0:
        stride = cols
    elif stride_kind == 1:
        stride = cols + int(rng.integers(1, 38))
    else:
        stride = (cols + 15) // 16 * 16
    s = uniform_scales(rng, max(rows, 0), cols, 100, 140, row_stride=max(stride, cols))
    total = rows if dim == DIM_M else cols
    # sizes: a mix of empty and non-empty groups; sometimes stop short of total
    weights = rng.random(G) * (rng.random(G) < 0.7)
    used = total if rng.random() < 0.8 else int(rng.integers(0, total + 1))
    if weights.sum() == 0 or used == 0:
        sizes = np.zeros(G, dtype=np.int64)
        if used > 0:
            sizes[int(rng.integers(0, G))] = used
    else:
        raw = np.floor(weights / weights.sum() * used).astype(np.int64)
        raw[int(np.argmax(weights))] += used - raw.sum()
        sizes = raw
    return Case(f"random_{seed}", dim, s, ends_from_sizes(sizes), seed,
                f"random small dim={dim} rows={rows} cols={cols} stride={stride} G={G}")
