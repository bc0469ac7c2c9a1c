"""The seeded generators produce the stated workload shapes and group splits."""
import numpy as np

from scale_factor_layout_b200 import synth


def test_m_tiny():
    c = synth.m_tiny()
    assert c.scales.shape == (1000, 44) and c.dim == synth.DIM_M and c.num_groups == 4
    sizes = np.diff(np.concatenate([[0], c.ends]))
    assert c.ends[-1] == 1000 and (sizes == 0).sum() == 1 and (sizes >= 0).all()
    assert c.scales.min() >= 110 and c.scales.max() <= 135


def test_m_skinny_and_wide():
    s = synth.m_skinny()
    assert s.scales.shape == (131072, 44) and s.row_stride == 44 and s.ends[-1] == 131072 and s.num_groups == 8
    w = synth.m_wide()
    sizes = np.diff(np.concatenate([[0], w.ends]))
    assert w.scales.shape == (131072, 224) and w.ends[-1] == 131072 and (sizes % 32 == 0).all()
    assert w.scales.min() >= 100 and w.scales.max() <= 140


def test_k_groups_and_sweep():
    k = synth.k_groups()
    sizes = np.diff(np.concatenate([[0], k.ends]))
    assert k.scales.shape == (7168, 4096) and k.ends[-1] == 4096 and (sizes >= 1).all()
    pts = synth.sweep_points()
    assert len(pts) == 70
    p = synth.k_sweep_point(0, 0)
    assert p.scales.shape == (128, 32) and p.ends[-1] == 32 and p.num_groups == 8


def test_determinism_and_strided():
    a, b = synth.m_tiny(), synth.m_tiny()
    assert np.array_equal(a.scales, b.scales) and np.array_equal(a.ends, b.ends)
    s = synth.strided(a, 5)
    assert s.row_stride == 49 and s.scales.shape == (1000, 44)
    base = np.lib.stride_tricks.as_strided(s.scales, shape=(1000, 49), strides=(49, 1))
    assert (base[:-1, 44:] == 0xFF).all()


def test_random_small_valid():
    for seed in range(200):
        c = synth.random_small(seed)
        total = c.rows if c.dim == synth.DIM_M else c.cols
        assert 1 <= c.num_groups <= 64
        assert (np.diff(np.concatenate([[0], c.ends])) >= 0).all() and c.ends[-1] <= total
