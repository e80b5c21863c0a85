"""Pins of the oracle's ablation variants and operating point.

"Prism: Dynamic Sparse Attention for Native 2K Joint Video-Audio Generation
Model Training": Table 10 (page xyznot.com/id) varies the exponent alpha of
the shape mapping b_d ~ g_d^-alpha (1/3, 1/2, 2), compares an isotropic
mapping and the fixed-block baseline; page paper.rainbus.top gives the
operating point "Top-k 95%, Top-p 0.2" (k as a sparsity: 5% of the blocks).
Each check below is pinned to something other than the oracle's own formula:
hand-worked closed forms, the proportionality and volume constraints, the tie
rule of the snapping, exact integer ceilings and brute-force selection.
"""

import numpy as np
import pytest

from oracle import prism_oracle as po

F32 = np.float32


@pytest.mark.parametrize("alpha,g,vol,want", [
    # l* = -alpha log2 g + (S + alpha sum log2 g) / 3, worked by hand
    (2.0, (1.0, 4.0, 16.0), 64, (6.0, 2.0, -2.0)),
    (1.0 / 3.0, (1.0, 4.0, 16.0), 64, (8.0 / 3.0, 2.0, 4.0 / 3.0)),
    (0.5, (1.0, 4.0, 16.0), 64, (3.0, 2.0, 1.0)),
    (2.0, (2.0, 2.0, 2.0), 128, (7.0 / 3.0, 7.0 / 3.0, 7.0 / 3.0)),
])
def test_alpha_closed_form_worked_examples(alpha, g, vol, want):
    ell = po.ideal_log_edges(np.array(g, dtype=F32), F32(vol), alpha)
    np.testing.assert_allclose(ell, want, atol=2e-6)


@pytest.mark.parametrize("alpha", [1.0 / 3.0, 0.5, 2.0])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_alpha_proportionality_and_volume(alpha, seed):
    """sum l* = log2 B and l*_d + alpha log2 g_d is the same on every axis
    (b_d g_d^alpha constant: the mapping b_d ~ g_d^-alpha with prod b_d = B)."""
    rng = np.random.default_rng(seed)
    g = rng.uniform(1e-4, 1.0, size=(200, 3)).astype(F32)
    for vol in (64, 128, 256):
        ell = po.ideal_log_edges(g, F32(vol), alpha).astype(np.float64)
        np.testing.assert_allclose(ell.sum(axis=1), np.log2(vol), atol=5e-5)
        c = ell + alpha * np.log2(g.astype(np.float64))
        np.testing.assert_allclose(c - c[:, :1], 0.0, atol=5e-5)


def test_alpha_half_is_the_method():
    rng = np.random.default_rng(5)
    g = rng.uniform(1e-4, 1.0, size=(100, 3)).astype(F32)
    for vol in (64, 128, 256):
        np.testing.assert_array_equal(po.ideal_log_edges(g, F32(vol)), po.ideal_log_edges(g, F32(vol), 0.5))


def test_larger_alpha_is_more_anisotropic():
    """With one axis twice as dynamic, alpha = 1/3 keeps the cube, 2 stretches it."""
    g = np.array([0.5, 0.25, 0.25], dtype=F32)
    lo = po.SHAPES[po.snap(po.ideal_log_edges(g, F32(64), 1.0 / 3.0), 64)]
    hi = po.SHAPES[po.snap(po.ideal_log_edges(g, F32(64), 2.0), 64)]
    assert lo == (4, 4, 4)
    assert hi[0] == 2 and hi[0] < min(hi[1], hi[2])


def _field(seed, T=16, H=16, W=24, D=8):
    rng = np.random.default_rng(seed)
    V = rng.standard_normal((T * H * W, D))
    # a few zones with structure so that the volumes differ
    V[: 512 * 2] *= 3.0
    a = rng.uniform(0.05, 1.0, size=(T, H, W)).astype(np.float32)
    return V, a, T, H, W


def test_isotropic_mode_takes_the_cube_of_each_volume():
    """g equal on the axes: l* = log2(B)/3; the nearest candidates tie three ways
    at B = 128 and 256 and the lower index wins: 4x4x4, 4x4x8, 4x8x8."""
    V, a, T, H, W = _field(1)
    st = po.zone_shapes(V, a, T, H, W, 1e-4, shape_mode=po.SHAPE_ISOTROPIC)
    cube = {64: (4, 4, 4), 128: (4, 4, 8), 256: (4, 8, 8)}
    assert len(set(st["B"].tolist())) >= 2
    for sid, B in zip(st["shape_id"], st["B"]):
        assert po.SHAPES[int(sid)] == cube[int(B)]
    # the volumes are the method's: isotropy only changes the shape
    ref = po.zone_shapes(V, a, T, H, W, 1e-4)
    np.testing.assert_array_equal(st["B"], ref["B"])


@pytest.mark.parametrize("fixed", [3, 8, 13, 0])
def test_fixed_mode_partitions_every_zone_alike(fixed):
    V, a, T, H, W = _field(2)
    st = po.zone_shapes(V, a, T, H, W, 1e-4, shape_mode=po.SHAPE_FIXED, fixed_shape=fixed)
    vol = int(np.prod(po.SHAPES[fixed]))
    assert (st["shape_id"] == fixed).all() and (st["B"] == vol).all()
    src, starts = po.partition(st["shape_id"], T, H, W)
    nz = (T // 8) * (H // 8) * (W // 8)
    assert len(starts) - 1 == nz * (512 // vol)
    assert (np.diff(starts) == vol).all()
    np.testing.assert_array_equal(np.sort(src), np.arange(T * H * W))


@pytest.mark.parametrize("frac,nb,want", [
    (0.05, 8, 1), (0.05, 20, 1), (0.05, 21, 2), (0.05, 4300, 215), (0.05, 4336, 217),
    (1.0, 37, 37), (0.5, 7, 4), (0.25, 1024, 256),
])
def test_k_of_fraction_is_the_ceiling(frac, nb, want):
    assert po.k_of_fraction(frac, nb) == want


def test_k_of_fraction_bounds():
    """ceil(frac * N_b) in fp32 equals the exact ceiling or one more, the latter
    only when frac * N_b lies within fp32 rounding of an integer."""
    for frac in (0.05, 0.1, 0.2, 1.0 / 3.0):
        for nb in range(1, 3000):
            k = po.k_of_fraction(frac, nb)
            exact = frac * nb
            assert k >= exact - 1e-9 and k <= exact + 1
            if abs(exact - round(exact)) > 1e-3:
                assert k == int(np.ceil(exact))


@pytest.mark.parametrize("seed", [0, 1])
def test_fractional_k_selection_bruteforce(seed):
    """k = ceil(frac N_b) with p = 0: every row keeps exactly its k most probable
    blocks (ties to the lower index), checked against an exhaustive ranking."""
    rng = np.random.default_rng(seed)
    nb, D = 23, 6
    Qb, Kb = rng.standard_normal((nb, D)), rng.standard_normal((nb, D))
    for frac in (0.05, 0.2, 0.5):
        sel, _, P = po.select(Qb, Kb, 0, 0.0, k_frac=frac)
        k = po.k_of_fraction(frac, nb)
        for i in range(nb):
            ranked = sorted(range(nb), key=lambda j: (-float(P[i, j]), j))
            assert sorted(ranked[:k]) == list(sel[i])


def test_operating_point_union_with_top_p():
    """The pages' point (5% of the blocks, p = 0.2): the set is the first
    max(k, L) of the order, L the shortest prefix with mass >= p."""
    rng = np.random.default_rng(7)
    nb, D = 40, 8
    Qb, Kb = 2.0 * rng.standard_normal((nb, D)), 2.0 * rng.standard_normal((nb, D))
    sel, _, P = po.select(Qb, Kb, 0, 0.2, k_frac=0.05)
    k = po.k_of_fraction(0.05, nb)
    for i in range(nb):
        order = sorted(range(nb), key=lambda j: (-float(P[i, j]), j))
        cum = np.cumsum(P[i, order], dtype=np.float32)      # sequential fp32 prefix sums
        L = next(l for l in range(1, nb + 1) if cum[l - 1] >= np.float32(0.2))
        assert len(sel[i]) == max(k, L)
        assert set(sel[i]) == set(order[:max(k, L)])


def test_all_blocks_with_fraction_one():
    rng = np.random.default_rng(3)
    Qb, Kb = rng.standard_normal((9, 4)), rng.standard_normal((9, 4))
    sel, _, _ = po.select(Qb, Kb, 0, 0.0, k_frac=1.0)
    assert all(list(s) == list(range(9)) for s in sel)
