"""Pins of the oracle's block scores, tie margins and statistics readings.

Each check compares the oracle with something other than itself: hand-worked
softmax values (tests/golden/block_scores.json, page xyznot.com/id, section
"Metode" 3), torch's float64 softmax, a brute-force ranking of an
independently computed P, sorted candidate distances written out here, and
closed-form values of the statistics on hand-built fields.  Every check is a
function of the oracle routine it pins, so the planted-mistake tests below can
run it on a mutated copy (the mistake is planted in the oracle, on the CPU)
and show that it fails.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import prism_oracle as po

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------ block scores
def check_block_probs(fn):
    """P_i = softmax_j(Qbar_i . Kbar_j / sqrt(D)) over the key blocks."""
    gold = json.load(open(os.path.join(GOLD, "block_scores.json")))
    for case in gold["cases"]:
        Qb = np.array(case["Qbar"], dtype=np.float64)
        Kb = np.array(case["Kbar"], dtype=np.float64)
        s, P = fn(Qb, Kb)
        np.testing.assert_allclose(s, case["logits"], atol=1e-6, err_msg=case["name"])
        np.testing.assert_allclose(P, case["P"], atol=1e-6, err_msg=case["name"])
    rng = np.random.default_rng(41)
    for D in (16, 64, 128):
        Qb = rng.normal(size=(9, D))
        Kb = rng.normal(size=(23, D)) * 0.7
        s, P = fn(Qb, Kb)
        ref = torch.softmax(torch.tensor(Qb) @ torch.tensor(Kb).T / np.sqrt(D), dim=1).numpy()
        np.testing.assert_allclose(P, ref, rtol=2e-6, atol=1e-9)
        np.testing.assert_allclose(np.asarray(P, np.float64).sum(axis=1), 1.0, atol=1e-5)


def test_block_probs_pinned():
    check_block_probs(po.block_probs)


def _no_scale(Qb, Kb):
    s = (np.asarray(Qb, np.float64) @ np.asarray(Kb, np.float64).T).astype(np.float32)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return s, (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def _scale_by_d(Qb, Kb):
    D = Qb.shape[1]
    s = (np.asarray(Qb, np.float64) @ np.asarray(Kb, np.float64).T / D).astype(np.float32)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return s, (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def _softmax_over_queries(Qb, Kb):
    D = Qb.shape[1]
    s = (np.asarray(Qb, np.float64) @ np.asarray(Kb, np.float64).T / np.sqrt(D)).astype(np.float32)
    e = np.exp(s - s.max(axis=0, keepdims=True))
    return s, (e / e.sum(axis=0, keepdims=True)).astype(np.float32)


def _unnormalised(Qb, Kb):
    D = Qb.shape[1]
    s = (np.asarray(Qb, np.float64) @ np.asarray(Kb, np.float64).T / np.sqrt(D)).astype(np.float32)
    return s, np.exp(s - s.max(axis=1, keepdims=True)).astype(np.float32)


@pytest.mark.parametrize("mutant", [_no_scale, _scale_by_d, _softmax_over_queries, _unnormalised])
def test_planted_block_prob_mistakes_are_caught(mutant):
    with pytest.raises(AssertionError):
        check_block_probs(mutant)


def _ranked_set(P64, k, p):
    """The first max(k, L) blocks of (P desc, j asc); L = shortest prefix with mass >= p."""
    nb = len(P64)
    order = sorted(range(nb), key=lambda j: (-P64[j], j))
    if p >= 1.0:
        L = nb
    elif p <= 0.0:
        L = 0
    else:
        acc, L = 0.0, nb
        for n, j in enumerate(order):
            acc += P64[j]
            if acc >= p:
                L = n + 1
                break
    return sorted(order[:max(min(k, nb), L)]), order


@pytest.mark.parametrize("seed", range(6))
def test_selection_from_independent_block_scores(seed):
    """po.select's sets equal the brute-force ranking of a P computed here with
    torch in float64 (near-ties of the Top-p threshold or of P excepted)."""
    rng = np.random.default_rng(500 + seed)
    D = int(rng.choice([16, 64, 128]))
    nq, nb = 7, int(rng.integers(6, 40))
    Qb = rng.normal(size=(nq, D)) * rng.uniform(0.2, 2.0)
    Kb = rng.normal(size=(nb, D))
    P64 = torch.softmax(torch.tensor(Qb) @ torch.tensor(Kb).T / np.sqrt(D), dim=1).numpy()
    checked = 0
    for k in (1, 3, nb + 5):
        for p in (0.0, 0.3, 0.8, 0.95, 1.0):
            sel, _, _ = po.select(Qb, Kb, k, p)
            for i in range(nq):
                want, order = _ranked_set(P64[i], k, p)
                cum = np.cumsum(P64[i][order])
                if 0 < p < 1 and np.min(np.abs(cum - p)) < 1e-5:
                    continue
                srt = np.sort(P64[i])[::-1]
                if np.min(np.abs(np.diff(srt))) < 1e-6:
                    continue
                assert sel[i].tolist() == want, (seed, k, p, i)
                checked += 1
    assert checked > 50


# ------------------------------------------------------------- snap margin
def _sorted_candidate_distances(ell, vol):
    """Squared log2 distances to every candidate of volume vol, written out."""
    out = []
    for bt, bh, bw in po.SHAPES:
        if bt * bh * bw != vol:
            continue
        lb = (np.log2(bt), np.log2(bh), np.log2(bw))
        out.append(sum((lb[d] - float(ell[d])) ** 2 for d in range(3)))
    return sorted(out)


def check_snap_margin(fn):
    # l* on a candidate: the nearest is at 0, the next at 2 (two unit steps)
    assert fn(np.array([2.0, 2.0, 2.0]), 64) == pytest.approx(2.0, abs=1e-12)
    assert fn(np.array([1.0, 2.0, 3.0]), 64) == pytest.approx(2.0, abs=1e-12)
    assert fn(np.array([2.0, 3.0, 3.0]), 256) == pytest.approx(2.0, abs=1e-12)
    # isotropic g at B = 128: three candidates at 6/9 -> an exact tie
    assert abs(fn(np.full(3, 7.0 / 3.0), 128)) < 1e-12
    # halfway between 4x4x4 and 4x2x8: both at 0.5
    assert abs(fn(np.array([2.0, 1.5, 2.5]), 64)) < 1e-12
    rng = np.random.default_rng(77)
    for _ in range(200):
        vol = int(rng.choice([64, 128, 256]))
        ell = rng.uniform(0.5, 3.5, size=3)
        ds = _sorted_candidate_distances(ell, vol)
        assert fn(ell, vol) == pytest.approx(ds[1] - ds[0], abs=1e-12)


def test_snap_margin_pinned():
    check_snap_margin(po.snap_margin)


def _margin_zero(ell, vol):
    return 0.0


def _margin_best(ell, vol):
    return _sorted_candidate_distances(ell, vol)[0]


def _margin_third(ell, vol):
    ds = _sorted_candidate_distances(ell, vol)
    return ds[2] - ds[0]


def _margin_euclid(ell, vol):
    ds = np.sqrt(_sorted_candidate_distances(ell, vol))
    return ds[1] - ds[0]


@pytest.mark.parametrize("mutant", [_margin_zero, _margin_best, _margin_third, _margin_euclid])
def test_planted_snap_margin_mistakes_are_caught(mutant):
    with pytest.raises(AssertionError):
        check_snap_margin(mutant)


# --------------------------------------------- density, volume, rho margin
def _channel_ramp_field(D, ramps_per_zone):
    """8x8x(8 * zones) grid, zone z carries V = h (the local h index) on its
    first ramps_per_zone[z] channels and zero elsewhere: density_raw = 5.25 *
    ramps / D (the variance of 0..7 over a frame is 63/12, no frame change)."""
    nz = len(ramps_per_zone)
    T, H, W = 8, 8, 8 * nz
    V = np.zeros((T, H, W, D))
    h = np.arange(H)[None, :, None]
    for z, n in enumerate(ramps_per_zone):
        for c in range(n):
            V[:, :, 8 * z:8 * z + 8, c] = h
    return V.reshape(-1, D), T, H, W


def check_rho_margin(fn):
    rho = np.array([0.0, 0.25, 0.375, 0.5, 1.0])
    np.testing.assert_allclose(fn(rho, 0.5, 0.25), [0.25, 0.0, 0.125, 0.0, 0.5], atol=1e-15)
    # thresholds of the workloads (tau128 0.5, tau256 0.25) met exactly by
    # constructed zones: densities 1, 1/2, 1/4, 3/8 of the maximum
    V, T, H, W = _channel_ramp_field(8, [8, 4, 2, 3])
    st = po.zone_shapes(V, None, T, H, W, eps=1e-4)
    np.testing.assert_array_equal(st["rho"], np.float32([1.0, 0.5, 0.25, 0.375]))
    np.testing.assert_allclose(fn(po.normalise_by_max(po.density_raw(po.zones_of(V, T, H, W))), 0.5, 0.25),
                               [0.5, 0.0, 0.0, 0.125], atol=1e-15)


def test_rho_margin_pinned():
    check_rho_margin(po.rho_margin_of)


def test_volume_rule_is_strict_at_the_thresholds():
    """B = 256 below tau256, 128 below tau128, else 64: rho = 0.5 gives 64 and
    rho = 0.25 gives 128 (strict '<' at each threshold)."""
    V, T, H, W = _channel_ramp_field(8, [8, 4, 2, 3, 1])
    st = po.zone_shapes(V, None, T, H, W, eps=1e-4)
    np.testing.assert_array_equal(st["B"], [64, 64, 128, 128, 256])


@pytest.mark.parametrize("mutant", [
    lambda r, a, b: np.zeros_like(np.asarray(r, np.float64)),
    lambda r, a, b: np.abs(np.asarray(r, np.float64) - a),
    lambda r, a, b: np.minimum(np.asarray(r, np.float64) - a, np.asarray(r, np.float64) - b),
])
def test_planted_rho_margin_mistakes_are_caught(mutant):
    with pytest.raises(AssertionError):
        check_rho_margin(mutant)


# ------------------------------------------- closed forms of the readings
def _zone(fn_of_thw, D=2):
    t, h, w = np.meshgrid(np.arange(8), np.arange(8), np.arange(8), indexing="ij")
    v = fn_of_thw(t.astype(float), h.astype(float), w.astype(float))
    return np.repeat(v[..., None], D, axis=-1)[None]            # [1, 8, 8, 8, D]


def check_density(fn):
    """rho_raw = mean over frames of the frame's spatial variance + variance of
    the frame differences, closed forms: 63/12 for a ramp in h, 2 * 63/12 for
    h + w, 0 for a ramp in t (every difference is 1), 192/49 for (-1)^t (the
    differences are -2, 2, -2, 2, -2, 2, -2), 0 for a constant."""
    cases = [
        (lambda t, h, w: h, 63 / 12),
        (lambda t, h, w: h + w, 2 * 63 / 12),
        (lambda t, h, w: 3 * t, 0.0),
        (lambda t, h, w: (-1.0) ** t, 192 / 49),
        (lambda t, h, w: h + (-1.0) ** t, 63 / 12 + 192 / 49),
        (lambda t, h, w: 0 * t + 5.0, 0.0),
    ]
    for f, want in cases:
        assert fn(_zone(f))[0] == pytest.approx(want, rel=1e-12, abs=1e-12)


def test_density_reading_closed_forms():
    check_density(po.density_raw)


def _density_spatial_only(Vz):
    return np.asarray(Vz, np.float64).var(axis=(2, 3)).mean(axis=1).mean(axis=-1)


def _density_mean_square_differences(Vz):
    Vz = np.asarray(Vz, np.float64)
    spatial = Vz.var(axis=(2, 3)).mean(axis=1)
    diff = Vz[:, 1:] - Vz[:, :-1]
    return (spatial + (diff ** 2).mean(axis=(1, 2, 3))).mean(axis=-1)


@pytest.mark.parametrize("mutant", [_density_spatial_only, _density_mean_square_differences])
def test_planted_density_mistakes_are_caught(mutant):
    with pytest.raises(AssertionError):
        check_density(mutant)


def test_directional_variance_closed_forms():
    """Profiles along d are plane means: a ramp along one axis has variance
    63/12 along that axis and none along the others."""
    np.testing.assert_allclose(po.directional_variance(_zone(lambda t, h, w: t))[0], [63 / 12, 0, 0],
                               atol=1e-12)
    np.testing.assert_allclose(po.directional_variance(_zone(lambda t, h, w: 2 * h))[0], [0, 4 * 63 / 12, 0],
                               atol=1e-12)
    np.testing.assert_allclose(po.directional_variance(_zone(lambda t, h, w: h * w))[0],
                               [0, 3.5 ** 2 * 63 / 12, 3.5 ** 2 * 63 / 12], atol=1e-9)


def check_audio(fn):
    """Zone 0 carries a = t, zone 1 a = 7, zone 2 a = h + w (local indices):
    zone means 3.5, 7, 7 -> a_bar 0.5, 1, 1 (divided by the max); v_hat =
    (1, 0, 0), 0 (a constant map: the silent-region case), (0, 1/2, 1/2)."""
    T, H, W = 8, 8, 24
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    a = np.where(w < 8, t, np.where(w < 16, 7.0, h + (w % 8))).astype(np.float32)
    abar, vhat = fn(a, T, H, W)
    np.testing.assert_allclose(abar, [0.5, 1.0, 1.0], atol=1e-12)
    np.testing.assert_allclose(vhat, [[1, 0, 0], [0, 0, 0], [0, 0.5, 0.5]], atol=1e-12)


def test_audio_reading_closed_forms():
    check_audio(po.audio_terms)


def _audio_normalised_by_sum(a, T, H, W):
    abar, vhat = po.audio_terms(a, T, H, W)
    return abar / abar.sum(), vhat


def _audio_vhat_unnormalised(a, T, H, W):
    a64 = np.asarray(a, np.float64)
    az = po.zones_of(a64.reshape(-1, 1), T, H, W)[..., 0]
    sig = np.stack([az.mean(axis=p).var(axis=1) for p in ((2, 3), (1, 3), (1, 2))], axis=1)
    return po.audio_terms(a, T, H, W)[0], sig


@pytest.mark.parametrize("mutant", [_audio_normalised_by_sum, _audio_vhat_unnormalised])
def test_planted_audio_mistakes_are_caught(mutant):
    with pytest.raises(AssertionError):
        check_audio(mutant)
