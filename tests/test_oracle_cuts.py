"""Pins of the oracle's adaptive temporal zone boundaries.

Reading (page paper.rainbus.top, section "独立分析的弱点" item (1) and section
"未来方向"; page xyznot.com/th, limitations): a zone is split where a shot cut
shows in its frame differences, and each part is planned like a zone.  Pinned
here against hand-built fields whose energies, split positions and statistics
are known in closed form, against per-token brute force on a part, and by the
invariants of the partition (no block crosses the split, every token once).
"""
import numpy as np
import pytest

from oracle import prism_oracle as po


def _field(T, H, W, D, fn):
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    return np.stack([fn(t, h, w, c) for c in range(D)], axis=-1).reshape(-1, D).astype(np.float64)


def _nearest_split(b):
    """Nearest of {2, 4, 6} to a boundary b in 1..7, ties to 4 (written out)."""
    best = min((abs(b - c), c != 4, c) for c in (2, 4, 6))
    return best[2]


@pytest.mark.parametrize("b", range(1, 8))
def test_hard_cut_is_found_and_snapped(b):
    """Frames before b and from b on are independent draws (a shot cut): the
    largest frame-difference energy sits at the pair (b - 1, b), and the zone
    splits at the admissible position nearest to b."""
    rng = np.random.default_rng(b)
    D = 8
    A, Bf = rng.normal(size=(8, 8, 8, D)), rng.normal(size=(8, 8, 8, D))
    smooth = np.linspace(0, 0.2, 8)[:, None, None, None]           # slow drift inside each shot
    Vz = np.where(np.arange(8)[:, None, None, None] < b, A * 0.2 + smooth, Bf * 0.2 + 3 + smooth)
    V = Vz.reshape(-1, D)
    e = po.frame_diff_energy(po.zones_of(V, 8, 8, 8))[0]
    assert int(np.argmax(e)) == b - 1
    st = po.zone_shapes(V, None, 8, 8, 8, eps=1e-4, cut_ratio=4.0)
    assert st["cut"][0] == _nearest_split(b)
    c = st["cut"][0]
    for sid, L in ((st["shape_id"][0], c), (st["shape_id2"][0], 8 - c)):
        bt, bh, bw = po.SHAPES[sid]
        assert L % bt == 0 and bt * bh * bw <= po.max_volume(L)


def test_energy_closed_forms_and_threshold():
    """V = t: every e_t = 1 (no cut).  V = t^2: e_t = (2t + 1)^2 = 1, 9, ..., 169,
    median 49: no cut at ratio 4 (169 < 196), a cut after frame 6 at ratio 3
    (169 > 147), snapped to 6.  A step at frame 4: e = (0, 0, 0, 1, 0, 0, 0),
    median 0, a cut at 4.  A constant zone: no cut."""
    ramp = _field(8, 8, 8, 2, lambda t, h, w, c: t * 1.0)
    np.testing.assert_allclose(po.frame_diff_energy(po.zones_of(ramp, 8, 8, 8))[0], np.ones(7))
    assert po.zone_shapes(ramp, None, 8, 8, 8, 1e-4, cut_ratio=4.0)["cut"][0] == 0
    sq = _field(8, 8, 8, 2, lambda t, h, w, c: t * t * 1.0)
    np.testing.assert_allclose(po.frame_diff_energy(po.zones_of(sq, 8, 8, 8))[0],
                               [(2 * t + 1) ** 2 for t in range(7)])
    assert po.zone_shapes(sq, None, 8, 8, 8, 1e-4, cut_ratio=4.0)["cut"][0] == 0
    assert po.zone_shapes(sq, None, 8, 8, 8, 1e-4, cut_ratio=3.0)["cut"][0] == 6
    step = _field(8, 8, 8, 2, lambda t, h, w, c: (t >= 4) * 1.0)
    np.testing.assert_allclose(po.frame_diff_energy(po.zones_of(step, 8, 8, 8))[0], [0, 0, 0, 1, 0, 0, 0])
    st = po.zone_shapes(step, None, 8, 8, 8, 1e-4, cut_ratio=4.0)
    assert st["cut"][0] == 4
    # each part is constant: r = 1/3, density 0 (max 0 -> rho 0 -> B = 256), and
    # the only 256-token candidate with b_T dividing 4 frames is 4 x 8 x 8
    assert po.SHAPES[st["shape_id"][0]] == (4, 8, 8) and po.SHAPES[st["shape_id2"][0]] == (4, 8, 8)
    np.testing.assert_allclose(st["region_r"], 1 / 3)
    const = np.ones((512, 2))
    assert po.zone_shapes(const, None, 8, 8, 8, 1e-4, cut_ratio=4.0)["cut"][0] == 0


def test_cut_off_equals_whole_zones():
    rng = np.random.default_rng(0)
    T, H, W, D = 16, 16, 8, 8
    Q, K, V = (rng.normal(size=(T * H * W, D)) for _ in range(3))
    V[: 4 * 64 * 2] += 5.0                                   # a jump inside the first zone row
    a = rng.uniform(size=(T, H, W)).astype(np.float32)
    p0 = po.plan_head(Q, K, V, a, T, H, W, 3, 0.5, 1e-4)
    p1 = po.plan_head(Q, K, V, a, T, H, W, 3, 0.5, 1e-4, cut_ratio=0.0)
    for k in ("shape_id", "src", "starts"):
        np.testing.assert_array_equal(p0[k], p1[k])
    assert not p1["cut"].any()


def _bruteforce_part(Vz, t0, t1):
    """Per-token loops over frames [t0, t1) of one zone: sigma^2_{v,d} and rho_raw."""
    D = Vz.shape[-1]
    L = t1 - t0
    frames = range(t0, t1)
    sig = []
    for d in range(3):
        n_sl = L if d == 0 else 8
        tot = 0.0
        for c in range(D):
            prof = []
            for i in range(n_sl):
                vals = [Vz[t, h, w, c] for t in frames for h in range(8) for w in range(8)
                        if (t - t0, h, w)[d] == i]
                prof.append(sum(vals) / len(vals))
            mu = sum(prof) / n_sl
            tot += sum((x - mu) ** 2 for x in prof) / n_sl
        sig.append(tot / D)
    rho = 0.0
    for c in range(D):
        sp = 0.0
        for t in frames:
            vals = [Vz[t, h, w, c] for h in range(8) for w in range(8)]
            mu = sum(vals) / 64
            sp += sum((x - mu) ** 2 for x in vals) / 64
        diffs = [Vz[t + 1, h, w, c] - Vz[t, h, w, c] for t in range(t0, t1 - 1) for h in range(8) for w in range(8)]
        mu = sum(diffs) / len(diffs)
        rho += sp / L + sum((x - mu) ** 2 for x in diffs) / len(diffs)
    return np.array(sig), rho / D


@pytest.mark.parametrize("b", [2, 4, 6])
def test_part_statistics_match_bruteforce(b):
    rng = np.random.default_rng(20 + b)
    D = 3
    Vz = rng.normal(size=(8, 8, 8, D))
    Vz[b:] = 4.0 + rng.normal(size=(8 - b, 8, 8, D)) * 0.5        # a new shot from frame b
    V = Vz.reshape(-1, D)
    st = po.zone_shapes(V, None, 8, 8, 8, 1e-4, cut_ratio=4.0)
    assert st["cut"][0] == b and st["regions"] == [(0, 0, b), (0, b, 8)]
    raws = []
    for k, (m, t0, t1) in enumerate(st["regions"]):
        sig, rho = _bruteforce_part(Vz, t0, t1)
        np.testing.assert_allclose(st["region_r"][k], sig / sig.sum(), rtol=1e-10)
        raws.append(rho)
    np.testing.assert_allclose(st["region_rho"], np.float32(np.array(raws) / max(raws)), rtol=1e-6)


def test_region_audio_closed_form():
    """a = t over one zone cut at 4: part 0 has mean 1.5 and slice means 0..3
    along T (variance 1.25, none along H, W), part 1 mean 5.5: a_bar = 1.5/5.5, 1;
    v_hat = (1, 0, 0) for both."""
    V = _field(8, 8, 8, 2, lambda t, h, w, c: (t >= 4) * 10.0 + 0.01 * h)
    a = _field(8, 8, 8, 1, lambda t, h, w, c: t * 1.0)[:, 0].reshape(8, 8, 8).astype(np.float32)
    st = po.zone_shapes(V, a, 8, 8, 8, 1e-4, cut_ratio=4.0)
    assert st["cut"][0] == 4
    np.testing.assert_allclose(st["region_abar"], [1.5 / 5.5, 1.0], rtol=1e-12)
    np.testing.assert_allclose(st["region_vhat"], [[1, 0, 0], [1, 0, 0]], atol=1e-12)


def test_partition_with_cuts_keeps_blocks_inside_parts():
    T, H, W = 16, 8, 16
    rng = np.random.default_rng(4)
    nz = (T // 8) * (H // 8) * (W // 8)
    cut = np.array([2, 4, 6, 0])
    sid, sid2 = [], []
    for c in cut:
        ok0 = [i for i, s in enumerate(po.SHAPES) if (c or 8) % s[0] == 0 and np.prod(s) <= po.max_volume(c or 8)]
        ok1 = [i for i, s in enumerate(po.SHAPES) if (8 - c) % s[0] == 0 and np.prod(s) <= po.max_volume(8 - c)]
        sid.append(int(rng.choice(ok0)))
        sid2.append(int(rng.choice(ok1)) if c else -1)
    src, starts = po.partition(np.array(sid), T, H, W, cut, np.array(sid2))
    assert sorted(src.tolist()) == list(range(T * H * W))
    assert np.all(starts % 64 == 0) and starts[-1] == T * H * W
    tt, hh, ww = src // (H * W), (src // W) % H, src % W
    vols = np.diff(starts)
    assert np.all(starts[:-1][vols == 256] % 256 == 0) and np.all(starts[:-1][vols == 128] % 128 == 0)
    for j in range(len(starts) - 1):
        a_, b_ = starts[j], starts[j + 1]
        m = a_ // 512
        zt, rem = divmod(m, (H // 8) * (W // 8))
        lt = tt[a_:b_] - 8 * zt
        c = cut[m]
        if c:
            assert np.all(lt < c) or np.all(lt >= c), f"block {j} crosses the split of zone {m}"
        key = (tt[a_:b_] * H + hh[a_:b_]) * W + ww[a_:b_]
        assert np.all(np.diff(key) > 0)                     # raster order inside the block
        assert np.ptp(tt[a_:b_]) + 1 in (2, 4, 8)


def test_no_cuts_on_smooth_synthetic_fields():
    """The smoothed fields of the workload generator (no shot cut) stay whole at
    ratio 2.5: their largest energy stays below 1.7 times the median."""
    from dynamic_block_sparse_indicator_b200 import synthetic as syn
    w = syn.workload(2, T=16, H=32, W=32)
    Q, K, V = syn.make_qkv(w, heads=1)
    st = po.zone_shapes(V[0].double().numpy(), None, w.T, w.H, w.W, w.eps, cut_ratio=2.5)
    assert not st["cut"].any()


def test_synthetic_shot_cut_is_found():
    """A workload with a shot cut at global frame 12 (local frame 4 of the second
    zone row) and a local cut in one zone: exactly those zones split.  (Zones
    with a per-frame component, the generator's T-fast zones, change strongly
    at every frame and are left out: their median energy hides a cut.)"""
    from dynamic_block_sparse_indicator_b200 import synthetic as syn
    w = syn.workload(2, T=16, H=32, W=32, shot_cuts=[12], local_cuts=[(0, 1, 2, 3)],
                     n_tfast=0, n_hfast=0, n_wfast=0)
    Q, K, V = syn.make_qkv(w, heads=1)
    st = po.zone_shapes(V[0].double().numpy(), None, w.T, w.H, w.W, w.eps, cut_ratio=2.5)
    zh_n, zw_n = w.H // 8, w.W // 8
    want = np.zeros(w.zones, np.int64)
    want[zh_n * zw_n:] = 4                                  # every zone of the second zone row
    want[(0 * zh_n + 1) * zw_n + 2] = 4                     # local cut at frame 3 -> 4
    np.testing.assert_array_equal(st["cut"], want)


def _argmin_cuts(e, cut_ratio):
    e = np.asarray(e, np.float64)
    cut = np.zeros(e.shape[0], np.int64)
    for m in range(e.shape[0]):
        t = int(np.argmin(e[m]))
        if e[m].max() > cut_ratio * np.sort(e[m])[3]:
            cut[m] = po.CUT_SNAP[t + 1]
    return cut, np.full(e.shape[0], np.inf)


def _mean_instead_of_median(e, cut_ratio):
    e = np.asarray(e, np.float64)
    cut = np.zeros(e.shape[0], np.int64)
    for m in range(e.shape[0]):
        t = int(np.argmax(e[m]))
        if e[m, t] > cut_ratio * e[m].mean():
            cut[m] = po.CUT_SNAP[t + 1]
    return cut, np.full(e.shape[0], np.inf)


@pytest.mark.parametrize("mutant", [_argmin_cuts, _mean_instead_of_median])
def test_planted_cut_mistakes_are_caught(mutant, monkeypatch):
    monkeypatch.setattr(po, "zone_cuts", mutant)
    with pytest.raises(AssertionError):
        test_energy_closed_forms_and_threshold()
        for b in range(1, 8):
            test_hard_cut_is_found_and_snapped(b)
