"""Pins of the CPU oracle against what the Prism pages and the mathematics fix.

Each test checks the oracle against something other than itself: the pages'
printed hyperparameters and shape set, hand-worked closed-form examples, a
numerical minimisation of the block-shape objective, per-token brute force
on tiny grids, set-theoretic Top-k / Top-p on tiny rows, and PyTorch's own
dense attention and autograd in float64.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

from oracle import prism_oracle as po

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------- shapes
def test_candidate_set_matches_pages():
    gold = json.load(open(os.path.join(GOLD, "candidate_shapes.json")))
    shapes = po.candidate_shapes()
    assert len(shapes) == gold["count"] == 16
    for vol, n in gold["per_volume"].items():
        assert sum(1 for s in shapes if np.prod(s) == int(vol)) == n
    for s in shapes:
        assert all(e in (2, 4, 8) for e in s)
        assert np.prod(s) in (64, 128, 256)
    for s in gold["named_in_table11"]:
        assert tuple(s) in shapes
    # every permutation of a candidate is a candidate of the same volume
    for s in shapes:
        for p in itertools.permutations(s):
            assert p in shapes
    # ids grouped by volume, lexicographic inside each volume
    for vol in (64, 128, 256):
        grp = [s for s in shapes if np.prod(s) == vol]
        assert grp == sorted(grp)


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLD, "closed_form.json")))["cases"])
def test_closed_form_worked_examples(case):
    g = np.array([case["g"]], dtype=np.float32)
    ell = po.ideal_log_edges(g, np.array([case["B"]], dtype=np.float32))[0]
    np.testing.assert_allclose(ell, case["ell"], atol=2e-6)
    sid = po.snap(ell, case["B"])
    assert po.SHAPES[sid] == tuple(case["shape"])


def _argmin_J(g, S, n=1201, span=8.0):
    """Numerically minimise J = sum_d g_d (4^l_d - 1) on the plane sum l = S."""
    best = None
    grid = np.linspace(-span, span, n)
    lt, lh = np.meshgrid(grid, grid, indexing="ij")
    lw = S - lt - lh
    J = g[0] * (4.0 ** lt - 1) + g[1] * (4.0 ** lh - 1) + g[2] * (4.0 ** lw - 1)
    i = np.unravel_index(np.argmin(J), J.shape)
    best = np.array([lt[i], lh[i], lw[i]])
    # refine around the coarse minimum
    step = grid[1] - grid[0]
    f = np.linspace(-2 * step, 2 * step, 401)
    lt2, lh2 = np.meshgrid(best[0] + f, best[1] + f, indexing="ij")
    lw2 = S - lt2 - lh2
    J2 = g[0] * (4.0 ** lt2 - 1) + g[1] * (4.0 ** lh2 - 1) + g[2] * (4.0 ** lw2 - 1)
    j = np.unravel_index(np.argmin(J2), J2.shape)
    return np.array([lt2[j], lh2[j], lw2[j]])


@pytest.mark.parametrize("seed", range(6))
def test_closed_form_minimises_block_objective(seed):
    """l* is the minimiser of sum g_d (b_d^2 - 1) subject to prod b_d = B (Lagrange)."""
    rng = np.random.default_rng(seed)
    g = np.exp(rng.uniform(-2.5, 2.5, size=3))
    for vol in (64, 128, 256):
        S = np.log2(vol)
        num = _argmin_J(g, S)
        ell = po.ideal_log_edges(g.astype(np.float32)[None], np.array([vol], np.float32))[0]
        np.testing.assert_allclose(ell, num, atol=2e-3)


@pytest.mark.parametrize("seed", range(20))
def test_ideal_edges_invariants(seed):
    rng = np.random.default_rng(100 + seed)
    g = np.exp(rng.uniform(-4, 4, size=(1, 3))).astype(np.float32)
    for vol in (64, 128, 256):
        ell = po.ideal_log_edges(g, np.array([vol], np.float32))[0].astype(np.float64)
        assert abs(ell.sum() - np.log2(vol)) < 1e-4                  # product = B
        lag = g[0].astype(np.float64) * 4.0 ** ell                   # g_d b_d^2 equal
        assert np.ptp(np.log(lag)) < 1e-4
        ell2 = po.ideal_log_edges(g * np.float32(7.5), np.array([vol], np.float32))[0]
        np.testing.assert_allclose(ell2, ell, atol=1e-4)             # scale-free
        sid = po.snap(ell.astype(np.float32), vol)
        b = po.SHAPES[sid]
        assert np.prod(b) == vol
        for d, e in itertools.permutations(range(3), 2):
            if g[0, d] > g[0, e]:
                assert b[d] <= b[e]                                  # faster axis, shorter edge


def test_snap_is_nearest_candidate_bruteforce():
    rng = np.random.default_rng(7)
    for _ in range(200):
        vol = int(rng.choice([64, 128, 256]))
        ell = rng.uniform(0.0, 3.5, size=3).astype(np.float32)
        sid = po.snap(ell, vol)
        d = {i: float(np.sum((np.log2(s) - ell.astype(np.float64)) ** 2))
             for i, s in enumerate(po.SHAPES) if np.prod(s) == vol}
        best = min(d.values())
        assert d[sid] <= best + 1e-6


# ------------------------------------------------------------ zone statistics
def _bruteforce_zone_stats(Vz, az):
    """Per-token loops over one zone, written straight from the formulas."""
    D = Vz.shape[-1]
    sig = []
    for d in range(3):
        tot = 0.0
        for c in range(D):
            prof = []
            for i in range(8):
                s, n = 0.0, 0
                for t in range(8):
                    for h in range(8):
                        for w in range(8):
                            if (t, h, w)[d] == i:
                                s += Vz[t, h, w, c]
                                n += 1
                prof.append(s / n)
            mu = sum(prof) / 8
            tot += sum((x - mu) ** 2 for x in prof) / 8
        sig.append(tot / D)
    rho = 0.0
    for c in range(D):
        sp = 0.0
        for t in range(8):
            vals = [Vz[t, h, w, c] for h in range(8) for w in range(8)]
            mu = sum(vals) / 64
            sp += sum((x - mu) ** 2 for x in vals) / 64
        diffs = [Vz[t + 1, h, w, c] - Vz[t, h, w, c]
                 for t in range(7) for h in range(8) for w in range(8)]
        mu = sum(diffs) / len(diffs)
        rho += sp / 8 + sum((x - mu) ** 2 for x in diffs) / len(diffs)
    rho /= D
    amean = float(az.sum()) / 512
    asig = []
    for d in range(3):
        prof = []
        for i in range(8):
            vals = [az[t, h, w] for t in range(8) for h in range(8) for w in range(8)
                    if (t, h, w)[d] == i]
            prof.append(sum(vals) / 64)
        asig.append(sum((x - amean) ** 2 for x in prof) / 8)
    return np.array(sig), rho, amean, np.array(asig)


def test_zone_statistics_match_bruteforce():
    rng = np.random.default_rng(3)
    T, H, W, D = 8, 16, 8, 3
    V = rng.normal(size=(T * H * W, D)) * rng.uniform(0.2, 2, size=D)
    V[: 64 * 8] += np.linspace(0, 1, 8).repeat(64)[:, None]     # a trend along T in zone 0
    a = rng.uniform(0, 1, size=(T, H, W)).astype(np.float32).astype(np.float64)
    Vz = po.zones_of(V, T, H, W)
    sig = po.directional_variance(Vz)
    rho = po.density_raw(Vz)
    az = po.zones_of(a.reshape(-1, 1), T, H, W)[..., 0]
    abar, vhat = po.audio_terms(a, T, H, W)
    means = []
    for m in range(Vz.shape[0]):
        bs, br, am, asg = _bruteforce_zone_stats(Vz[m], az[m])
        np.testing.assert_allclose(sig[m], bs, rtol=1e-10)
        np.testing.assert_allclose(rho[m], br, rtol=1e-10)
        np.testing.assert_allclose(vhat[m], asg / asg.sum(), rtol=1e-10)
        means.append(am)
    np.testing.assert_allclose(abar, np.array(means) / max(means), rtol=1e-10)
    # zone m covers raster tokens t in [0,8), h in [8m, 8m+8): check the view itself
    np.testing.assert_array_equal(Vz[1, 2, 3, 4], V[(2 * H + 8 + 3) * W + 4])


def test_handbuilt_fields():
    T = H = W = 8
    D = 4
    rng = np.random.default_rng(5)
    t = np.arange(T).repeat(H * W)
    # varies only along T: r_T = 1, so the shape takes the short time edge
    V = np.stack([np.sin(t + c) for c in range(D)], axis=1)
    st = po.zone_shapes(V, None, T, H, W, eps=1e-6)
    np.testing.assert_allclose(st["r"][0], [1, 0, 0], atol=1e-12)
    assert po.SHAPES[st["shape_id"][0]][0] == 2
    assert st["B"][0] == 64                                        # the only zone holds the max
    # varies only along W
    w = np.tile(np.arange(W), T * H)
    V = np.stack([np.cos(0.7 * w + c) for c in range(D)], axis=1)
    st = po.zone_shapes(V, None, T, H, W, eps=1e-6)
    np.testing.assert_allclose(st["r"][0], [0, 0, 1], atol=1e-12)
    assert po.SHAPES[st["shape_id"][0]][2] == 2
    # constant zone: r = 1/3 (reading), rho = 0 -> max 0 -> rho 0 -> B = 256
    V = np.ones((512, D))
    st = po.zone_shapes(V, None, T, H, W, eps=1e-6)
    np.testing.assert_allclose(st["r"][0], [1 / 3] * 3)
    assert st["B"][0] == 256 and po.SHAPES[st["shape_id"][0]] == (4, 8, 8)
    # constant audio map (a float32 value, as the map is float32): v_hat = 0,
    # so g = r + eps whatever a_bar is
    V = rng.normal(size=(512, D))
    s0 = po.zone_shapes(V, None, T, H, W, eps=1e-6)
    a_const = np.full((T, H, W), np.float32(0.7), dtype=np.float32)
    s1 = po.zone_shapes(V, a_const, T, H, W, eps=1e-6)
    np.testing.assert_array_equal(s0["g"], s1["g"])
    np.testing.assert_array_equal(s1["vhat"], 0)


def test_audio_term_tilts_shape():
    """A T-varying audio norm inside a zone shortens b_T (the talking-mouth case)."""
    T, H, W, D = 8, 8, 16, 8
    rng = np.random.default_rng(11)
    V = rng.normal(size=(T * H * W, D))                         # isotropic noise
    a = np.full((T, H, W), 0.05)
    a[:, :, :8] += np.linspace(0, 1, 8)[:, None, None]          # zone 0: audio varies along T
    st = po.zone_shapes(V, a, T, H, W, eps=1e-4)
    assert st["abar"][0] == pytest.approx(1.0)
    assert st["vhat"][0][0] == pytest.approx(1.0)
    assert st["g"][0][0] > st["g"][0][1] and st["g"][0][0] > st["g"][0][2]
    assert po.SHAPES[st["shape_id"][0]][0] == 2
    # zone 1 has constant audio: its v_hat vanishes
    np.testing.assert_array_equal(st["vhat"][1], 0)


# ------------------------------------------------------------------ partition
def test_partition_blocks_are_boxes():
    T, H, W = 16, 8, 24
    rng = np.random.default_rng(2)
    nz = (T // 8) * (H // 8) * (W // 8)
    sid = rng.integers(0, 16, size=nz)
    src, starts = po.partition(sid, T, H, W)
    assert sorted(src.tolist()) == list(range(T * H * W))
    assert starts[0] == 0 and starts[-1] == T * H * W
    assert np.all(starts % 64 == 0)
    tt, hh, ww = src // (H * W), (src // W) % H, src % W
    blk = 0
    for m in range(nz):
        bt, bh, bw = po.SHAPES[sid[m]]
        for k in range(512 // (bt * bh * bw)):
            a, b = starts[blk], starts[blk + 1]
            assert b - a == bt * bh * bw
            ct, ch, cw = tt[a:b], hh[a:b], ww[a:b]
            assert ct.max() - ct.min() + 1 == bt and ct.min() % bt == 0
            assert ch.max() - ch.min() + 1 == bh and ch.min() % bh == 0
            assert cw.max() - cw.min() + 1 == bw and cw.min() % bw == 0
            assert len(set(zip(ct, ch, cw))) == b - a
            # raster order inside the block
            key = (ct * H + ch) * W + cw
            assert np.all(np.diff(key) > 0)
            blk += 1
    assert blk == len(starts) - 1
    X = rng.normal(size=(T * H * W, 3))
    Pm = po.pool(X, src, starts)
    for j in (0, 5, len(starts) - 2):
        np.testing.assert_allclose(Pm[j], X[src[starts[j]:starts[j + 1]]].mean(0))


# ------------------------------------------------------------------ selection
def _bruteforce_select(P, k, p):
    nb = len(P)
    idx = sorted(range(nb), key=lambda j: (-P[j], j))
    topk = set(idx[:min(k, nb)])
    if p <= 0:
        topp = set()
    else:
        topp = None
        for L in range(1, nb + 1):
            # best mass among all subsets of size L (exhaustive for tiny rows)
            best = max(sum(P[j] for j in c) for c in itertools.combinations(range(nb), L))
            if best >= p:
                topp = set(idx[:L])
                break
        if topp is None:
            topp = set(range(nb))
    return sorted(topk | topp)


@pytest.mark.parametrize("seed", range(30))
def test_selection_matches_set_definition(seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(2, 9))
    s = rng.normal(scale=rng.uniform(0.3, 3.0), size=nb).astype(np.float32)
    P = np.exp(s - s.max())
    P = (P / P.sum()).astype(np.float32)
    for k in (0, 1, 2, 4, 16):
        for p in (0.0, 0.2, 0.5, 0.9, 0.97, 1.0):
            if k == 0 and p <= 0:
                continue
            cum = np.cumsum(np.sort(P.astype(np.float64))[::-1])
            if np.min(np.abs(cum - p)) < 1e-5 and 0 < p < 1:
                continue                                     # skip near-ties of the threshold
            got, _, _ = po.select_row(P, k, p)
            want = _bruteforce_select(P.astype(np.float64), k, p)
            assert got.tolist() == want


def test_selection_degenerate_cases():
    rng = np.random.default_rng(9)
    Qb, Kb = rng.normal(size=(6, 8)), rng.normal(size=(6, 8))
    sel, _, _ = po.select(Qb, Kb, k=6, p=0.0)
    assert all(len(s) == 6 for s in sel)
    sel, _, _ = po.select(Qb, Kb, k=1, p=1.0)
    assert all(len(s) == 6 for s in sel)
    sel, s, _ = po.select(Qb, Kb, k=1, p=0.0)
    assert [x.tolist() for x in sel] == [[int(np.argmax(r))] for r in s]
    # equal logits: ties go to the lower block index
    sel, _, _ = po.select(np.zeros((2, 4)), np.zeros((5, 4)), k=2, p=0.0)
    assert [x.tolist() for x in sel] == [[0, 1], [0, 1]]


# ------------------------------------------------------------------ attention
def _tiny_plan(seed=0, k=3, p=0.5):
    T, H, W, D = 8, 16, 16, 16
    rng = np.random.default_rng(seed)
    Q, K, V = (rng.normal(size=(T * H * W, D)) for _ in range(3))
    pl = po.plan_head(Q, K, V, None, T, H, W, k, p, eps=1e-6)
    return Q, K, V, pl, D


def _torch_masked(Q, K, V, mask):
    q, k, v = (torch.tensor(x, dtype=torch.float64) for x in (Q, K, V))
    m = torch.tensor(mask)
    return q, k, v, m


def test_attention_all_blocks_equals_dense_attention():
    T, H, W, D = 8, 16, 16, 16
    rng = np.random.default_rng(1)
    Q, K, V = (rng.normal(size=(T * H * W, D)) for _ in range(3))
    pl = po.plan_head(Q, K, V, None, T, H, W, k=10 ** 6, p=0.0, eps=1e-6)
    O, lse = po.attention_fwd(Q, K, V, pl["src"], pl["starts"], pl["sel"])
    q, k, v = (torch.tensor(x)[None, None] for x in (Q, K, V))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v)[0, 0].numpy()
    np.testing.assert_allclose(O, ref, atol=1e-10)
    s = torch.tensor(Q) @ torch.tensor(K).T / np.sqrt(D)
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=1).numpy(), atol=1e-10)
    # p = 1 keeps all blocks as well
    pl1 = po.plan_head(Q, K, V, None, T, H, W, k=1, p=1.0, eps=1e-6)
    assert all(len(s_) == len(pl1["starts"]) - 1 for s_ in pl1["sel"])


def test_masked_attention_forward_and_backward_match_torch():
    Q, K, V, pl, D = _tiny_plan()
    mask = po.token_mask(pl["src"], pl["starts"], pl["sel"])
    assert 0 < mask.mean() < 1
    q, k, v, m = _torch_masked(Q, K, V, mask)
    for t in (q, k, v):
        t.requires_grad_(True)
    ref = torch.nn.functional.scaled_dot_product_attention(q[None, None], k[None, None],
                                                           v[None, None], attn_mask=m)[0, 0]
    O, lse = po.attention_fwd(Q, K, V, pl["src"], pl["starts"], pl["sel"])
    np.testing.assert_allclose(O, ref.detach().numpy(), atol=1e-10)
    s = (q @ k.T / np.sqrt(D)).masked_fill(~m, float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, 1).detach().numpy(), atol=1e-10)
    dO = np.random.default_rng(4).normal(size=O.shape)
    ref.backward(torch.tensor(dO))
    dQ, dK, dV = po.attention_bwd(Q, K, V, dO, pl["src"], pl["starts"], pl["sel"])
    np.testing.assert_allclose(dQ, q.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dK, k.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dV, v.grad.numpy(), atol=1e-10)
    rows = np.array([0, 17, 300, 2047])
    Or, lr, dQr = po.attention_rows(Q, K, V, pl["src"], pl["starts"], pl["sel"], rows, dO=dO)
    np.testing.assert_allclose(Or, O[rows], atol=1e-12)
    np.testing.assert_allclose(lr, lse[rows], atol=1e-12)
    np.testing.assert_allclose(dQr, dQ[rows], atol=1e-12)


def test_tiny_workload_plan_properties():
    """The time-varying zone of the tiny workload is the densest and the fastest along T.

    Without the audio term (first layer) it takes the short time edge b_T = 2;
    with the isotropic audio blob on it, g_T is still the largest g, so b_T is
    no longer than the other edges.
    """
    from dynamic_block_sparse_indicator_b200 import synthetic as syn
    w = syn.workload(0)
    Q, K, V = syn.make_qkv(w)
    a = syn.make_amap(w).numpy()
    zh_n, zw_n = w.H // 8, w.W // 8
    m = (0 * zh_n + 1) * zw_n + 1                                # zone (0, 1, 1)
    for h in range(w.heads):
        st = po.zone_shapes(V[h].numpy(), None, w.T, w.H, w.W, w.eps)
        assert st["rho"][m] == 1.0 and st["B"][m] == 64
        assert np.argmax(st["r"][m]) == 0
        assert po.SHAPES[st["shape_id"][m]][0] == 2
        st = po.zone_shapes(V[h].numpy(), a, w.T, w.H, w.W, w.eps)
        assert st["abar"][m] == 1.0
        assert np.argmax(st["g"][m]) == 0
        b = po.SHAPES[st["shape_id"][m]]
        assert b[0] <= b[1] and b[0] <= b[2]


@pytest.mark.parametrize("seed,k,p", [(0, 3, 0.5), (1, 1, 0.0), (2, 2, 0.9)])
def test_key_rows_match_torch_autograd(seed, k, p):
    """attention_key_rows gives torch's float64 autograd dK, dV of the masked
    attention at every key row; attention_rows its O, LSE and dQ rows."""
    Q, K, V, pl, D = _tiny_plan(seed, k, p)
    mask = po.token_mask(pl["src"], pl["starts"], pl["sel"])
    q, kk, v, m = _torch_masked(Q, K, V, mask)
    for t in (q, kk, v):
        t.requires_grad_(True)
    out = torch.nn.functional.scaled_dot_product_attention(q[None, None], kk[None, None],
                                                           v[None, None], attn_mask=m)[0, 0]
    dO = np.random.default_rng(40 + seed).normal(size=Q.shape)
    out.backward(torch.tensor(dO))
    keys = np.arange(Q.shape[0])
    dKr, dVr = po.attention_key_rows(Q, K, V, dO, pl["src"], pl["starts"], pl["sel"], keys)
    np.testing.assert_allclose(dKr, kk.grad.numpy(), atol=1e-10)
    np.testing.assert_allclose(dVr, v.grad.numpy(), atol=1e-10)
    rows = np.random.default_rng(seed).choice(Q.shape[0], 100, replace=False)
    Or, lr, dQr = po.attention_rows(Q, K, V, pl["src"], pl["starts"], pl["sel"], rows, dO=dO, chunk=32)
    np.testing.assert_allclose(Or, out.detach().numpy()[rows], atol=1e-10)
    np.testing.assert_allclose(dQr, q.grad.numpy()[rows], atol=1e-10)
    s = (q @ kk.T / np.sqrt(D)).masked_fill(~m, float("-inf"))
    np.testing.assert_allclose(lr, torch.logsumexp(s, 1).detach().numpy()[rows], atol=1e-10)


def test_token_order_inside_a_block_affects_no_result():
    """Reading 6 (tokens inside a block in raster order) is free: any order of the
    tokens inside each block gives the same pooled means, block scores,
    selection, O, LSE and gradients in raster order."""
    Q, K, V, pl, D = _tiny_plan(3, 3, 0.6)
    src, st, sel = pl["src"], pl["starts"], pl["sel"]
    rng = np.random.default_rng(8)
    src2 = src.copy()
    for i in range(len(st) - 1):
        src2[st[i]:st[i + 1]] = rng.permutation(src[st[i]:st[i + 1]])
    assert not np.array_equal(src2, src)
    for X in (Q, K):
        np.testing.assert_allclose(po.pool(X, src2, st), po.pool(X, src, st), atol=1e-12)
    sel2, s2, _ = po.select(po.pool(Q, src2, st), po.pool(K, src2, st), 3, 0.6)
    assert [x.tolist() for x in sel2] == [x.tolist() for x in sel]
    O, lse = po.attention_fwd(Q, K, V, src, st, sel)
    O2, lse2 = po.attention_fwd(Q, K, V, src2, st, sel)
    np.testing.assert_allclose(O2, O, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, atol=1e-12)
    dO = rng.normal(size=Q.shape)
    for g2, g in zip(po.attention_bwd(Q, K, V, dO, src2, st, sel), po.attention_bwd(Q, K, V, dO, src, st, sel)):
        np.testing.assert_allclose(g2, g, atol=1e-10)
