"""GPU parity of the adaptive temporal zone boundaries (cut_ratio > 0).

Grids with shot cuts (from a frame on every token is a fresh draw) and local
cuts (one zone changes content from a local frame on), planned by the CUDA path
and by the oracle: the frame-difference energies, the split frames, both
parts' shapes, the parts' statistics, the block offsets, the permutation and
the selection must agree (near-tie rules of tests/parity.py, the cut margin
included); O and the gradients are compared with the oracle on the plan the
oracle computes, imported through prism_plan_import_cuts.
"""
import numpy as np
import pytest
import torch

import parity
from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn
from oracle import prism_oracle as po

pytestmark = pytest.mark.gpu

RATIO = 2.5
CASES = {
    # shot cut at global frame 12 (local 4 of the second zone row), local cuts at
    # local frames 3 (-> 4), 1 (-> 2) and 7 (-> 6)
    "grid16x32x32_bf16_d128": dict(wid=2, T=16, H=32, W=32, heads=2, shot_cuts=[12],
                                   local_cuts=[(0, 1, 2, 3), (0, 2, 1, 1), (1, 0, 3, 7)]),
    # shot cut at frame 6 (-> 6) on the tiny fp32 head_dim-64 workload
    "tiny_fp32_d64": dict(wid=0, T=8, H=16, W=16, heads=2, shot_cuts=[6], local_cuts=[(0, 0, 0, 2)]),
}


def _workload(c):
    kw = {k: v for k, v in c.items() if k not in ("wid", "heads")}
    return syn.workload(c["wid"], **kw), c["heads"]


def _params(w, heads, **over):
    dt = _lib.PRISM_F32 if w.dtype == "f32" else _lib.PRISM_BF16
    return _lib.make_params(w.T, w.H, w.W, heads, w.head_dim, dt, w.top_k, w.top_p, w.eps, **over)


@pytest.mark.parametrize("name", list(CASES))
def test_plan_with_cuts_matches_oracle(name, cuda_device):
    w, heads = _workload(CASES[name])
    Q, K, V = syn.make_qkv(w, heads=heads)
    a = syn.make_amap(w)
    pl = _lib.plan(Q.cuda(), K.cuda(), V.cuda(), a.cuda(), _params(w, heads, cut_ratio=RATIO))
    O, lse = pl.attn_fwd()
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    Nz, NB, WORDS = w.zones, w.N // 64, (w.N // 64 + 31) // 32
    gcut = pl.export("zone_cut").reshape(heads, Nz)
    gsid = pl.export("shape_id").reshape(heads, Nz)
    gsid2 = pl.export("shape_id2").reshape(heads, Nz)
    gen = pl.export("zone_energy").reshape(heads, Nz, 7)
    grs = pl.export("region_stats").reshape(heads, Nz, 2, 4)
    nblocks = pl.export("nblocks")
    bstart = pl.export("blk_start").reshape(heads, NB + 1)
    src = pl.export("src").reshape(heads, w.N)
    bits = pl.export("sel_bits").reshape(heads, NB, WORDS)
    O = O.double().cpu().numpy()
    split_seen = 0
    for h in range(heads):
        q, k, v = (x[h].double().numpy() for x in (Q, K, V))
        o = po.plan_head(q, k, v, a.numpy(), w.T, w.H, w.W, w.top_k, w.top_p, w.eps, cut_ratio=RATIO)
        st = o["stats"]
        np.testing.assert_allclose(gen[h], st["energy"], rtol=1e-4, atol=1e-7)
        _, tie, bad = parity.shapes_agree(gsid[h], st, gcut[h], gsid2[h])
        assert not bad, f"head {h}: zones {bad} differ beyond the tie margins"
        split_seen += int((gcut[h] > 0).sum())
        if tie:   # downstream stages against the oracle run on the GPU's accepted stage one
            o = po.plan_head(q, k, v, a.numpy(), w.T, w.H, w.W, w.top_k, w.top_p, w.eps, cut_ratio=RATIO,
                             shape_id=gsid[h], cut=gcut[h], shape_id2=gsid2[h])
        # the parts' statistics of every split zone
        for kk, (m, t0, t1) in enumerate(st["regions"]):
            if st["cut"][m] == 0 or m in tie:
                continue
            part = 0 if t0 == 0 else 1
            sig = grs[h, m, part, :3].astype(np.float64)
            np.testing.assert_allclose(sig / sig.sum(), st["region_r"][kk], rtol=2e-4, atol=1e-6)
        nb = len(o["starts"]) - 1
        assert nblocks[h] == nb
        np.testing.assert_array_equal(bstart[h, :nb + 1], o["starts"])
        np.testing.assert_array_equal(src[h], o["src"])
        gsets = parity.bits_to_sets(bits[h], nb, WORDS)
        exact = []
        for i in range(nb):
            assert parity.selection_agrees(gsets[i], o["logits"][i], o["P"][i], w.top_k, w.top_p), (h, i)
            if np.array_equal(gsets[i], o["sel"][i]):
                exact.append(i)
        rows = np.concatenate([o["src"][o["starts"][i]:o["starts"][i + 1]] for i in exact])
        qa, ka, va = ((x.astype(np.float16).astype(np.float64) if w.dtype == "f32" else x) for x in (q, k, v))
        Oo, _ = po.attention_fwd(qa, ka, va, o["src"], o["starts"], o["sel"])
        good, rl2, ma = parity.close(O[h][rows], Oo[rows])
        assert good, f"head {h}: O relL2 {rl2:.2e} maxabs {ma:.2e}"
    assert split_seen >= 2 * heads


@pytest.mark.parametrize("name", list(CASES))
def test_imported_cut_plan_forward_backward(name, cuda_device):
    w, heads = _workload(CASES[name])
    Q, K, V = syn.make_qkv(w, heads=heads)
    a = syn.make_amap(w)
    dO = syn.make_dout(w, heads=heads, out_dtype=torch.bfloat16).float()
    orc = [po.plan_head(*(x[h].double().numpy() for x in (Q, K, V)), a.numpy(), w.T, w.H, w.W, w.top_k,
                        w.top_p, w.eps, cut_ratio=RATIO) for h in range(heads)]
    NB, WORDS = w.N // 64, (w.N // 64 + 31) // 32
    u8 = lambda key: torch.from_numpy(np.stack([o[key] for o in orc]).astype(np.int64).clip(0, 255)
                                      .astype(np.uint8)).cuda()
    bits = torch.from_numpy(np.stack([parity.sets_to_bits(o["sel"], NB, WORDS) for o in orc]).view(np.int32)).cuda()
    pl = _lib.plan_import(Q.cuda(), K.cuda(), V.cuda(), u8("shape_id"), bits, _params(w, heads),
                          zone_cut=u8("cut"), shape_id2=u8("shape_id2"))
    O, lse = pl.attn_fwd()
    dQ, dK, dV = pl.attn_bwd(dO.cuda(), O, lse)
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    for h in range(heads):
        o = orc[h]
        np.testing.assert_array_equal(pl.export("src").reshape(heads, w.N)[h], o["src"])
        ins = [x[h].double().numpy() for x in (Q, K, V)]
        if w.dtype == "f32":
            ins = [x.astype(np.float16).astype(np.float64) for x in ins]
        Oo, lo = po.attention_fwd(*ins, o["src"], o["starts"], o["sel"])
        good, rl2, ma = parity.close(O[h].double().cpu().numpy(), Oo)
        assert good, f"head {h}: O relL2 {rl2:.2e} maxabs {ma:.2e}"
        ref = po.attention_bwd(*ins, dO[h].double().numpy(), o["src"], o["starts"], o["sel"])
        for got, want, nm in zip((dQ, dK, dV), ref, ("dQ", "dK", "dV")):
            good, rl2, ma, worst = parity.close_grad(got[h].double().cpu().numpy(), want)
            assert good, f"head {h} {nm}: relL2 {rl2:.2e} maxabs {ma:.2e} worst {worst:.2f}"


def test_cut_ratio_zero_is_the_whole_zone_plan(cuda_device):
    w, heads = _workload(CASES["grid16x32x32_bf16_d128"])
    Q, K, V = (x.cuda() for x in syn.make_qkv(w, heads=heads))
    a = syn.make_amap(w).cuda()
    p0 = _lib.plan(Q, K, V, a, _params(w, heads))
    p1 = _lib.plan(Q, K, V, a, _params(w, heads, cut_ratio=1e9))       # no zone reaches the ratio
    for item in ("shape_id", "blk_start", "src", "sel_bits"):
        np.testing.assert_array_equal(p0.export(item), p1.export(item))
    assert not p1.export("zone_cut").any()
    assert p0.export("shape_id").size and _lib.load().prism_plan_item_bytes(p0.handle, 12) == 0


def test_invalid_cut_arguments(cuda_device):
    w, heads = _workload(CASES["tiny_fp32_d64"])
    Q, K, V = (x.cuda() for x in syn.make_qkv(w, heads=1))
    with pytest.raises(_lib.PrismError) as e:
        _lib.plan(Q, K, V, None, _params(w, 1, cut_ratio=-1.0))
    assert e.value.status == _lib.PRISM_ERR_INVALID_ARG
    with pytest.raises(_lib.PrismError) as e:
        _lib.plan(Q, K, V, None, _params(w, 1, cut_ratio=2.5, shape_mode=_lib.PRISM_SHAPE_FIXED, fixed_shape=3))
    assert e.value.status == _lib.PRISM_ERR_INVALID_ARG
    # an imported split frame of 3 (no candidate tiles 3 frames) is a device-check error
    Nz, NB, WORDS = w.zones, w.N // 64, (w.N // 64 + 31) // 32
    sid = torch.full((1, Nz), 7, dtype=torch.uint8, device="cuda")          # 2 x 8 x 8
    cut = torch.full((1, Nz), 3, dtype=torch.uint8, device="cuda")
    bits = torch.full((1, NB, WORDS), -1, dtype=torch.int32, device="cuda")
    pl = _lib.plan_import(Q, K, V, sid, bits, _params(w, 1), zone_cut=cut, shape_id2=sid)
    O, lse = pl.attn_fwd()
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_ERR_DEVICE_CHECK
