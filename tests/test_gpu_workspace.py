"""Workspace sizing: head groups, index lists sized from their counts, and
grids beyond 3.1M tokens.

  * A 16-head layer of 147,456 tokens (two forward key-range passes; the
    forward state and the gradient scratch hold 14 heads, so the heads run in
    two groups), planned with the core workspace and the lists sized from their
    counts, equals 16 one-head calls: plan, O and LSE bit for bit, dQ, dK and
    dV to fp32 summation order (partial sums of three query chunks and of many
    key tiles are reduce-added in the order the CTAs finish).
  * The 2K training layer with all 40 heads in one call (1,013,760 tokens per
    head, bf16 outputs): the core workspace plus the exact lists fit beside the
    layer's tensors on one GPU; two heads equal their one-head calls.
  * A native-4K grid (72 x 176 x 320, 4,055,040 tokens: 63,360 blocks per head at
    most, past the 48K that one block row of the selection keeps in shared
    memory): the plan against the oracle's, and with the oracle's plan imported
    O and dQ on sampled rows, dK and dV on sampled key rows.
"""
import numpy as np
import pytest
import torch

import parity
from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn
from oracle import prism_oracle as po

pytestmark = pytest.mark.gpu


def _params(w, heads, **over):
    return _lib.make_params(w.T, w.H, w.W, heads, w.head_dim, _lib.PRISM_BF16, w.top_k, w.top_p, w.eps, **over)


def _run(Q, K, V, a, dO, prm, compact):
    pl = _lib.plan(Q, K, V, a, prm, compact=compact)
    O, lse = pl.attn_fwd()
    grads = pl.attn_bwd(dO, O, lse)
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    return pl, (O, lse) + tuple(grads)


def _assert_sum_order(g, r, what):
    diff, scale = (g - r).abs().max().item(), r.abs().max().item()
    assert diff <= 1e-5 * scale, f"{what}: max diff {diff:.3e} at scale {scale:.3e}"


def test_head_groups_and_compact_lists_equal_one_head_calls(cuda_device):
    w = syn.workload(2, T=16, H=64, W=144, top_p=0.6)
    heads = 16
    Q, K, V = syn.make_qkv(w, device="cuda", heads=heads)
    dO = syn.make_dout(w, device="cuda", heads=heads, out_dtype=torch.bfloat16).float()
    a = syn.make_amap(w, device="cuda")
    prm = _params(w, heads)
    assert _lib.core_bytes(prm) < _lib.workspace_bytes(prm)
    pl, outs = _run(Q, K, V, a, dO, prm, compact=True)
    nbytes = int(pl._lists.numel())
    dense = _lib.workspace_bytes(prm) - _lib.core_bytes(prm)
    assert nbytes < dense / 4, (nbytes, dense)
    NB = w.N // 64
    for h in (0, 7, 13, 14, 15):                             # both head groups
        sl = slice(h, h + 1)
        p1, o1 = _run(Q[sl], K[sl], V[sl], a, dO[sl], _params(w, 1), compact=False)
        for item, shape in (("shape_id", (w.zones,)), ("blk_start", (NB + 1,)), ("src", (w.N,)),
                            ("sel_bits", (NB, (NB + 31) // 32))):
            np.testing.assert_array_equal(pl.export(item).reshape(heads, *shape)[h], p1.export(item).reshape(shape),
                                          err_msg=f"head {h} {item}")
        for got, want, nm in zip(outs, o1, ("O", "LSE", "dQ", "dK", "dV")):
            g, r = got[h].cpu(), want[0].cpu()
            if nm in ("O", "LSE"):
                assert torch.equal(g, r), f"head {h} {nm}: max diff {(g - r).abs().max().item():.3e}"
            else:                                            # reduce-adds across chunks and key tiles
                _assert_sum_order(g, r, f"head {h} {nm}")


def test_forty_heads_at_one_million_tokens_in_one_call(cuda_device):
    w = syn.workload(3)
    heads = w.heads
    assert heads == 40
    prm = _params(w, heads, out_dtype=_lib.PRISM_BF16)
    core = _lib.core_bytes(prm)
    # Q, K, V, dO, O, dQ, dK, dV in bf16 and the LSE: with the lists at their dense
    # bound the workspace would not fit beside them on a 180 GB GPU
    tensors = 8 * heads * w.N * w.head_dim * 2 + 4 * heads * w.N
    assert _lib.workspace_bytes(prm) + tensors > 180e9
    Q, K, V = syn.make_qkv(w, device="cuda")
    dO = syn.make_dout(w, device="cuda", out_dtype=torch.bfloat16)
    a = syn.make_amap(w, device="cuda")
    pl = _lib.plan(Q, K, V, a, prm, compact=True)
    O, lse = pl.attn_fwd()
    dQ, dK, dV = pl.attn_bwd(dO, O, lse)
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    used = core + pl._lists.numel()
    assert used + tensors < 180e9
    keep = {h: [t[h].clone() for t in (O, lse, dQ, dK, dV)] for h in (0, heads - 1)}
    items = {k: pl.export(k) for k in ("shape_id", "src")}
    del pl, O, lse, dQ, dK, dV
    torch.cuda.empty_cache()
    print(f"40-head 1M-token plan: core {core / 1e9:.1f} GB + lists {used / 1e9 - core / 1e9:.1f} GB")
    for h, got in keep.items():
        sl = slice(h, h + 1)
        p1, o1 = _run(Q[sl], K[sl], V[sl], a, dO[sl], _params(w, 1, out_dtype=_lib.PRISM_BF16), compact=True)
        np.testing.assert_array_equal(items["shape_id"].reshape(heads, -1)[h], p1.export("shape_id"))
        np.testing.assert_array_equal(items["src"].reshape(heads, -1)[h], p1.export("src"))
        for g, r, nm in zip(got, o1, ("O", "LSE", "dQ", "dK", "dV")):
            g, r = g.float().cpu(), r[0].float().cpu()
            if nm in ("O", "LSE"):
                assert torch.equal(g, r), f"head {h} {nm}"
            else:
                # bf16 outputs of fp32 sums taken in a different order: adjacent bf16
                # values (up to two ulps where the sums straddle a binade)
                diff = (g - r).abs()
                bound = 2.0 ** -6 * r.abs() + 2.0 ** -10 * r.abs().max()
                assert bool((diff <= bound).all()), f"head {h} {nm}: {diff.max().item():.3e}"


def test_native_4k_grid(cuda_device):
    w = syn.workload(3, H=176, W=320, top_k=16, top_p=0.0)
    assert w.N // 64 > 48 * 1024
    Q, K, V = syn.make_qkv(w, device="cuda", heads=1)
    dO = syn.make_dout(w, device="cuda", heads=1, out_dtype=torch.bfloat16).float()
    a = syn.make_amap(w, device="cuda")
    prm = _params(w, 1)
    pl = _lib.plan(Q, K, V, a, prm, compact=True)
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    q, k, v, g = (x[0].double().cpu().numpy() for x in (Q, K, V, dO))
    o = po.plan_head(q, k, v, a.cpu().numpy(), w.T, w.H, w.W, w.top_k, w.top_p, w.eps)
    NB, WORDS = w.N // 64, (w.N // 64 + 31) // 32
    _, tie, bad = parity.shapes_agree(pl.export("shape_id"), o["stats"])
    assert not bad
    if not tie:
        nb = len(o["starts"]) - 1
        np.testing.assert_array_equal(pl.export("blk_start")[:nb + 1], o["starts"])
        np.testing.assert_array_equal(pl.export("src"), o["src"])
        gsets = parity.bits_to_sets(pl.export("sel_bits").reshape(NB, WORDS), nb, WORDS)
        for i in range(nb):
            assert parity.selection_agrees(gsets[i], o["logits"][i], o["P"][i], w.top_k, w.top_p), i
    del pl
    # attention with the oracle's plan imported
    sid = torch.from_numpy(o["shape_id"].astype(np.uint8)[None]).cuda()
    bits = torch.from_numpy(parity.sets_to_bits(o["sel"], NB, WORDS)[None].view(np.int32)).cuda()
    pl = _lib.plan_import(Q, K, V, sid, bits, prm, compact=True)
    O, lse = pl.attn_fwd()
    dQ, dK, dV = pl.attn_bwd(dO, O, lse)
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    rng = np.random.default_rng(44)
    src, starts = o["src"], o["starts"]
    nb = len(starts) - 1
    blocks = np.unique(np.r_[0, nb - 1, rng.choice(nb, 30, replace=False)])
    rows = np.concatenate([rng.choice(src[starts[i]:starts[i + 1]], 3, replace=False) for i in blocks])
    Oo, lo, dQo = po.attention_rows(q, k, v, src, starts, o["sel"], rows, dO=g, chunk=16)
    good, rl2, ma = parity.close(O[0].double().cpu().numpy()[rows], Oo)
    assert good, f"O relL2 {rl2:.2e} maxabs {ma:.2e}"
    np.testing.assert_allclose(lse[0].double().cpu().numpy()[rows], lo, atol=2e-2, rtol=1e-3)
    good, rl2, ma, worst = parity.close_grad(dQ[0].double().cpu().numpy()[rows], dQo)
    assert good, f"dQ relL2 {rl2:.2e} maxabs {ma:.2e}"
    keys = np.unique(np.concatenate([src[:128:16], src[w.N - 128::16]] +
                                    [rng.choice(src[starts[j]:starts[j + 1]], 4, replace=False)
                                     for j in rng.choice(nb, 8, replace=False)]))
    dKo, dVo = po.attention_key_rows(q, k, v, g, src, starts, o["sel"], keys)
    for got, want, nm in ((dK, dKo, "dK"), (dV, dVo, "dV")):
        good, rl2, ma, worst = parity.close_grad(got[0].double().cpu().numpy()[keys], want)
        assert good, f"{nm} key rows relL2 {rl2:.2e} maxabs {ma:.2e}"
