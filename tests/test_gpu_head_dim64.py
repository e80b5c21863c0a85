"""head_dim 64 with bf16 inputs: the kernels' D = 64 instances on a two-chunk grid.

The other parity cases run head_dim 64 only with fp32 inputs on a one-chunk
grid (the tiny workload).  Here a bf16 8 x 64 x 144 grid (73,728 tokens, 1,152
blocks at most, two query chunks of the dK/dV kernel) at head_dim 64:
  * the plan (zone statistics, shapes, block offsets, permutation, pooled
    means, every selected set) against the oracle's, with the near-tie rules;
  * with the oracle's plan imported, O, LSE, dQ, dK and dV element by element
    (the dK/dV kernel without the fused dQ, and the separate dQ kernel over the
    forward lists, whose partial sums are not reduced across chunks).
Tolerances (tests/parity.py): relative L2 <= 1e-2 and max-abs <= 3e-2; for the
gradients max-abs 3e-2 plus half a bf16 ulp of each element.
"""
import numpy as np
import pytest
import torch

import parity
from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn
from oracle import prism_oracle as po

pytestmark = pytest.mark.gpu


def test_bf16_head_dim_64_two_chunks(cuda_device):
    w = syn.workload(2, T=8, H=64, W=144, head_dim=64, top_p=0.6)
    assert w.N > 512 * 128
    Q, K, V = syn.make_qkv(w, device="cuda", heads=1)
    a = syn.make_amap(w, device="cuda")
    dO = syn.make_dout(w, device="cuda", heads=1, out_dtype=torch.bfloat16).float()
    prm = _lib.make_params(w.T, w.H, w.W, 1, 64, _lib.PRISM_BF16, w.top_k, w.top_p, w.eps)
    q, k, v, g = (x[0].double().cpu().numpy() for x in (Q, K, V, dO))
    o = po.plan_head(q, k, v, a.cpu().numpy(), w.T, w.H, w.W, w.top_k, w.top_p, w.eps)
    NB, WORDS = w.N // 64, (w.N // 64 + 31) // 32

    # the GPU plan against the oracle's
    pl = _lib.plan(Q, K, V, a, prm)
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    _, tie, bad = parity.shapes_agree(pl.export("shape_id"), o["stats"])
    assert not bad
    if not tie:
        nb = len(o["starts"]) - 1
        np.testing.assert_array_equal(pl.export("blk_start")[:nb + 1], o["starts"])
        np.testing.assert_array_equal(pl.export("src"), o["src"])
        np.testing.assert_allclose(pl.export("qbar").reshape(NB, 64)[:nb], o["Qbar"], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(pl.export("kbar").reshape(NB, 64)[:nb], o["Kbar"], rtol=1e-5, atol=1e-6)
        gsets = parity.bits_to_sets(pl.export("sel_bits").reshape(NB, WORDS), nb, WORDS)
        for i in range(nb):
            assert parity.selection_agrees(gsets[i], o["logits"][i], o["P"][i], w.top_k, w.top_p), i
    del pl

    # forward and backward with the oracle's plan imported
    sid = torch.from_numpy(o["shape_id"].astype(np.uint8)[None]).cuda()
    bits = torch.from_numpy(parity.sets_to_bits(o["sel"], NB, WORDS)[None].view(np.int32)).cuda()
    pl = _lib.plan_import(Q, K, V, sid, bits, prm)
    O, lse = pl.attn_fwd()
    dQ, dK, dV = pl.attn_bwd(dO, O, lse)
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    host = lambda t: t[0].double().cpu().numpy()
    Oo, lo = po.attention_fwd(q, k, v, o["src"], o["starts"], o["sel"])
    good, rl2, ma = parity.close(host(O), Oo)
    assert good, f"O relL2 {rl2:.2e} maxabs {ma:.2e}"
    np.testing.assert_allclose(host(lse), lo, atol=2e-2, rtol=1e-3)
    ref = po.attention_bwd(q, k, v, g, o["src"], o["starts"], o["sel"])
    for got, want, nm in zip((dQ, dK, dV), ref, ("dQ", "dK", "dV")):
        good, rl2, ma, worst = parity.close_grad(host(got), want)
        assert good, f"{nm}: relL2 {rl2:.2e} maxabs {ma:.2e} (worst element at {worst:.2f} of its bound)"
