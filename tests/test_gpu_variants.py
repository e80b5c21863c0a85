"""GPU parity of the ablation variants and of the pages' operating point.

"Prism: Dynamic Sparse Attention for Native 2K Joint Video-Audio Generation
Model Training": Table 10 (page xyznot.com/id) varies the shape-mapping
exponent alpha (1/3, 1/2, 2) and compares an isotropic mapping and fixed
blocks; page paper.rainbus.top sets the operating point Top-k 95% (k as a
sparsity: 5% of the blocks) and Top-p 0.2.  Each variant runs the GPU plan
and forward on a bf16 grid of 32 zones (16x32x32, head_dim 128, 2 heads)
against the oracle with the same parameters, under the parity rules of the
method's own tests; the operating point also runs the backward.
"""
import numpy as np
import pytest
import torch

import parity
from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn
from oracle import prism_oracle as po
from test_gpu_parity import _attn_inputs, _check_plan, _dout, _inputs, _rows_of_blocks, _to_dev

pytestmark = pytest.mark.gpu

W = syn.workload(2, T=16, H=32, W=32)
HEADS = 2

VARIANTS = {
    "alpha_one_third": dict(alpha=1.0 / 3.0),
    "alpha_two": dict(alpha=2.0),
    "isotropic": dict(shape_mode=_lib.PRISM_SHAPE_ISOTROPIC),
    "fixed_4x4x4": dict(shape_mode=_lib.PRISM_SHAPE_FIXED, fixed_shape=3),
    "fixed_4x8x8": dict(shape_mode=_lib.PRISM_SHAPE_FIXED, fixed_shape=13),
    "operating_point_k5pct_p0.2": dict(top_k_frac=0.05, top_p=0.2, top_k=0),
}


def _params(v):
    return _lib.make_params(W.T, W.H, W.W, HEADS, W.head_dim, _lib.PRISM_BF16, v.get("top_k", W.top_k),
                            v.get("top_p", W.top_p), W.eps, alpha=v.get("alpha", 0.5),
                            shape_mode=v.get("shape_mode", _lib.PRISM_SHAPE_DYNAMIC),
                            fixed_shape=v.get("fixed_shape", 0), top_k_frac=v.get("top_k_frac", 0.0))


def _oracle(Q, K, V, a, v):
    return [po.plan_head(Q[h].double().numpy(), K[h].double().numpy(), V[h].double().numpy(), a.numpy(),
                         W.T, W.H, W.W, v.get("top_k", W.top_k), v.get("top_p", W.top_p), W.eps,
                         alpha=v.get("alpha", 0.5), shape_mode=v.get("shape_mode", po.SHAPE_DYNAMIC),
                         fixed_shape=v.get("fixed_shape", 0), k_frac=v.get("top_k_frac", 0.0))
            for h in range(HEADS)]


def _k_of(v):
    frac = v.get("top_k_frac", 0.0)
    return (lambda nb: po.k_of_fraction(frac, nb)) if frac > 0 else v.get("top_k", W.top_k)


@pytest.mark.parametrize("name", list(VARIANTS))
def test_variant_plan_and_forward(name, cuda_device):
    v = VARIANTS[name]
    Q, K, V, a = _inputs(W, HEADS)
    Qd, Kd, Vd, ad = _to_dev(Q, K, V, a)
    pl = _lib.plan(Qd, Kd, Vd, ad, _params(v))
    O, lse = pl.attn_fwd()
    torch.cuda.synchronize()
    assert pl.status() == 0
    orc = _oracle(Q, K, V, a, v)
    if v.get("shape_mode") == _lib.PRISM_SHAPE_FIXED:
        sid = pl.export("shape_id").reshape(HEADS, W.zones)
        assert (sid == v["fixed_shape"]).all()
    if v.get("shape_mode") == _lib.PRISM_SHAPE_ISOTROPIC:
        sid = pl.export("shape_id").reshape(HEADS, W.zones)
        assert set(np.unique(sid).tolist()) <= {3, 8, 13}
    exact = _check_plan(pl, orc, W, HEADS, k=_k_of(v), p=v.get("top_p", W.top_p))
    O, lse = O.double().cpu().numpy(), lse.double().cpu().numpy()
    for h in range(HEADS):
        assert exact[h] is not None, f"{name} head {h}: shapes inside the tie margin"
        o = orc[h]
        Oo, lo = po.attention_fwd(*_attn_inputs(W, Q, K, V, h), o["src"], o["starts"], o["sel"])
        rows = _rows_of_blocks(o, exact[h])
        assert len(rows) >= 0.95 * W.N
        good, rl2, ma = parity.close(O[h][rows], Oo[rows])
        assert good, f"{name} head {h}: O relL2 {rl2:.2e} maxabs {ma:.2e}"
        np.testing.assert_allclose(lse[h][rows], lo[rows], atol=2e-2, rtol=1e-3)


def test_operating_point_backward(cuda_device):
    """The pages' operating point: plan, forward and backward on the GPU, every
    gradient element against the oracle where the whole plan agrees."""
    v = VARIANTS["operating_point_k5pct_p0.2"]
    Q, K, V, a = _inputs(W, HEADS)
    dO = _dout(W, HEADS)
    Qd, Kd, Vd, ad, dOd = _to_dev(Q, K, V, a, dO)
    pl = _lib.plan(Qd, Kd, Vd, ad, _params(v))
    O, lse = pl.attn_fwd()
    dQ, dK, dV = pl.attn_bwd(dOd, O, lse)
    torch.cuda.synchronize()
    assert pl.status() == 0
    orc = _oracle(Q, K, V, a, v)
    exact = _check_plan(pl, orc, W, HEADS, k=_k_of(v), p=v["top_p"])
    compared = 0
    for h in range(HEADS):
        o = orc[h]
        if exact[h] is None or len(exact[h]) != len(o["starts"]) - 1:
            continue
        ref = po.attention_bwd(*_attn_inputs(W, Q, K, V, h), dO[h].double().numpy(), o["src"],
                               o["starts"], o["sel"])
        for got, want, nm in zip((dQ, dK, dV), ref, ("dQ", "dK", "dV")):
            good, rl2, ma, worst = parity.close_grad(got[h].double().cpu().numpy(), want)
            assert good, f"head {h} {nm}: relL2 {rl2:.2e} maxabs {ma:.2e} worst {worst:.2f}"
        compared += 1
    assert compared >= 1, "no head whose whole selection matched the oracle"
