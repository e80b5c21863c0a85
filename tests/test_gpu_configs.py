"""Parity at the full sizes of the remaining workloads, on sampled outputs.

  * 720p-like layer (grid 24 x 48 x 80, 92,160 tokens, 40 heads in one plan,
    Top-k 8, Top-p 0.9, forward only): shapes of every head and the selection of
    two heads against the oracle's plans, O on sampled rows of those heads;
  * 1080p-like training layer (grid 32 x 72 x 128, 294,912 tokens, Top-k 16,
    Top-p 0.9, forward and backward; two heads in one plan): the same plan
    checks, O and dQ on sampled rows, dV and dK through the identities that hold
    at any size (rows of dV sum to rows of dO, rows of dK sum to zero);
  * 2K inference sweep (grid 64 x 88 x 152, 856,064 tokens, forward: seven key
    range passes), the peaked (Q, K x 3) and diffuse (x 0.5) regimes at the
    sweep's corners (Top-k 8 / Top-p 0.8 and Top-k 32 / Top-p 0.95).
The comparison rules are those of tests/parity.py (near-tie margins of the
oracle for integer decisions; relative L2 1e-2 and max-abs 3e-2 for outputs).
"""
import numpy as np
import pytest
import torch

import parity
from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn
from oracle import prism_oracle as po

pytestmark = pytest.mark.gpu


def _host(t, h):
    return t[h].double().cpu().numpy()


def _plan_check(w, pl, heads_checked, Q, K, V, a, heads):
    """Shapes of every head within the tie rules; for `heads_checked`, the whole
    plan and the selection.  Returns the oracle plans and the exact-selection rows."""
    NB, WORDS, Nz = w.N // 64, (w.N // 64 + 31) // 32, w.zones
    sid = pl.export("shape_id").reshape(heads, Nz)
    bits = pl.export("sel_bits").reshape(heads, NB, WORDS)
    src = pl.export("src").reshape(heads, w.N)
    an = a.cpu().numpy()
    out = {}
    for h in range(heads):
        st = po.zone_shapes(_host(V, h), an, w.T, w.H, w.W, w.eps)
        _, tie, bad = parity.shapes_agree(sid[h], st)
        assert not bad, f"head {h}: zones {bad} differ beyond the tie margin"
        if h not in heads_checked:
            continue
        o = po.plan_head(_host(Q, h), _host(K, h), _host(V, h), an, w.T, w.H, w.W, w.top_k, w.top_p, w.eps)
        if tie:
            continue                                     # downstream stages may differ legitimately
        nb = len(o["starts"]) - 1
        np.testing.assert_array_equal(src[h], o["src"])
        gsets = parity.bits_to_sets(bits[h], nb, WORDS)
        exact = []
        for i in range(nb):
            assert parity.selection_agrees(gsets[i], o["logits"][i], o["P"][i], w.top_k, w.top_p), (h, i)
            if np.array_equal(gsets[i], o["sel"][i]):
                exact.append(i)
        assert len(exact) >= 0.99 * nb
        out[h] = (o, exact)
    return out


def _rows(o, exact, rng, nblocks=6):
    blocks = rng.permutation(exact)[:nblocks]
    return np.array([o["src"][o["starts"][i] + int(rng.integers(o["starts"][i + 1] - o["starts"][i]))]
                     for i in blocks])


def test_config_720p_forward(cuda_device):
    w = syn.workload(1)
    Q, K, V = syn.make_qkv(w, device="cuda")
    a = syn.make_amap(w, device="cuda")
    p = _lib.make_params(w.T, w.H, w.W, w.heads, w.head_dim, _lib.PRISM_BF16, w.top_k, w.top_p, w.eps)
    pl = _lib.plan(Q, K, V, a, p)
    O, lse = pl.attn_fwd()
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    checked = _plan_check(w, pl, (0, 23), Q, K, V, a, w.heads)
    rng = np.random.default_rng(11)
    for h, (o, exact) in checked.items():
        rows = _rows(o, exact, rng)
        Oo, lo, _ = po.attention_rows(_host(Q, h), _host(K, h), _host(V, h), o["src"], o["starts"], o["sel"], rows)
        good, rl2, ma = parity.close(_host(O, h)[rows], Oo)
        assert good, f"head {h}: O relL2 {rl2:.2e} maxabs {ma:.2e}"
        np.testing.assert_allclose(lse[h].double().cpu().numpy()[rows], lo, atol=2e-2, rtol=1e-3)


def test_config_1080p_forward_backward(cuda_device):
    w = syn.workload(2)
    heads = 2
    Q, K, V = syn.make_qkv(w, device="cuda", heads=heads)
    dO = syn.make_dout(w, device="cuda", heads=heads, out_dtype=torch.bfloat16).float()
    a = syn.make_amap(w, device="cuda")
    p = _lib.make_params(w.T, w.H, w.W, heads, w.head_dim, _lib.PRISM_BF16, w.top_k, w.top_p, w.eps)
    pl = _lib.plan(Q, K, V, a, p)
    O, lse = pl.attn_fwd()
    dQ, dK, dV = pl.attn_bwd(dO, O, lse)
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    checked = _plan_check(w, pl, (0, 1), Q, K, V, a, heads)
    rng = np.random.default_rng(12)
    for h, (o, exact) in checked.items():
        rows = _rows(o, exact, rng)
        Oo, lo, dQo = po.attention_rows(_host(Q, h), _host(K, h), _host(V, h), o["src"], o["starts"], o["sel"],
                                        rows, dO=_host(dO, h))
        good, rl2, ma = parity.close(_host(O, h)[rows], Oo)
        assert good, f"head {h} O: relL2 {rl2:.2e} maxabs {ma:.2e}"
        good, rl2, ma, worst = parity.close_grad(_host(dQ, h)[rows], dQo)
        assert good, f"head {h} dQ: relL2 {rl2:.2e} maxabs {ma:.2e} worst {worst:.2f}"
    for h in range(heads):
        dv, do_, dk = _host(dV, h), _host(dO, h), _host(dK, h)
        assert np.abs(dv.sum(0) - do_.sum(0)).max() <= 1e-2 * np.abs(dv).sum(0).max()
        assert np.abs(dk.sum(0)).max() <= 1e-2 * np.abs(dk).sum(0).max()


@pytest.mark.parametrize("scale,k,pp", [(3.0, 8, 0.8), (0.5, 32, 0.95)])
def test_config_2k_inference_sweep_corners(scale, k, pp, cuda_device):
    w = syn.workload(4, qk_scale=scale, top_k=k, top_p=pp)
    Q, K, V = syn.make_qkv(w, device="cuda", heads=1)
    a = syn.make_amap(w, device="cuda")
    p = _lib.make_params(w.T, w.H, w.W, 1, w.head_dim, _lib.PRISM_BF16, w.top_k, w.top_p, w.eps)
    pl = _lib.plan(Q, K, V, a, p)
    O, lse = pl.attn_fwd()
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    checked = _plan_check(w, pl, (0,), Q, K, V, a, 1)
    rng = np.random.default_rng(13)
    for h, (o, exact) in checked.items():
        rows = _rows(o, exact, rng)
        Oo, lo, _ = po.attention_rows(_host(Q, h), _host(K, h), _host(V, h), o["src"], o["starts"], o["sel"], rows)
        good, rl2, ma = parity.close(_host(O, h)[rows], Oo)
        assert good, f"O relL2 {rl2:.2e} maxabs {ma:.2e}"
