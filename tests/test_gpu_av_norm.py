"""GPU parity of the guidance map producer (prism_av_norm) against the oracle.

a_{t,h,w} = ||h_hat_{t,h,w}||_2 with h_hat = CrossAttn(h, K_a, V_a) per head,
heads concatenated (page paper.rainbus.top, section "前置知识"; page
xyznot.com/id, section "Metode" 1).  Inputs are bf16; the oracle runs in
float64 on the same bf16 values.  Bars: h_hat within relative L2 1e-2 and
max-abs 3e-2 (the attention-output bars); the map within 1e-2 relative per
token, which the relative-L2 bar on each token's concatenated h_hat implies
(| ||x|| - ||y|| | <= ||x - y||).
"""
import numpy as np
import pytest
import torch

import parity
from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn
from oracle import prism_oracle as po

pytestmark = pytest.mark.gpu

MAP_REL = 1e-2


def _f64(x):
    return x.double().cpu().numpy()


def _check(Qv, Ka, Va, a, hh, rows=None):
    """Compares the map (every token, or `rows`) and h_hat against the oracle."""
    if rows is None:
        ao, ho = po.av_norm_map(_f64(Qv), _f64(Ka), _f64(Va))
        ag, hg = a.cpu().double().numpy(), None if hh is None else _f64(hh)
    else:
        # only the sampled rows leave the device (the full Qv would be 41 GB in float64)
        idx = torch.as_tensor(rows, device=Qv.device)
        ao, ho = po.av_norm_rows(_f64(Qv[:, idx]), _f64(Ka), _f64(Va), np.arange(len(rows)))
        ag = a.cpu().double().numpy()[rows]
        hg = None if hh is None else _f64(hh[:, idx.to(hh.device)])
    rel = np.abs(ag - ao) / np.maximum(ao, 1e-30)
    assert np.all(np.isfinite(ag))
    assert rel.max() <= MAP_REL, f"map: max relative error {rel.max():.3e} at token {int(rel.argmax())}"
    if hg is not None:
        for h in range(ho.shape[0]):
            good, rl2, ma = parity.close(hg[h], ho[h])
            assert good, f"h_hat head {h}: relL2 {rl2:.3e}, max-abs {ma:.3e}"
    return float(rel.max())


def _status_ok(status):
    st, site = _lib.status_read(status)
    assert st == _lib.PRISM_OK, f"device status {_lib.status_string(st)} at site {site}"


# name: (workload, heads, M, hhat dtype, q/k scale, tokens kept (None: the grid's))
CASES = {
    "tiny_d64_m100": (syn.workload(0), 2, 100, _lib.PRISM_BF16, 1.0, None),
    "grid16x32x32_d128_m1000": (syn.workload(2, T=16, H=32, W=32), 4, 1000, _lib.PRISM_F32, 1.0, None),
    "one_audio_token": (syn.workload(0), 2, 1, _lib.PRISM_F32, 1.0, None),
    "m64_half_tile": (syn.workload(1, T=8, H=16, W=16), 3, 64, _lib.PRISM_F32, 1.0, None),
    "m128_one_tile": (syn.workload(1, T=8, H=16, W=16), 1, 128, _lib.PRISM_F32, 1.0, None),
    "m129_one_key_tail": (syn.workload(1, T=8, H=16, W=16), 2, 129, _lib.PRISM_BF16, 1.0, None),
    "ragged_tokens_1000": (syn.workload(1, T=8, H=16, W=16), 3, 300, _lib.PRISM_F32, 1.0, 1000),
    "peaked_logits_x3": (syn.workload(1, T=8, H=16, W=16), 2, 700, _lib.PRISM_F32, 3.0, None),
    "diffuse_logits_x05": (syn.workload(1, T=8, H=16, W=16), 2, 700, _lib.PRISM_F32, 0.5, None),
}


@pytest.mark.parametrize("name", list(CASES))
def test_av_norm_matches_oracle(name, cuda_device):
    w, heads, M, hdt, scale, keep = CASES[name]
    Qv, Ka, Va = syn.make_av_inputs(w, M, heads=heads, qk_scale=scale)
    if keep is not None:
        Qv = Qv[:, :keep].contiguous()
    Qd, Kd, Vd = (x.cuda() for x in (Qv, Ka, Va))
    a, hh, status = _lib.av_norm(Qd, Kd, Vd, hhat_dtype=hdt, want_hhat=True)
    torch.cuda.synchronize()
    _status_ok(status)
    _check(Qv, Ka, Va, a, hh)


def test_map_alone_equals_map_with_hhat(cuda_device):
    """Without h_hat the kernel writes the same map, bit for bit."""
    w = syn.workload(2, T=16, H=32, W=32)
    Qd, Kd, Vd = (x.cuda() for x in syn.make_av_inputs(w, 500, heads=3))
    a1, _, s1 = _lib.av_norm(Qd, Kd, Vd, want_hhat=True)
    a2, h2, s2 = _lib.av_norm(Qd, Kd, Vd)
    torch.cuda.synchronize()
    _status_ok(s1)
    _status_ok(s2)
    assert h2 is None
    assert torch.equal(a1, a2)


def test_map_feeds_the_plan(cuda_device):
    """The produced map is the next layer's a_map: the plan built from it on the
    GPU takes the oracle's shapes for that same map (near-ties excepted)."""
    w = syn.workload(2, T=16, H=32, W=32)
    heads = 2
    Qv, Ka, Va = (x.cuda() for x in syn.make_av_inputs(w, 256, heads=4))
    amap, _, status = _lib.av_norm(Qv, Ka, Va)
    torch.cuda.synchronize()
    _status_ok(status)
    amap = amap.view(w.T, w.H, w.W)
    Q, K, V = syn.make_qkv(w, heads=heads)
    p = _lib.make_params(w.T, w.H, w.W, heads, w.head_dim, _lib.PRISM_BF16, w.top_k, w.top_p, w.eps)
    pl = _lib.plan(Q.cuda(), K.cuda(), V.cuda(), amap, p)
    sid = pl.export("shape_id").reshape(heads, w.zones)
    an = amap.cpu().numpy()
    for h in range(heads):
        st = po.zone_shapes(V[h].double().numpy(), an, w.T, w.H, w.W, w.eps)
        _, tie, bad = parity.shapes_agree(sid[h], st)
        assert not bad, f"head {h}: zones {bad} differ beyond the tie margin"


def test_full_size_sampled_rows(cuda_device):
    """The 2K layer (72x88x160 = 1,013,760 video tokens, 40 heads, D 128) with
    1,000 audio tokens, as the benchmark runs it: the map and h_hat on 384
    seeded rows (and the first and last) against the oracle row by row."""
    w = syn.workload(3)
    M = 1000
    Qv, Ka, Va = syn.make_av_inputs(w, M, device="cuda")
    a, hh, status = _lib.av_norm(Qv, Ka, Va, want_hhat=True)
    torch.cuda.synchronize()
    _status_ok(status)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, w.N - 1], rng.integers(0, w.N, 384)]))
    _check(Qv, Ka, Va, a, hh, rows=rows)
    assert bool(torch.isfinite(a).all()) and float(a.min()) > 0.0


def test_invalid_shapes_rejected(cuda_device):
    Qv = torch.zeros(2, 256, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.PrismError):
        _lib.av_norm(Qv, Qv[:, :10].contiguous(), Qv[:, :10].contiguous())
