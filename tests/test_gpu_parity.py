"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Small grids that the oracle finishes in seconds but that still span several
zones, 128-token tiles and block volumes; plus the degenerate cases (every
block selected, a single block selected, one zone, no audio map).
"""
import numpy as np
import pytest
import torch

import parity
from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn
from oracle import prism_oracle as po

pytestmark = pytest.mark.gpu


def _dtype_code(w):
    return _lib.PRISM_F32 if w.dtype == "f32" else _lib.PRISM_BF16


def _inputs(w, heads, with_audio=True):
    Q, K, V = syn.make_qkv(w, heads=heads)
    a = syn.make_amap(w) if with_audio else None
    return Q, K, V, a


def _to_dev(*xs):
    return [None if x is None else x.cuda() for x in xs]


def _params(w, heads):
    return _lib.make_params(w.T, w.H, w.W, heads, w.head_dim, _dtype_code(w), w.top_k, w.top_p,
                            w.eps)


def _oracle_plans(w, Q, K, V, a, heads):
    an = None if a is None else a.numpy()
    return [po.plan_head(Q[h].double().numpy(), K[h].double().numpy(), V[h].double().numpy(), an,
                         w.T, w.H, w.W, w.top_k, w.top_p, w.eps) for h in range(heads)]


def _check_plan(pl, orc, w, heads, k=None, p=None):
    """Stage-wise comparison; returns per head the set of query blocks whose
    selection equals the oracle's exactly (None when the shapes differ).
    k (an int, or a function of the head's block count) and p default to the
    workload's."""
    p = w.top_p if p is None else p
    NB, WORDS, Nz, N = w.N // 64, (w.N // 64 + 31) // 32, w.zones, w.N
    sid = pl.export("shape_id").reshape(heads, Nz)
    nblocks = pl.export("nblocks")
    bstart = pl.export("blk_start").reshape(heads, NB + 1)
    src = pl.export("src").reshape(heads, N)
    qbar = pl.export("qbar").reshape(heads, NB, w.head_dim)
    kbar = pl.export("kbar").reshape(heads, NB, w.head_dim)
    bits = pl.export("sel_bits").reshape(heads, NB, WORDS)
    row_ptr = pl.export("row_ptr").reshape(heads, NB + 1)
    col_idx = pl.export("col_idx")
    loff = pl.export("list_offsets").reshape(4, heads)
    col_ptr = pl.export("col_ptr").reshape(heads, NB + 1)
    row_idx = pl.export("row_idx")
    exact_rows = []
    for h in range(heads):
        o = orc[h]
        ok, tie, bad = parity.shapes_agree(sid[h], o["stats"])
        assert not bad, f"head {h}: shape mismatch outside the tie margin in zones {bad}"
        if tie:
            exact_rows.append(None)
            continue
        nb = len(o["starts"]) - 1
        assert nblocks[h] == nb
        np.testing.assert_array_equal(bstart[h, :nb + 1], o["starts"])
        np.testing.assert_array_equal(src[h], o["src"])
        np.testing.assert_allclose(qbar[h, :nb], o["Qbar"], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(kbar[h, :nb], o["Kbar"], rtol=1e-5, atol=1e-6)
        gsets = parity.bits_to_sets(bits[h], nb, WORDS)
        kk = w.top_k if k is None else (k(nb) if callable(k) else k)
        exact = set()
        for i in range(nb):
            assert parity.selection_agrees(gsets[i], o["logits"][i], o["P"][i], kk, p), \
                f"head {h} row {i}: selection differs beyond the tie margin"
            if np.array_equal(gsets[i], o["sel"][i]):
                exact.add(i)
        # CSR rows = the bitmap rows; CSC = the transpose
        for i in range(nb):
            np.testing.assert_array_equal(col_idx[loff[0, h] + row_ptr[h, i]:loff[0, h] + row_ptr[h, i + 1]],
                                          gsets[i])
        cols = [[] for _ in range(nb)]
        for i in range(nb):
            for j in gsets[i]:
                cols[j].append(i)
        for j in range(nb):
            np.testing.assert_array_equal(row_idx[loff[1, h] + col_ptr[h, j]:loff[1, h] + col_ptr[h, j + 1]],
                                          cols[j])
        exact_rows.append(exact)
    return exact_rows


def _attn_inputs(w, Q, K, V, h):
    """Values the attention kernels compute on: the tensor-core operands are
    fp16, so fp32 inputs are rounded to fp16 (bf16 inputs convert exactly)."""
    if w.dtype == "f32":
        return [x[h].to(torch.float16).double().numpy() for x in (Q, K, V)]
    return [x[h].double().numpy() for x in (Q, K, V)]


def _rows_of_blocks(o, blocks):
    return np.concatenate([o["src"][o["starts"][i]:o["starts"][i + 1]] for i in sorted(blocks)])


CASES = {
    "tiny_fp32_d64": (syn.workload(0), 2, True),
    "grid16x32x32_bf16_d128": (syn.workload(2, T=16, H=32, W=32), 2, True),
    "grid8x8x8_single_zone_no_audio": (syn.workload(1, T=8, H=8, W=8), 1, False),
    "grid8x16x24_k1_p0": (syn.workload(1, T=8, H=16, W=24, top_k=1, top_p=0.0), 2, True),
    "grid16x16x16_all_blocks": (syn.workload(2, T=16, H=16, W=16, top_k=10 ** 6, top_p=0.0), 1, True),
    "grid8x16x16_p1": (syn.workload(0, top_p=1.0, top_k=1), 1, True),
}


PLAN_RUNS = [(n, False) for n in CASES] + [("tiny_fp32_d64", True), ("grid16x32x32_bf16_d128", True)]


@pytest.mark.parametrize("name,compact", PLAN_RUNS)
def test_plan_and_forward_match_oracle(name, compact, cuda_device):
    """compact: the workspace holds the core only and the index lists go to a
    buffer sized from their counts (prism_plan_list_bytes / attach_lists)."""
    w, heads, audio = CASES[name]
    Q, K, V, a = _inputs(w, heads, audio)
    Qd, Kd, Vd, ad = _to_dev(Q, K, V, a)
    pl = _lib.plan(Qd, Kd, Vd, ad, _params(w, heads), compact=compact)
    if compact:
        assert pl._ws.numel() < _lib.workspace_bytes(_params(w, heads)) and pl._lists is not None
    O, lse = pl.attn_fwd()
    torch.cuda.synchronize()
    assert pl.status() == 0
    orc = _oracle_plans(w, Q, K, V, a, heads)
    exact = _check_plan(pl, orc, w, heads)
    O, lse = O.double().cpu().numpy(), lse.double().cpu().numpy()
    for h in range(heads):
        if exact[h] is None:
            continue
        o = orc[h]
        Oo, lo = po.attention_fwd(*_attn_inputs(w, Q, K, V, h), o["src"], o["starts"], o["sel"])
        rows = _rows_of_blocks(o, exact[h])
        if w.dtype == "f32":       # against the unrounded fp32 inputs too, at the same bar
            Ou, _ = po.attention_fwd(Q[h].double().numpy(), K[h].double().numpy(),
                                     V[h].double().numpy(), o["src"], o["starts"], o["sel"])
            good, rl2, ma = parity.close(O[h][rows], Ou[rows])
            assert good, f"{name} head {h}: O vs unrounded inputs relL2 {rl2:.2e} maxabs {ma:.2e}"
        assert len(rows) >= 0.95 * w.N
        good, rl2, ma = parity.close(O[h][rows], Oo[rows])
        assert good, f"{name} head {h}: O relL2 {rl2:.2e} maxabs {ma:.2e}"
        np.testing.assert_allclose(lse[h][rows], lo[rows], atol=2e-2, rtol=1e-3)


@pytest.mark.parametrize("name", ["tiny_fp32_d64", "grid16x32x32_bf16_d128"])
def test_imported_oracle_plan_forward(name, cuda_device):
    """The oracle's own shapes and selection fed through prism_plan_import:
    every output row is compared."""
    w, heads, audio = CASES[name]
    Q, K, V, a = _inputs(w, heads, audio)
    orc = _oracle_plans(w, Q, K, V, a, heads)
    NB, WORDS = w.N // 64, (w.N // 64 + 31) // 32
    sid = np.stack([o["shape_id"] for o in orc]).astype(np.uint8)
    bits = np.stack([parity.sets_to_bits(o["sel"], NB, WORDS) for o in orc])
    Qd, Kd, Vd = _to_dev(Q, K, V)
    sid_d = torch.from_numpy(sid).cuda()
    bits_d = torch.from_numpy(bits.view(np.int32)).cuda()
    pl = _lib.plan_import(Qd, Kd, Vd, sid_d, bits_d, _params(w, heads))
    O, lse = pl.attn_fwd()
    torch.cuda.synchronize()
    assert pl.status() == 0
    O, lse = O.double().cpu().numpy(), lse.double().cpu().numpy()
    for h in range(heads):
        o = orc[h]
        Oo, lo = po.attention_fwd(*_attn_inputs(w, Q, K, V, h), o["src"], o["starts"], o["sel"])
        good, rl2, ma = parity.close(O[h], Oo)
        assert good, f"{name} head {h}: O relL2 {rl2:.2e} maxabs {ma:.2e}"
        np.testing.assert_allclose(lse[h], lo, atol=2e-2, rtol=1e-3)


def test_invalid_workspace_is_rejected(cuda_device):
    w = syn.workload(0)
    Q, K, V, a = _inputs(w, 1)
    Qd, Kd, Vd, ad = _to_dev(Q, K, V, a)
    p = _params(w, 1)
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(_lib.PrismError) as e:
        _lib.plan(Qd, Kd, Vd, ad, p, workspace=small)
    assert e.value.status == _lib.PRISM_ERR_WORKSPACE


def _dout(w, heads):
    """dO ~ N(0,1), cast to bf16 (as every synthetic tensor), held in fp32."""
    return syn.make_dout(w, heads=heads, out_dtype=torch.bfloat16).float()


@pytest.mark.parametrize("name", ["tiny_fp32_d64", "grid16x32x32_bf16_d128", "grid8x16x24_k1_p0"])
def test_imported_oracle_plan_backward(name, cuda_device):
    """dQ, dK, dV with the oracle's own plan imported: every element compared."""
    w, heads, audio = CASES[name]
    Q, K, V, a = _inputs(w, heads, audio)
    dO = _dout(w, heads)
    orc = _oracle_plans(w, Q, K, V, a, heads)
    NB, WORDS = w.N // 64, (w.N // 64 + 31) // 32
    sid = np.stack([o["shape_id"] for o in orc]).astype(np.uint8)
    bits = np.stack([parity.sets_to_bits(o["sel"], NB, WORDS) for o in orc])
    Qd, Kd, Vd, dOd = _to_dev(Q, K, V, dO)
    pl = _lib.plan_import(Qd, Kd, Vd, torch.from_numpy(sid).cuda(),
                          torch.from_numpy(bits.view(np.int32)).cuda(), _params(w, heads))
    O, lse = pl.attn_fwd()
    dQ, dK, dV = pl.attn_bwd(dOd, O, lse)
    torch.cuda.synchronize()
    assert pl.status() == 0
    for h in range(heads):
        o = orc[h]
        qa, ka, va = _attn_inputs(w, Q, K, V, h)
        ref = po.attention_bwd(qa, ka, va, dO[h].double().numpy(), o["src"], o["starts"], o["sel"])
        for got, want, nm in zip((dQ, dK, dV), ref, ("dQ", "dK", "dV")):
            good, rl2, ma, worst = parity.close_grad(got[h].double().cpu().numpy(), want)
            assert good, f"{name} head {h} {nm}: relL2 {rl2:.2e} maxabs {ma:.2e} worst {worst:.2f}"


def test_full_pipeline_backward_tiny(cuda_device):
    """GPU plan + forward + backward on the tiny fp32 workload against the oracle."""
    w, heads, audio = CASES["tiny_fp32_d64"]
    Q, K, V, a = _inputs(w, heads, audio)
    dO = _dout(w, heads)
    Qd, Kd, Vd, ad, dOd = _to_dev(Q, K, V, a, dO)
    pl = _lib.plan(Qd, Kd, Vd, ad, _params(w, heads))
    O, lse = pl.attn_fwd()
    dQ, dK, dV = pl.attn_bwd(dOd, O, lse)
    torch.cuda.synchronize()
    assert pl.status() == 0
    orc = _oracle_plans(w, Q, K, V, a, heads)
    exact = _check_plan(pl, orc, w, heads)
    for h in range(heads):
        o = orc[h]
        assert exact[h] is not None and len(exact[h]) == len(o["starts"]) - 1
        # against the fp16 rounding of the inputs (the tensor-core operands) and
        # against the unrounded fp32 inputs, at the same bar
        unrounded = [x[h].double().numpy() for x in (Q, K, V)]
        for inputs, what in ((_attn_inputs(w, Q, K, V, h), "fp16-rounded"), (unrounded, "unrounded")):
            Oo, _ = po.attention_fwd(*inputs, o["src"], o["starts"], o["sel"])
            good, rl2, ma = parity.close(O[h].double().cpu().numpy(), Oo)
            assert good, f"head {h} O vs {what} inputs: relL2 {rl2:.2e} maxabs {ma:.2e}"
            ref = po.attention_bwd(*inputs, dO[h].double().numpy(), o["src"], o["starts"], o["sel"])
            for got, want, nm in zip((dQ, dK, dV), ref, ("dQ", "dK", "dV")):
                good, rl2, ma, worst = parity.close_grad(got[h].double().cpu().numpy(), want)
                assert good, f"head {h} {nm} vs {what} inputs: relL2 {rl2:.2e} maxabs {ma:.2e} worst {worst:.2f}"


def _scaled_run(w, scales):
    """Plan from the oracle (imported), forward and backward on Q, K, V scaled by
    exact powers of two; returns the inputs as given and the outputs."""
    Q, K, V = syn.make_qkv(w, heads=1)
    Q, K, V = ((x.float() * f).to(torch.bfloat16) for x, f in zip((Q, K, V), scales))
    dO = _dout(w, 1)
    q, k, v = (x[0].double().numpy() for x in (Q, K, V))
    o = po.plan_head(q, k, v, None, w.T, w.H, w.W, w.top_k, w.top_p, w.eps)
    NB, WORDS = w.N // 64, (w.N // 64 + 31) // 32
    sid = torch.from_numpy(o["shape_id"].astype(np.uint8)[None]).cuda()
    bits = torch.from_numpy(parity.sets_to_bits(o["sel"], NB, WORDS)[None].view(np.int32)).cuda()
    pl = _lib.plan_import(Q.cuda(), K.cuda(), V.cuda(), sid, bits, _params(w, 1))
    O, lse = pl.attn_fwd()
    grads = pl.attn_bwd(dO.cuda(), O, lse)
    torch.cuda.synchronize()
    assert pl.status() == 0
    host = lambda t: t[0].double().cpu().numpy()
    return (q, k, v, dO[0].double().numpy(), o), host(O), [host(t) for t in grads]


@pytest.mark.parametrize("name,scales", [
    ("tiny_V", (1.0, 1.0, 2.0 ** -20)),                  # V ~ 1e-6: below fp16's normal range
    ("huge_V_tiny_Q_huge_K", (2.0 ** -20, 2.0 ** 20, 2.0 ** 20)),   # |K|, |V| ~ 1e6: beyond fp16's 65504
])
def test_any_input_magnitude_keeps_the_bar(name, scales, cuda_device):
    """The fp16 copies are scaled per head by exact powers of two, so inputs far
    below fp16's normal range or far beyond its largest value meet the usual bar
    against the oracle on the exact inputs.  Q 2^a, K 2^-a leaves the logits
    unchanged; O scales with V, dS with V, so dQ with K and V, dK with Q and V,
    and dV not at all (compared at unit scale)."""
    w = syn.workload(2, T=8, H=16, W=16)
    (q, k, v, g, o), O, (dQ, dK, dV) = _scaled_run(w, scales)
    sq, sk, sv = scales
    Oo, _ = po.attention_fwd(q, k, v, o["src"], o["starts"], o["sel"])
    good, rl2, ma = parity.close(O / sv, Oo / sv)
    assert good, f"{name} O: relL2 {rl2:.2e} maxabs {ma:.2e} (at unit scale)"
    rQ, rK, rV = po.attention_bwd(q, k, v, g, o["src"], o["starts"], o["sel"])
    for got, want, f, nm in ((dQ, rQ, sk * sv, "dQ"), (dK, rK, sq * sv, "dK"), (dV, rV, 1.0, "dV")):
        good, rl2, ma, worst = parity.close_grad(got / f, want / f)
        assert good, f"{name} {nm}: relL2 {rl2:.2e} maxabs {ma:.2e} (at unit scale)"
