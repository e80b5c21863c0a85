"""Element-wise backward parity where the dK/dV kernel takes its multi-chunk path.

The dK/dV kernel runs one CTA per (128-key tile, chunk of 512 query tiles): a
key tile's partial dK and dV of each chunk are reduce-added into fp32
accumulators, which one finalize kernel scales and scatters to raster order.
Grids above 65,536 tokens therefore sum several chunks per key.  Cases, each
with the oracle's own shapes and selection imported (prism_plan_import), so
every key's set of attending queries is exactly the oracle's:
  * 8 x 64 x 144 (73,728 tokens, two chunks) at Top-k 16 / Top-p 0.6 (about
    a third of the token pairs: every key tile has long lists in both chunks):
    O, LSE, dQ, dK, dV compared in full;
  * 16 x 64 x 144 (147,456 tokens, three chunks) at the pages' operating point
    (k = 5% of the blocks, Top-p 0.2): O, LSE, dQ, dK, dV in full;
  * the 1080p-like grid 32 x 72 x 128 (294,912 tokens, five chunks) and the 2K
    grid 72 x 88 x 160 (1,013,760 tokens, sixteen chunks; the bench's launch
    configuration) with Top-k selections (k 32 and 16, p 0), dK and dV on
    sampled key rows (the first and the last key tile, and keys of 64-, 128- and
    256-token blocks spread over the grid) computed one by one by the oracle,
    O and dQ on sampled query rows.
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

CHUNK_TOKENS = 512 * 128


def _imported_run(w, k, p, k_frac=0.0):
    """Oracle plan of one head, imported; GPU forward and backward."""
    Q, K, V = syn.make_qkv(w, device="cuda", heads=1)
    a = syn.make_amap(w, device="cuda").cpu()
    dO = syn.make_dout(w, device="cuda", heads=1, out_dtype=torch.bfloat16).float()
    q, kk, v, g = (x[0].double().cpu().numpy() for x in (Q, K, V, dO))
    o = po.plan_head(q, kk, v, a.numpy(), w.T, w.H, w.W, k, p, w.eps, k_frac=k_frac)
    NB, WORDS = w.N // 64, (w.N // 64 + 31) // 32
    sid = torch.from_numpy(o["shape_id"].astype(np.uint8)[None]).cuda()
    bits = torch.from_numpy(parity.sets_to_bits(o["sel"], NB, WORDS)[None].view(np.int32)).cuda()
    prm = _lib.make_params(w.T, w.H, w.W, 1, w.head_dim, _lib.PRISM_BF16, k, p, w.eps, top_k_frac=k_frac)
    pl = _lib.plan_import(Q, K, V, sid, bits, prm)
    O, lse = pl.attn_fwd()
    dQ, dK, dV = pl.attn_bwd(dO, O, lse)
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    host = lambda t: t[0].double().cpu().numpy()
    return dict(q=q, k=kk, v=v, g=g, o=o, O=host(O), lse=lse[0].double().cpu().numpy(),
                dQ=host(dQ), dK=host(dK), dV=host(dV))


def _assert_close(got, want, what):
    good, rl2, ma = parity.close(got, want)
    assert good, f"{what}: relL2 {rl2:.2e} maxabs {ma:.2e}"


def _assert_grad(got, want, what):
    good, rl2, ma, worst = parity.close_grad(got, want)
    assert good, f"{what}: relL2 {rl2:.2e} maxabs {ma:.2e} (worst element at {worst:.2f} of its bound)"


@pytest.mark.parametrize("case", ["p06_2chunks", "operating_point_3chunks"])
def test_multichunk_backward_full(case, cuda_device):
    if case == "p06_2chunks":
        w = syn.workload(2, T=8, H=64, W=144)
        r = _imported_run(w, w.top_k, 0.6)
    else:
        w = syn.workload(2, T=16, H=64, W=144)
        r = _imported_run(w, 0, 0.2, k_frac=0.05)
    chunks = -(-w.N // CHUNK_TOKENS)
    assert chunks == (2 if case == "p06_2chunks" else 3)
    o = r["o"]
    Oo, lo = po.attention_fwd(r["q"], r["k"], r["v"], o["src"], o["starts"], o["sel"])
    _assert_close(r["O"], Oo, f"{case} O")
    np.testing.assert_allclose(r["lse"], lo, atol=2e-2, rtol=1e-3)
    ref = po.attention_bwd(r["q"], r["k"], r["v"], r["g"], o["src"], o["starts"], o["sel"])
    for got, want, nm in zip((r["dQ"], r["dK"], r["dV"]), ref, ("dQ", "dK", "dV")):
        _assert_grad(got, want, f"{case} {nm}")
        # per-key rows: no key tile's rows land elsewhere or cancel
        rows = np.linalg.norm(got - want, axis=1) / np.maximum(np.linalg.norm(want, axis=1), 1e-3)
        assert np.quantile(rows, 0.999) < 0.05, f"{case} {nm}: worst rows {np.sort(rows)[-5:]}"


def _sample_key_rows(o, N, rng, per_block=6):
    """Raster keys: the first and the last 128-key tile of the block order, and
    keys of blocks of each volume (64, 128, 256) spread over the grid."""
    src, starts = o["src"], o["starts"]
    vols = np.diff(starts)
    picks = [src[:128:8], src[N - 128::8]]
    for vol in (64, 128, 256):
        blocks = np.nonzero(vols == vol)[0]
        if len(blocks) == 0:
            continue
        for j in rng.choice(blocks, size=min(4, len(blocks)), replace=False):
            picks.append(rng.choice(src[starts[j]:starts[j + 1]], size=per_block, replace=False))
    return np.unique(np.concatenate(picks))


def _sample_query_rows(o, rng, nblocks=48, per_block=4):
    src, starts = o["src"], o["starts"]
    nb = len(starts) - 1
    blocks = np.unique(np.r_[0, nb - 1, rng.choice(nb, nblocks, replace=False)])
    return np.unique(np.concatenate([rng.choice(src[starts[i]:starts[i + 1]], per_block, replace=False)
                                     for i in blocks]))


@pytest.mark.parametrize("wid,k", [(2, 32), (3, 16)])
def test_fullsize_backward_sampled_key_rows(wid, k, cuda_device):
    w = syn.workload(wid)
    r = _imported_run(w, k, 0.0)
    o = r["o"]
    assert w.N > 4 * CHUNK_TOKENS
    rng = np.random.default_rng(11 + wid)
    keys = _sample_key_rows(o, w.N, rng)
    vols = np.diff(o["starts"])[po.block_of_token(o["src"], o["starts"])[keys]]
    assert {64, 128, 256} & set(vols.tolist())
    dKo, dVo = po.attention_key_rows(r["q"], r["k"], r["v"], r["g"], o["src"], o["starts"], o["sel"], keys)
    _assert_grad(r["dK"][keys], dKo, f"workload {wid} dK key rows")
    _assert_grad(r["dV"][keys], dVo, f"workload {wid} dV key rows")
    rows = _sample_query_rows(o, rng)
    Oo, lo, dQo = po.attention_rows(r["q"], r["k"], r["v"], o["src"], o["starts"], o["sel"], rows, dO=r["g"])
    _assert_close(r["O"][rows], Oo, f"workload {wid} O rows")
    _assert_grad(r["dQ"][rows], dQo, f"workload {wid} dQ rows")
    np.testing.assert_allclose(r["lse"][rows], lo, atol=2e-2, rtol=1e-3)
