"""Head sharding on one GPU: the plan, forward and backward of a layer split by
head over two calls equal the one-call result.

The path shards by head with no exchange (every statistic, normalisation and
selection of the plan is per head; the audio terms depend only on the map), so
ranks that each take a contiguous range of heads (bench.py's head_order, two
ranks) must reproduce the one-call plan bit for bit and the one-call outputs:
O and LSE bit for bit (each query tile is reduced in one fixed order), dK and
dV bit for bit on a one-chunk grid (each key tile's sums stay in TMEM and are
added once into zeroed accumulators), and dQ to fp32 rounding (its partial sums
from different key tiles are reduce-added in the order the CTAs finish: within
1e-5 of the tensor's largest magnitude).  The
two "ranks" run one after the other on the same GPU; nothing waits on the other.
"""
import numpy as np
import pytest
import torch

import bench
from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

ITEMS = ("shape_id", "nblocks", "blk_start", "src", "sel_bits", "qbar", "kbar")


def _run(Q, K, V, dO, a, w, heads):
    p = _lib.make_params(w.T, w.H, w.W, heads, w.head_dim, _lib.PRISM_BF16, w.top_k, w.top_p, w.eps)
    pl = _lib.plan(Q, K, V, a, p)
    O, lse = pl.attn_fwd()
    dQ, dK, dV = pl.attn_bwd(dO, O, lse)
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    items = {k: pl.export(k) for k in ITEMS}
    return items, (O, lse, dQ, dK, dV)


@pytest.mark.parametrize("wid,grid", [(2, (16, 32, 32)), (0, (8, 16, 16))])
def test_two_head_shards_equal_one_call(wid, grid, cuda_device):
    T, H, W = grid
    w = syn.workload(wid, T=T, H=H, W=W, head_dim=128 if wid else 64, dtype="bf16",
                     **({} if wid else dict(eps=1e-4)))
    heads, world = 4, 2
    Q, K, V = syn.make_qkv(w, device="cuda", heads=heads)
    dO = syn.make_dout(w, device="cuda", heads=heads, out_dtype=torch.bfloat16).float()
    a = syn.make_amap(w, device="cuda")
    whole_items, whole = _run(Q, K, V, dO, a, w, heads)
    per = heads // world
    NB, Nz = w.N // 64, w.zones
    for rank in range(world):
        hs = bench.head_order(rank, world, per, heads)
        assert hs == list(range(hs[0], hs[0] + per))       # a contiguous range: a view of the tensors
        sl = slice(hs[0], hs[0] + per)
        items, outs = _run(Q[sl], K[sl], V[sl], dO[sl], a, w, per)
        shape = {"shape_id": (Nz,), "nblocks": (), "blk_start": (NB + 1,), "src": (w.N,),
                 "sel_bits": (NB, (NB + 31) // 32), "qbar": (NB, w.head_dim), "kbar": (NB, w.head_dim)}
        nbs = whole_items["nblocks"][sl]
        for k in ITEMS:
            got = items[k].reshape(per, *shape[k])
            want = whole_items[k].reshape(heads, *shape[k])[sl]
            if k in ("qbar", "kbar"):      # rows past a head's block count are padding
                for i in range(per):
                    np.testing.assert_array_equal(got[i, :nbs[i]], want[i, :nbs[i]], err_msg=f"rank {rank} {k}")
                continue
            np.testing.assert_array_equal(got, want, err_msg=f"rank {rank} {k}")
        for got, want, nm in zip(outs, whole, ("O", "LSE", "dQ", "dK", "dV")):
            g, r = got.cpu(), want[sl].cpu()
            if nm == "dQ":
                # fp32 sums of the key tiles' partial dQ, in the order the CTAs finish
                diff, scale = (g - r).abs().max().item(), r.abs().max().item()
                assert diff <= 1e-5 * scale, f"rank {rank} dQ: max diff {diff:.3e} at scale {scale:.3e}"
            else:
                assert torch.equal(g, r), f"rank {rank} {nm}: max diff {(g - r).abs().max().item():.3e}"
