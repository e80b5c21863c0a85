"""Plans read straight from sequence shards (prism_plan_sharded) on one GPU.

A sequence-parallel rank holds frames [s T/P, (s + 1) T/P) of every head; the
sharded plan of a head range reads every shard's rows itself (on several GPUs
through peer mappings), so no all-to-all precedes it.  Here the P shards are
separate buffers on one GPU standing in for the ranks' memory.  For every head
range (the ranks of the head layout) the sharded plan must equal prism_plan on
the gathered heads: shapes, block offsets, permutation, pooled means of every
block, the per-head input maxima and the selection bit for bit, O and LSE bit for bit, the
gradients to fp32 summation order.  Cases: bf16 with 4 shards of 4 frames
(every 8-frame zone spans two shards) and adaptive temporal boundaries on, and
the fp32 tiny workload with 2 shards.  The forward and the backward in the
shard layout (prism_attn_fwd_sharded, prism_attn_bwd_sharded): every rank's
rows of O, dQ, dK, dV land in the shards equal to the gathered run's.  The
sharded import (prism_plan_import_sharded) rebuilds a sharded plan from its own
shapes, splits and selection.  sequence_parallel.symmetric_shard, in an NCCL
group of one rank, gives shard addresses the sharded plan reads.  Invalid shard
counts and head ranges are rejected before any launch.
"""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

ITEMS = ("shape_id", "nblocks", "blk_start", "src", "sel_bits", "qkv_max")


def _shards(x, P):
    n = x.shape[1] // P
    return [x[:, s * n:(s + 1) * n].contiguous() for s in range(P)]


def _run(pl, dO):
    O, lse = pl.attn_fwd()
    grads = pl.attn_bwd(dO, O, lse)
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    return (O, lse) + tuple(grads)


@pytest.mark.parametrize("case", ["bf16_4shards_cuts", "f32_2shards"])
def test_sharded_plan_equals_gathered_plan(case, cuda_device):
    if case == "bf16_4shards_cuts":
        w = syn.workload(2, T=16, H=32, W=32, shot_cuts=[6])
        P, heads, ranks, cut, dt = 4, 4, 2, 2.5, _lib.PRISM_BF16
    else:
        w = syn.workload(0)
        P, heads, ranks, cut, dt = 2, 2, 2, 0.0, _lib.PRISM_F32
    Q, K, V = syn.make_qkv(w, device="cuda", heads=heads)
    dO = syn.make_dout(w, device="cuda", heads=heads, out_dtype=torch.bfloat16).float()
    a = syn.make_amap(w, device="cuda")
    qs, ks, vs = _shards(Q, P), _shards(K, P), _shards(V, P)
    nh = heads // ranks
    for r in range(ranks):
        h0 = r * nh
        sl = slice(h0, h0 + nh)
        prm = _lib.make_params(w.T, w.H, w.W, nh, w.head_dim, dt, w.top_k, w.top_p, w.eps, cut_ratio=cut)
        ref = _lib.plan(Q[sl].contiguous(), K[sl].contiguous(), V[sl].contiguous(), a, prm)
        got = _lib.plan_sharded(qs, ks, vs, a, prm, head0=h0, heads_total=heads)
        for item in ITEMS + (("zone_cut", "shape_id2") if cut else ()):
            np.testing.assert_array_equal(got.export(item), ref.export(item), err_msg=f"{case} rank {r} {item}")
        # pooled means of each head's blocks (rows past a head's block count are not written)
        nb = ref.export("nblocks")
        for item in ("qbar", "kbar"):
            gm, rm = (x.export(item).reshape(nh, w.N // 64, w.head_dim) for x in (got, ref))
            for h in range(nh):
                np.testing.assert_array_equal(gm[h, :nb[h]], rm[h, :nb[h]], err_msg=f"{case} rank {r} {item} {h}")
        g_out, r_out = _run(got, dO[sl].contiguous()), _run(ref, dO[sl].contiguous())
        for g, e, nm in zip(g_out, r_out, ("O", "LSE", "dQ", "dK", "dV")):
            g, e = g.cpu(), e.cpu()
            if nm in ("O", "LSE"):
                assert torch.equal(g, e), f"{case} rank {r} {nm}"
            else:                      # partial sums reduced in the order the CTAs finish
                diff, scale = (g - e).abs().max().item(), e.abs().max().item()
                assert diff <= 1e-5 * scale, f"{case} rank {r} {nm}: {diff:.3e} at scale {scale:.3e}"


@pytest.mark.parametrize("case", ["bf16_4shards", "f32_2shards"])
def test_sequence_parallel_round_trip_in_place(case, cuda_device):
    """Every rank plans its heads from the shards and runs the forward and the
    backward with O, dO, dQ, dK, dV in the shard layout: the shards then hold
    exactly the gathered run's outputs (O bit for bit, the gradients to fp32
    summation order), with no exchange outside the kernels."""
    if case == "bf16_4shards":
        w = syn.workload(2, T=16, H=32, W=32)
        P, heads, ranks, dt = 4, 4, 2, _lib.PRISM_BF16
    else:
        w = syn.workload(0)
        P, heads, ranks, dt = 2, 2, 2, _lib.PRISM_F32
    Q, K, V = syn.make_qkv(w, device="cuda", heads=heads)
    dO = syn.make_dout(w, device="cuda", heads=heads, out_dtype=torch.float32)
    a = syn.make_amap(w, device="cuda")
    qs, ks, vs, dos = _shards(Q, P), _shards(K, P), _shards(V, P), _shards(dO, P)
    n = w.N // P
    mk = lambda: [torch.full((heads, n, w.head_dim), float("nan"), device="cuda") for _ in range(P)]
    o_s, dq_s, dk_s, dv_s = mk(), mk(), mk(), mk()
    nh = heads // ranks
    want = {}
    for r in range(ranks):
        h0 = r * nh
        sl = slice(h0, h0 + nh)
        prm = _lib.make_params(w.T, w.H, w.W, nh, w.head_dim, dt, w.top_k, w.top_p, w.eps)
        pl = _lib.plan_sharded(qs, ks, vs, a, prm, head0=h0, heads_total=heads)
        lse = pl.attn_fwd_sharded(o_s, h0, heads)
        torch.cuda.synchronize()
        pl.attn_bwd_sharded(dos, o_s, lse, dq_s, dk_s, dv_s, h0, heads)
        torch.cuda.synchronize()
        assert pl.status() == _lib.PRISM_OK
        ref = _lib.plan(Q[sl].contiguous(), K[sl].contiguous(), V[sl].contiguous(), a, prm)
        want[r] = _run(ref, dO[sl].contiguous())
    gather = lambda xs: torch.cat([x.cpu() for x in xs], dim=1)
    got = {nm: gather(xs) for nm, xs in (("O", o_s), ("dQ", dq_s), ("dK", dk_s), ("dV", dv_s))}
    for r in range(ranks):
        sl = slice(r * nh, (r + 1) * nh)
        for nm, e in zip(("O", "dQ", "dK", "dV"), (want[r][0], want[r][2], want[r][3], want[r][4])):
            g, e = got[nm][sl], e.cpu()
            if nm == "O":
                assert torch.equal(g, e), f"{case} rank {r} O"
            else:
                diff, scale = (g - e).abs().max().item(), e.abs().max().item()
                assert diff <= 1e-5 * scale, f"{case} rank {r} {nm}: {diff:.3e} at scale {scale:.3e}"


def test_sharded_import_equals_sharded_plan(cuda_device):
    """prism_plan_import_sharded given a sharded plan's own shapes, splits and
    selection rebuilds that plan: the reorder and pooling from the shards, and
    the forward, bit for bit."""
    w = syn.workload(2, T=16, H=32, W=32, shot_cuts=[6])
    P, heads, nh, h0 = 4, 4, 2, 2
    Q, K, V = syn.make_qkv(w, device="cuda", heads=heads)
    a = syn.make_amap(w, device="cuda")
    qs, ks, vs = _shards(Q, P), _shards(K, P), _shards(V, P)
    prm = _lib.make_params(w.T, w.H, w.W, nh, w.head_dim, _lib.PRISM_BF16, w.top_k, w.top_p, w.eps, cut_ratio=2.5)
    pl = _lib.plan_sharded(qs, ks, vs, a, prm, head0=h0, heads_total=heads)
    dev = lambda item, dt: torch.from_numpy(pl.export(item).view(dt)).cuda()
    sid, cut, sid2 = dev("shape_id", np.uint8), dev("zone_cut", np.uint8), dev("shape_id2", np.uint8)
    bits = dev("sel_bits", np.int32)
    im = _lib.plan_import_sharded(qs, ks, vs, sid, bits, prm, head0=h0, heads_total=heads, zone_cut=cut,
                                  shape_id2=sid2)
    for item in ("blk_start", "src", "sel_bits", "qkv_max"):
        np.testing.assert_array_equal(im.export(item), pl.export(item), err_msg=item)
    O1, l1 = pl.attn_fwd()
    O2, l2 = im.attn_fwd()
    torch.cuda.synchronize()
    assert im.status() == _lib.PRISM_OK
    assert torch.equal(O1, O2) and torch.equal(l1, l2)


def test_sharded_plan_rejects_bad_layouts(cuda_device):
    w = syn.workload(0)
    Q, K, V = syn.make_qkv(w, device="cuda", heads=2)
    a = syn.make_amap(w, device="cuda")
    prm = _lib.make_params(w.T, w.H, w.W, 2, w.head_dim, _lib.PRISM_F32, w.top_k, w.top_p, w.eps)
    N = w.N
    # 3 shards do not divide T = 8 (rejected by the binding before the call)
    with pytest.raises(ValueError):
        _lib.plan_sharded([Q] * 3, [K] * 3, [V] * 3, a, prm)
    qs, ks, vs = _shards(Q, 2), _shards(K, 2), _shards(V, 2)
    # the head range runs past the shards' heads: rejected by the library
    with pytest.raises(_lib.PrismError) as e:
        _lib.plan_sharded(qs, ks, vs, a, prm, head0=1, heads_total=2)
    assert e.value.status == _lib.PRISM_ERR_INVALID_ARG
    # a misaligned shard address
    with pytest.raises(_lib.PrismError) as e:
        _lib.plan_sharded([qs[0].data_ptr() + 4, qs[1].data_ptr()], ks, vs, a, prm, heads_total=2)
    assert e.value.status == _lib.PRISM_ERR_INVALID_ARG
    assert N % 2 == 0


SYMM_CHILD = r"""
import os, sys, json
import torch, torch.distributed as dist
sys.path.insert(0, sys.argv[1])
from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import sequence_parallel as sp
from dynamic_block_sparse_indicator_b200 import synthetic as syn
os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=sys.argv[2], RANK="0", WORLD_SIZE="1")
torch.cuda.set_device(0)
dist.init_process_group("nccl", rank=0, world_size=1)
try:
    w = syn.workload(0)
    Q, K, V = syn.make_qkv(w, device="cuda", heads=2)
    a = syn.make_amap(w, device="cuda")
    shards, keep = [], []
    for x in (Q, K, V):
        t, addrs, h = sp.symmetric_shard(tuple(x.shape), x.dtype)
        t.copy_(x)
        keep.append((t, h))
        shards.append(addrs)
    torch.cuda.synchronize()
    dist.barrier()
    prm = _lib.make_params(w.T, w.H, w.W, 2, w.head_dim, _lib.PRISM_F32, w.top_k, w.top_p, w.eps)
    got = _lib.plan_sharded(shards[0], shards[1], shards[2], a, prm, heads_total=2)
    ref = _lib.plan(Q, K, V, a, prm)
    O1, _ = got.attn_fwd()
    O2, _ = ref.attn_fwd()
    torch.cuda.synchronize()
    same = bool(torch.equal(O1, O2)) and got.status() == 0
    print(json.dumps({"same": same, "n": len(shards[0])}))
    del got, ref
finally:
    dist.destroy_process_group()
"""


def test_symmetric_shard_single_rank(cuda_device, tmp_path):
    """symmetric_shard on one rank (NCCL group of one): its address list feeds
    plan_sharded, whose forward equals prism_plan's."""
    import json
    import os
    import socket
    import subprocess
    import sys
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    script = tmp_path / "child.py"
    script.write_text(SYMM_CHILD)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, str(script), root, str(port)], capture_output=True, text=True,
                         timeout=300, env=dict(os.environ, NCCL_NVLS_ENABLE="0"))
    assert res.returncode == 0, res.stderr[-3000:]
    out = json.loads(res.stdout.strip().splitlines()[-1])
    assert out == {"same": True, "n": 1}
