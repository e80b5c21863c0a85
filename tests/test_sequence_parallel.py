"""Sequence-shard <-> head-shard exchange on host ranks (gloo, 2 and 4 processes).

Every rank builds the same global [H, N, D] tensor from one seed and keeps its
token slice; seq_to_heads must give exactly the global tensor's head slice of
the rank (every token), heads_to_seq must undo it bit for bit, and gather_map
must rebuild the whole per-token map on every rank; rank_heads must name the
rank's head slice (the head range a sharded plan on that rank covers).
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out, H, N, D):
    import torch.distributed as dist
    from dynamic_block_sparse_indicator_b200 import sequence_parallel as sp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(7)
        full = torch.randn(H, N, D, generator=g)
        amap = torch.rand(N, generator=g)
        n, h = N // world, H // world
        local = full[:, rank * n:(rank + 1) * n].contiguous()
        heads = sp.seq_to_heads(local)
        ok_fwd = torch.equal(heads, full[rank * h:(rank + 1) * h])
        back = sp.heads_to_seq(heads)
        ok_back = torch.equal(back, local)
        whole = sp.gather_map(amap[rank * n:(rank + 1) * n])
        ok_map = torch.equal(whole, amap)
        shape_ok = tuple(heads.shape) == (h, N, D) and tuple(back.shape) == (H, n, D)
        bad = False
        try:
            sp.seq_to_heads(local[:H - 1] if H > 1 else local)   # heads not a multiple of the group
        except ValueError:
            bad = True
        h0, nh = sp.rank_heads(rank, world, H)
        ok_range = (h0, nh) == (rank * h, h) and torch.equal(heads, full[h0:h0 + nh])
        out[rank] = (ok_fwd, ok_back, ok_map, shape_ok, bad, ok_range)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,H,N,D", [(2, 4, 96, 8), (4, 8, 64, 16)])
def test_seq_head_exchange(world, H, N, D):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out, H, N, D)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    for r in range(world):
        assert out[r] == (True, True, True, True, True, True), (r, out[r])
