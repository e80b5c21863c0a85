"""The multi-GPU host logic of bench.py on CPU: two gloo ranks.

The hot path shards by head with no exchange; the only cross-rank steps are
the barrier and the max-over-ranks of the timings.  Two processes check that
their heads are disjoint and that every rank sees the slowest rank's time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        heads = bench.head_order(rank, world, need=9, heads=40)
        mx = bench.max_over_ranks(100.0 + 7.0 * rank, world)
        dist.barrier()
        out[rank] = (heads, mx)
    finally:
        dist.destroy_process_group()


def test_two_ranks_disjoint_heads_and_max_time():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    h0, m0 = out[0]
    h1, m1 = out[1]
    assert len(h0) == len(h1) == 9
    assert not set(h0) & set(h1)
    assert m0 == m1 == 107.0


def test_head_order_wraps():
    import bench
    assert bench.head_order(0, 1, 3, 40) == [0, 1, 2]
    assert bench.head_order(5, 8, 9, 40) == [(45 + i) % 40 for i in range(9)]
    with pytest.raises(TypeError):
        bench.head_order(0, 1)
