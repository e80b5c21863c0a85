"""Sequence-parallel callers: the exchange between sequence shards and head shards.

Prism's plan and attention need every token of a head on one GPU: the zone
statistics, the reorder and the block selection look at the whole latent grid.
A caller that holds the layer's activations sharded by sequence (the pages
train with sequence parallelism 8: page paper.rainbus.top, section
"方法步骤详情", training setup) therefore moves them to head shards first, runs
prism_plan / prism_attn_fwd / prism_attn_bwd on its heads, and moves the
results back:

    q_h = seq_to_heads(q_s)            # [H, N/P, D] -> [H/P, N, D]
    a   = gather_map(a_s)              # the guidance map is per token: replicate it
    ... plan / forward / backward on q_h, k_h, v_h ...
    o_s = heads_to_seq(o_h)            # [H/P, N, D] -> [H, N/P, D]

Rank r holds tokens [r N/P, (r + 1) N/P) of the raster order in the sequence
layout and heads [r H/P, (r + 1) H/P) in the head layout.  Each direction is one
all-to-all (NCCL over NVLink between GPUs; gloo on the host for the tests); the
plan itself needs no collective.  The library computes nothing here: this
module only moves tensors between ranks with torch.distributed.

Where the ranks' sequence shards are mapped into each other's address space
(`symmetric_shard`: torch symmetric memory), both exchanges can be left out:
`_lib.plan_sharded(qs, ks, vs, a, params, head0=h0, heads_total=H)` plans this
rank's heads (`rank_heads`) straight from every rank's Q, K, V shard (the
plan's reorder reads the other GPUs' rows over NVLink), and the plan's
`attn_fwd_sharded` / `attn_bwd_sharded` write O, dQ, dK, dV into (and read dO,
O from) the shards in place, so no all-to-all runs around the layer.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _world(group):
    return dist.get_world_size(group), dist.get_rank(group)


def symmetric_shard(shape, dtype, group=None):
    """A sequence shard in symmetric memory, for the `_sharded` entry points.

    Returns (t, addresses, handle): the local shard tensor `t` (write this rank's
    rows into it), every rank's shard mapped into this process as device addresses
    in rank order (pass them as the shard list), and the rendezvous handle, which
    must outlive every plan and launch that uses the addresses.  The ranks must have
    written their shards (a barrier on `group`, with the writes synchronised) before
    a kernel reads them, and must not reuse a shard while another rank's kernels may
    still read or write it.  Needs one GPU per rank with peer access (NVLink)."""
    import torch.distributed._symmetric_memory as symm_mem
    t = symm_mem.empty(*shape, dtype=dtype, device=torch.device("cuda", torch.cuda.current_device()))
    handle = symm_mem.rendezvous(t, group if group is not None else dist.group.WORLD)
    delta = t.data_ptr() - handle.buffer_ptrs[handle.rank]
    return t, [p + delta for p in handle.buffer_ptrs], handle


def rank_heads(rank: int, world: int, heads: int) -> tuple[int, int]:
    """(first head, head count) of `rank` in the head layout: heads [r H/P, (r + 1) H/P)."""
    if heads % world:
        raise ValueError(f"heads ({heads}) must be a multiple of the group size ({world})")
    return rank * (heads // world), heads // world


def seq_to_heads(x: torch.Tensor, group=None) -> torch.Tensor:
    """[H, N/P, D] (this rank's tokens, every head) -> [H/P, N, D] (this rank's heads, every token)."""
    P, _ = _world(group)
    H, n, D = x.shape
    if H % P:
        raise ValueError(f"heads ({H}) must be a multiple of the group size ({P})")
    # chunk p of the send buffer = the heads of rank p (contiguous along dim 0)
    send = x.reshape(P, H // P, n, D).contiguous()
    recv = torch.empty_like(send)                 # recv[q] = rank q's tokens of my heads
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 0, 2, 3).reshape(H // P, P * n, D).contiguous()


def heads_to_seq(y: torch.Tensor, group=None) -> torch.Tensor:
    """[H/P, N, D] (this rank's heads, every token) -> [H, N/P, D] (this rank's tokens, every head)."""
    P, _ = _world(group)
    h, N, D = y.shape
    if N % P:
        raise ValueError(f"tokens ({N}) must be a multiple of the group size ({P})")
    # chunk q of the send buffer = my heads' tokens of rank q
    send = y.reshape(h, P, N // P, D).permute(1, 0, 2, 3).contiguous()
    recv = torch.empty_like(send)                 # recv[p] = rank p's heads of my tokens
    dist.all_to_all_single(recv, send, group=group)
    return recv.reshape(P * h, N // P, D)


def gather_map(a_local: torch.Tensor, group=None) -> torch.Tensor:
    """The guidance map's token shards [N/P] -> the whole map [N] on every rank."""
    P, _ = _world(group)
    out = torch.empty(P * a_local.numel(), dtype=a_local.dtype, device=a_local.device)
    dist.all_gather_into_tensor(out, a_local.contiguous().reshape(-1), group=group)
    return out


__all__ = ["seq_to_heads", "heads_to_seq", "gather_map"]
