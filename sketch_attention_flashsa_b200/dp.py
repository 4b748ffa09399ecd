"""Data parallelism over users: one process per GPU, torch.distributed for the plumbing.

Every (user, head) of Sketch Attention is an independent problem (SequenceO1 §3.1: each user's
history is summarised by the shared prototypes on its own), so users shard across ranks with
no exchange in the forward. The backward has one: when the prototypes are shared by all users,
dQ is a sum over every user's contribution, hence a sum all-reduce of the [H, k, d] fp32
gradient (per-user prototypes need none). Host logic only; the compute runs in libska.so.
"""
from __future__ import annotations

import numpy as np


def partition_users(lengths, world: int) -> list[list[int]]:
    """Users -> ranks, balanced by valid history length (longest first onto the least-loaded rank,
    ties to the lower rank). Returns each rank's user indices in ascending order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    lengths = [int(x) for x in lengths]
    load = [0] * world
    parts: list[list[int]] = [[] for _ in range(world)]
    for u in sorted(range(len(lengths)), key=lambda i: (-lengths[i], i)):
        r = min(range(world), key=lambda j: (load[j], j))
        parts[r].append(u)
        load[r] += lengths[u]
    return [sorted(p) for p in parts]


def shard_ragged(cu_seqlens, users):
    """Token rows and the local cu_seqlens of a subset of users of a ragged batch.
    cu_seqlens: host int array [B+1]. Returns (row index array, local cu_seqlens int32)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    rows = [np.arange(cu[u], cu[u + 1]) for u in users]
    lens = [cu[u + 1] - cu[u] for u in users]
    local_cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32) if users else np.zeros(1, np.int32)
    return (np.concatenate(rows) if rows else np.zeros(0, np.int64)), local_cu


def allreduce_dq(dq, group=None):
    """Sum the shared prototypes' gradient over ranks, in place (no-op on one rank)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(dq, op=dist.ReduceOp.SUM, group=group)
    return dq


def max_over_ranks(values, device=None, group=None):
    """Element-wise max of a list of floats over ranks (the timing rule for multi-GPU numbers)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return [float(x) for x in t.cpu()]


def sum_over_ranks(values, device=None, group=None):
    """Element-wise sum of a list of floats over ranks (whole-job totals of per-rank work)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return [float(x) for x in t.cpu()]


def sa_backward_data_parallel(q, k, v, cu_seqlens, seqused, lse, dsketch, sketch=None, *, scale=1.0,
                              norm="proto", group=None, **kw):
    """Backward of this rank's users followed by the dQ all-reduce when the prototypes are shared
    (q of shape [H, k, d]); per-user prototypes ([B, H, k, d]) keep their local dQ."""
    from . import api
    dq, dk, dv = api.sa_backward(q, k, v, cu_seqlens, seqused, lse, dsketch, sketch, scale=scale, norm=norm, **kw)
    if q.dim() == 3:
        allreduce_dq(dq, group)
    return dq, dk, dv
