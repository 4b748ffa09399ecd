"""The multi-rank host path on CPU: world_size-2 process groups over gloo. Users are sharded
across ranks (balanced by history length); the forward needs no exchange, and the backward's
shared-prototype dQ is a sum all-reduce. The per-rank compute is the oracle here (test side),
so these check the partitioning, the row mapping and the collectives, not the kernels."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sketch_attention_flashsa_b200 import dp
from sketch_attention_flashsa_b200 import workloads as W

WORLD = 2


def f64(t):
    return t.float().numpy().astype(np.float64)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch(norm):
    return W.make_sa([700, 130, 1, 2500, 64, 900], 2, 64, 16, seed=77, norm=norm, with_dsketch=True,
                     dsketch_seed=78)


def _worker(rank, world, port, norm):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = _batch(norm)
        cu = inp.cu_seqlens.numpy()
        q, k, v, do = f64(inp.q), f64(inp.k), f64(inp.v), f64(inp.dsketch)
        parts = dp.partition_users(inp.valid_lengths(), world)
        mine = parts[rank]
        rows, lcu = dp.shard_ragged(cu, mine)
        # forward: this rank's users alone give the same sketch rows as the whole batch
        sk_full, _, _ = oracle.sa_forward(q, k, v, cu, None, inp.scale, norm)
        sk_loc, _, _ = oracle.sa_forward(q, k[rows], v[rows], lcu, None, inp.scale, norm)
        assert np.allclose(sk_loc, sk_full[mine], rtol=0, atol=1e-12)
        # backward: local dQ summed over ranks equals the whole batch's dQ
        gq, gk, gv = oracle.sa_backward(q, k, v, cu, None, do, inp.scale, norm)
        lq, lk, lv = oracle.sa_backward(q, k[rows], v[rows], lcu, None, do[mine], inp.scale, norm)
        t = torch.from_numpy(lq.copy())
        dp.allreduce_dq(t)
        assert np.allclose(t.numpy(), gq, rtol=1e-12, atol=1e-12), np.abs(t.numpy() - gq).max()
        assert np.allclose(lk, gk[rows], atol=1e-12) and np.allclose(lv, gv[rows], atol=1e-12)
        # timing: every rank reports the max over ranks
        assert dp.max_over_ranks([rank + 1.0, -float(rank)]) == [float(world), 0.0]
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("norm", [W.NORM_PROTO, W.NORM_TOKEN])
def test_two_ranks_gloo(norm):
    mp.spawn(_worker, args=(WORLD, _free_port(), norm), nprocs=WORLD, join=True)


def test_partition_users_properties():
    rng = np.random.default_rng(3)
    for world in (1, 2, 3, 8):
        lens = [int(x) for x in rng.integers(1000, 100_000, 64)]
        parts = dp.partition_users(lens, world)
        assert sorted(u for p in parts for u in p) == list(range(64))
        loads = [sum(lens[u] for u in p) for p in parts]
        # longest-first greedy: the spread is at most one user's length
        assert max(loads) - min(loads) <= max(lens)
        assert parts == dp.partition_users(lens, world)
    assert dp.partition_users([5, 5, 5, 5], 2) == [[0, 2], [1, 3]]  # ties go to the lower rank
    assert dp.partition_users([], 3) == [[], [], []]
    assert dp.partition_users([10], 4) == [[0], [], [], []]


def test_shard_ragged_rows():
    cu = np.array([0, 3, 3, 7, 8])
    rows, lcu = dp.shard_ragged(cu, [0, 2])
    assert rows.tolist() == [0, 1, 2, 3, 4, 5, 6] and lcu.tolist() == [0, 3, 7]
    rows, lcu = dp.shard_ragged(cu, [1, 3])
    assert rows.tolist() == [7] and lcu.tolist() == [0, 0, 1]
    rows, lcu = dp.shard_ragged(cu, [])
    assert rows.size == 0 and lcu.tolist() == [0]


def test_single_process_collectives_are_no_ops():
    t = torch.ones(3)
    assert dp.allreduce_dq(t) is t and t.tolist() == [1, 1, 1]
    assert dp.max_over_ranks([2.5]) == [2.5]
