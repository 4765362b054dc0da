"""A batch split over ranks (mixture_experts_top_b200/shard.py), on CPU.

* combine_stats: the exchange's arithmetic in closed form;
* exchange over two and three gloo ranks: every rank gets the same batch
  statistics, equal to combine_stats of all ranks' inputs;
* the reading the sharded dispatch implements: with each rank's slot
  positions offset by the earlier ranks' slots on the same expert and the
  capacity taken from the whole batch, the kept slots are exactly the
  oracle's single-batch ones ("Mixture-of-Experts Routing - LLM Internals",
  Follow-up; "Mixture of Experts: the Sparsely-Gated Layer", The code:
  first come first served in token order).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_top_b200 import shard
from oracle import moe_oracle as O


def test_combine_stats_closed_form():
    counts = [torch.tensor([3, 0, 1], dtype=torch.int32), torch.tensor([1, 2, 5], dtype=torch.int32)]
    P = [torch.tensor([0.5, 0.25, 0.25]), torch.tensor([0.0, 1.0, 0.0])]
    all_counts, Pg, T = shard.combine_stats(counts, P, [2, 6])
    assert T == 8
    assert all_counts.tolist() == [[3, 0, 1], [1, 2, 5]]
    assert torch.allclose(Pg, torch.tensor([1.0 / 8, 6.5 / 8, 0.5 / 8]))
    assert abs(float(Pg.sum()) - 1.0) < 1e-7


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(rank)
        E = 6
        counts = torch.randint(0, 50, (E,), generator=g, dtype=torch.int32)
        P = torch.rand(E, generator=g)
        P = P / P.sum()
        T_local = 10 + 7 * rank
        res = shard.exchange(counts, P, T_local)
        out[rank] = (counts, P, T_local, res)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_over_gloo_ranks(world):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    ref = shard.combine_stats([res[r][0] for r in range(world)], [res[r][1] for r in range(world)],
                              [res[r][2] for r in range(world)])
    for r in range(world):
        all_counts, P, T = res[r][3]
        assert torch.equal(all_counts, ref[0])
        assert torch.equal(P, ref[1])
        assert T == ref[2]


def _sharded_keep(idx, E, cf, blocks):
    """Keep decisions rank by rank: local positions in token order, offset by
    the earlier ranks' slots on the same expert; capacity of the whole batch."""
    T, k = idx.shape
    cap = O.capacity(cf, T, k, E)
    keep = np.zeros((T, k), bool)
    prefix = np.zeros(E, np.int64)
    t0 = 0
    for n in blocks:
        local = np.zeros(E, np.int64)
        for t in range(t0, t0 + n):
            for j in range(k):
                e = idx[t, j]
                pos = prefix[e] + local[e]
                keep[t, j] = cap is None or pos < cap
                local[e] += 1
        prefix += local
        t0 += n
    return keep


@pytest.mark.parametrize("cf", [0.0, 0.5, 1.0, 1.25])
@pytest.mark.parametrize("blocks", [[40, 60, 28], [1, 126, 1], [128]])
def test_prefix_rule_equals_single_batch_capacity(cf, blocks):
    rng = np.random.default_rng(len(blocks) + int(cf * 100))
    T, k, E = sum(blocks), 3, 8
    # skewed routing so the capacity binds
    logits = rng.standard_normal((T, E)) + np.array([2.0, 1.5, 0, 0, 0, 0, 0, -1.0])
    idx = O.top_k(logits.astype(np.float32), k)
    single = O.dispatch(idx, E, cf)
    assert np.array_equal(_sharded_keep(idx, E, cf, blocks), single["drop_mask"] == 0)
