"""A batch split over ranks (mixture_experts_top_b200/shard.py), on CPU.

* the exchange record's layout (E counts, E P bits, T) read back on the host;
* gather_records over two and three gloo ranks: every rank gets every
  rank's record, in rank order;
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


def test_record_layout_round_trip():
    counts = np.array([[3, 0, 1], [1, 2, 5]], np.int32)
    P = np.array([[0.5, 0.25, 0.25], [0.0, 1.0, 0.0]], np.float32)
    rec = np.concatenate([counts, P.view(np.int32), np.array([[2], [6]], np.int32)], axis=1)
    assert rec.shape[1] == shard.record_ints(3)
    c, p, t = shard.unpack_records(rec)
    assert c.tolist() == counts.tolist() and np.array_equal(p, P) and t.tolist() == [2, 6]


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
        record = torch.cat([counts, P.view(torch.int32), torch.tensor([T_local], dtype=torch.int32)])
        res = shard.gather_records(record)
        out[rank] = (counts.numpy(), P.numpy(), T_local, res.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gather_records_over_gloo_ranks(world):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        c, p, t = shard.unpack_records(res[r][3])
        for src in range(world):
            assert np.array_equal(c[src], res[src][0])
            assert np.array_equal(p[src], res[src][1])
            assert t[src] == res[src][2]


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
