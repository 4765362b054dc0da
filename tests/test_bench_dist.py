"""The multi-GPU host logic of bench.py on CPU, with two gloo ranks:
every rank's batch differs while the weights are replicated, the step time
is the max over ranks, and the value is the whole job's tokens over it."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from workloads import WORKLOADS, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        fake_ms = [10.0 + rank, 20.0 - rank, 1.0 * (rank + 1)]
        red = bench.max_over_ranks(fake_ms, world)
        w = WORKLOADS["tiny_linear"]
        inp = make_inputs(w, seed=bench.rank_token_seed(rank))
        weights = make_inputs(w, seed=0)["W_in"]
        x = torch.from_numpy(inp["x"].copy())
        xs = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(xs, x)
        out[rank] = (red, [t.numpy() for t in xs], weights)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    red0, xs0, w0 = res[0]
    red1, _, w1 = res[1]
    assert red0 == red1 == [11.0, 20.0, 2.0]          # element-wise max over ranks
    assert not np.array_equal(xs0[0], xs0[1])         # independent batches
    assert np.array_equal(w0, w1)                     # replicated weights
    assert bench.job_value(2, 8192, 5.0) == pytest.approx(2 * 8192 / 5e-3)
