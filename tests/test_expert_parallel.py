"""Expert parallelism's host side (mixture_experts_top_b200/expert_parallel.py)
on CPU: the expert plan, the exchange plan of a grouped layout, and the two
all-to-alls over 2 and 3 gloo ranks with an identity "expert" that tags each
row with the receiving rank: every row must reach the rank that holds its
expert and come back to its own slot."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_top_b200 import expert_parallel as ep


def test_plan_and_exchange_plan():
    assert ep.plan(8, 3) == [(0, 3), (3, 6), (6, 8)]
    assert ep.plan(64, 8)[7] == (56, 64)
    with pytest.raises(ValueError):
        ep.plan(4, 5)
    offsets = [0, 2, 2, 7, 9, 9, 12, 13, 20]
    sends = ep.exchange_plan(offsets, ep.plan(8, 3))
    assert sends == [(0, 7, [2, 0, 5]), (7, 12, [2, 0, 3]), (12, 20, [1, 7])]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, E, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(rank)
        kept = rng.integers(0, 6, size=E)
        offsets = np.concatenate([[0], np.cumsum(kept)]).tolist()
        R = offsets[-1]
        ranges = ep.plan(E, world)
        # row i of this rank: (source rank, expert, i)
        expert_of_row = np.repeat(np.arange(E), kept)
        x_perm = torch.tensor([[rank, int(expert_of_row[i]), i] for i in range(R)] +
                              [[-1, -1, -1]] * 3, dtype=torch.float32)
        y_perm = torch.full((R + 3, 4), -5.0)
        seen = {}

        def compute(x_recv, slice_counts, y_recv):
            lo, hi = ranges[rank]
            seen["experts_ok"] = bool(((x_recv[:, 1] >= lo) & (x_recv[:, 1] < hi)).all())
            seen["sources_in_order"] = bool((x_recv[:, 0][1:] >= x_recv[:, 0][:-1]).all())
            seen["counts"] = [int(sum(c)) for c in slice_counts] == \
                [int((x_recv[:, 0] == s).sum()) for s in range(world)]
            y_recv[:, :3] = x_recv
            y_recv[:, 3] = rank
            return ("computed on", rank)

        sends = ep.exchange_plan(offsets, ranges)
        _, result = ep.exchange_rows(sends, x_perm, y_perm, rank, world, ranges, compute)
        seen["result"] = result == ("computed on", rank)
        back_ok = torch.equal(y_perm[:R, :3], x_perm[:R])
        holder = np.searchsorted([b for _, b in ranges], expert_of_row, side="right")
        holder_ok = np.array_equal(y_perm[:R, 3].numpy().astype(int), holder)
        untouched = bool((y_perm[R:] == -5.0).all())
        out[rank] = (seen, back_ok, holder_ok, untouched)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,E", [(2, 8), (3, 8), (3, 5)])
def test_exchange_rows_over_gloo(world, E):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, E, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        seen, back_ok, holder_ok, untouched = res[r]
        assert seen == {"experts_ok": True, "sources_in_order": True, "counts": True,
                        "result": True}, (r, seen)
        assert back_ok and holder_ok and untouched, r
