"""Expert parallelism: the E experts split over `world` ranks (GPUs), each
rank holding a contiguous block of the experts' weights.

"Mixture-of-Experts Routing - LLM Internals" (mlgrind.dev), Follow-up: in a
distributed setting the routed tokens travel to the device that holds their
expert and back.  Every rank routes and dispatches its own tokens over all E
experts (moe_route, moe_dispatch); the grouped layout is expert-major, so the
rows bound for rank r are one contiguous slice of x_perm.  One all-to-all
sends each slice to its rank with the per-expert row counts; the receiver
runs its experts on every source's slice (moe_expert_ffn, one call per
source: each slice is already expert-major); a second all-to-all brings the
output rows back in the order they were sent, into the source's y_perm, and
the source combines them (moe_combine).  Every kept row meets the
same expert weights as on one GPU, so the result is the single-GPU layer's.

The steps are separate functions so that the exchange can be anything that
moves the blocks: ``ep_forward`` runs them over a torch.distributed group
(NCCL on GPUs: ``all_to_all_single``); a test plays every rank in one
process.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence, Tuple

import torch

from . import api


def plan(E: int, world: int) -> List[Tuple[int, int]]:
    """Expert range [lo, hi) held by each rank: contiguous blocks, the first
    E % world ranks one expert larger."""
    if world < 1 or world > E:
        raise ValueError("need 1 <= world <= E")
    base, extra = divmod(E, world)
    out, lo = [], 0
    for r in range(world):
        hi = lo + base + (1 if r < extra else 0)
        out.append((lo, hi))
        lo = hi
    return out


def exchange_plan(offsets: Sequence[int], ranges: Sequence[Tuple[int, int]]):
    """From a source's grouped-layout offsets (E+1): for each destination rank
    the row slice [start, stop) it receives and that slice's per-expert row
    counts, in the destination's expert order."""
    out = []
    for lo, hi in ranges:
        counts = [int(offsets[e + 1]) - int(offsets[e]) for e in range(lo, hi)]
        out.append((int(offsets[lo]), int(offsets[hi]), counts))
    return out


@dataclass
class SourceState:
    """One rank's tokens after routing and dispatch, and what it sends."""
    idx: torch.Tensor
    gates: torch.Tensor
    dest: torch.Tensor
    drop: torch.Tensor
    counts: torch.Tensor
    aux: torch.Tensor
    x_perm: torch.Tensor
    y_perm: torch.Tensor
    sends: list          # exchange_plan(...)


def ep_dispatch(cfg, x, W_router, logit_bias, noise, ws, world: int) -> SourceState:
    """Route and dispatch this rank's tokens over all E experts."""
    T, k, E = cfg.T, cfg.top_k, cfg.E
    dev = x.device
    i32 = dict(dtype=torch.int32, device=dev)
    idx = torch.empty((T, k), **i32)
    gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    P = torch.empty(E, dtype=torch.float32, device=dev)
    api.moe_route(cfg, x, W_router, logit_bias, noise, idx, gates, P, None, ws)
    counts = torch.empty(E, **i32)
    offsets = torch.empty(E + 1, **i32)
    dest = torch.empty((T, k), **i32)
    perm = torch.empty(T * k, **i32)
    drop = torch.empty((T, k), dtype=torch.uint8, device=dev)
    f = torch.empty(E, dtype=torch.float32, device=dev)
    aux = torch.empty(1, dtype=torch.float32, device=dev)
    x_perm = torch.empty((T * k, cfg.d), dtype=x.dtype, device=dev)
    api.moe_dispatch(cfg, x, idx, P, counts, offsets, dest, perm, drop, f, aux, x_perm, ws)
    y_perm = torch.zeros((T * k, cfg.d_out), dtype=torch.float32, device=dev)
    sends = exchange_plan(offsets.cpu().tolist(), plan(E, world))
    return SourceState(idx, gates, dest, drop, counts, aux, x_perm, y_perm, sends)


def ep_experts(cfg, n_local: int, x_recv, slice_counts: Sequence[Sequence[int]], W_in_local,
               W_up_local, W_out_local, y_recv):
    """This rank's experts on the rows received from every source, in source
    order: slice s holds rows of the local experts in expert order, with
    slice_counts[s][e] rows for local expert e.  Writes y_recv (fp32, same
    rows) and returns the workspace (its error word covers every call)."""
    total = int(x_recv.shape[0])
    dev = x_recv.device
    kind = {v: key for key, v in api.EXPERT_KINDS.items()}[cfg.expert_kind]
    dt = {v: key for key, v in api.DTYPES.items()}[cfg.act_dtype]
    lws = api.alloc_workspace(api.make_config(max(total, 1), cfg.d, cfg.d_hidden, cfg.d_out,
                                              n_local, 1, kind, dt), dev)
    start = 0
    for c in slice_counts:
        n = int(sum(c))
        if n > 0:
            off = [0]
            for v in c:
                off.append(off[-1] + int(v))
            lcfg = api.make_config(n, cfg.d, cfg.d_hidden, cfg.d_out, n_local, 1, kind, dt)
            api.moe_expert_ffn(lcfg, x_recv[start:start + n],
                               torch.tensor(off, dtype=torch.int32, device=dev),
                               W_in_local, W_up_local, W_out_local, y_recv[start:start + n], lws)
        start += n
    return lws


def ep_combine(cfg, st: SourceState, output) -> dict:
    """Combine the returned expert rows (already in st.y_perm)."""
    api.moe_combine(cfg, st.y_perm, st.dest, st.gates, output)
    return dict(output=output, expert_indices=st.idx, gates=st.gates, aux_loss=st.aux,
                counts=st.counts, drop_mask=st.drop)


def exchange_rows(sends, x_perm, y_perm, rank: int, world: int, ranges, compute, group=None):
    """The two all-to-alls over `group`.  sends = this rank's exchange_plan;
    compute(x_recv, slice_counts, y_recv) runs this rank's experts on the
    received rows (source order) and fills y_recv; the returned rows land in
    y_perm[:R] in the order they were sent.  Returns (slice_counts, what
    compute returned)."""
    import torch.distributed as dist
    dev = x_perm.device
    lo, hi = ranges[rank]
    width = max(b - a for a, b in ranges)
    cnt = torch.zeros((world, width), dtype=torch.int32)
    for r, (_, _, c) in enumerate(sends):
        cnt[r, :len(c)] = torch.tensor(c, dtype=torch.int32)
    cnt = cnt.to(dev)
    recv_cnt = torch.empty_like(cnt)
    dist.all_to_all_single(recv_cnt, cnt, group=group)
    recv_cnt = recv_cnt.cpu()
    slice_counts = [recv_cnt[s, :hi - lo].tolist() for s in range(world)]
    send_splits = [b - a for a, b, _ in sends]
    recv_splits = [int(sum(c)) for c in slice_counts]
    R = sends[-1][1]
    x_recv = torch.empty((sum(recv_splits),) + tuple(x_perm.shape[1:]), dtype=x_perm.dtype,
                         device=dev)
    dist.all_to_all_single(x_recv, x_perm[:R].contiguous(), recv_splits, send_splits, group=group)
    y_recv = torch.empty((sum(recv_splits),) + tuple(y_perm.shape[1:]), dtype=y_perm.dtype,
                         device=dev)
    result = compute(x_recv, slice_counts, y_recv)
    dist.all_to_all_single(y_perm[:R], y_recv, send_splits, recv_splits, group=group)
    return slice_counts, result


def ep_forward(cfg, rank: int, world: int, x, W_router, logit_bias, noise, W_in_local,
               W_up_local, W_out_local, ws, group=None) -> dict:
    """This rank's layer with the experts split over `world` ranks of a
    torch.distributed group: dispatch, all-to-all of the rows (and of the
    per-expert counts), the local experts, all-to-all back, combine.  aux and
    the capacity are this rank's batch's, as in moe_forward.

    The device error words of both workspaces (this rank's routing and
    dispatch, and its local experts) are read after the second all-to-all;
    a nonzero code (a bounded wait that ran out, offsets that are not a
    partition) raises api.MoeError instead of combining rows that may not
    have been written."""
    st = ep_dispatch(cfg, x, W_router, logit_bias, noise, ws, world)
    ranges = plan(cfg.E, world)
    lo, hi = ranges[rank]
    _, lws = exchange_rows(st.sends, st.x_perm, st.y_perm, rank, world, ranges,
                           lambda xr, sc, yr: ep_experts(cfg, hi - lo, xr, sc, W_in_local,
                                                         W_up_local, W_out_local, yr), group)
    check_device_status({"experts": lws, "dispatch": ws})
    output = torch.empty((cfg.T, cfg.d_out), dtype=x.dtype, device=x.device)
    return ep_combine(cfg, st, output)


def check_device_status(workspaces: dict) -> None:
    """Raise api.MoeError if any workspace's device error word is set (each
    read synchronises its stream and clears the word)."""
    for name, w in workspaces.items():
        code = api.moe_device_status(w)
        if code != 0:
            raise api.MoeError(api.MOE_ERR_DEVICE_CHECK, f"ep_forward ({name})",
                               f"device error code {code}")
