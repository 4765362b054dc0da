"""One batch split over ranks (GPUs) in contiguous token blocks.

Every token's route, expert work and combine are its own; two quantities
couple the tokens of a batch: the load-balancing loss (P_e and f_e are means
over the whole batch, "Mixture-of-Experts Routing - LLM Internals",
mlgrind.dev, Algorithm 4) and the capacity (a slot's position on its expert
counts every earlier slot of the batch, Algorithm 3 and Follow-up).  So each
rank contributes E slot counts and E probability sums, and the ranks
exchange them once per forward: an all-gather of E int32 and an all-reduce
of E values.  With those, ``moe_dispatch_shard`` keeps and drops exactly the
slots the single-batch layer would, and every rank gets the batch's aux loss.

``combine_stats`` is the arithmetic of the exchange (pure, host side);
``exchange`` runs it over a torch.distributed group (NCCL on GPUs, gloo on
CPU); ``shard_forward`` is one rank's whole layer.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch

from . import api


def combine_stats(counts: Sequence[torch.Tensor], prob_means: Sequence[torch.Tensor],
                  tokens: Sequence[int]) -> Tuple[torch.Tensor, torch.Tensor, int]:
    """Every rank's counts (E int32) and P (E fp32, the mean over its own
    tokens), in rank order -> (all_counts (world, E) int32, the batch's P
    (E fp32), the batch's token count).  P is the token-weighted mean of the
    ranks' P, summed in fp64 in rank order."""
    all_counts = torch.stack([c.to(torch.int32) for c in counts])
    T_global = int(sum(int(t) for t in tokens))
    acc = torch.zeros_like(prob_means[0], dtype=torch.float64)
    for p, t in zip(prob_means, tokens):
        acc += p.to(torch.float64) * int(t)
    P = (acc / T_global).to(torch.float32) if T_global > 0 else torch.zeros_like(acc,
                                                                               dtype=torch.float32)
    return all_counts, P, T_global


def exchange(counts: torch.Tensor, prob_mean: torch.Tensor, T_local: int, group=None):
    """all-gather of the counts, P and token counts over `group`, then
    combine_stats.  Every rank returns the same values."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    dev = counts.device
    c_all: List[torch.Tensor] = [torch.empty_like(counts) for _ in range(world)]
    p_all: List[torch.Tensor] = [torch.empty_like(prob_mean) for _ in range(world)]
    t_local = torch.tensor([T_local], dtype=torch.int64, device=dev)
    t_all: List[torch.Tensor] = [torch.empty_like(t_local) for _ in range(world)]
    dist.all_gather(c_all, counts, group=group)
    dist.all_gather(p_all, prob_mean, group=group)
    dist.all_gather(t_all, t_local, group=group)
    return combine_stats(c_all, p_all, [int(t.item()) for t in t_all])


def shard_forward(cfg, rank: int, x, W_router, logit_bias, noise, W_in, W_up, W_out, ws,
                  group=None):
    """This rank's layer on its block of the batch: route, count, exchange,
    sharded dispatch, experts, combine.  Returns a dict of the outputs
    (output, expert_indices, gates, drop_mask, counts (this rank's), f and
    aux_loss (the batch's))."""
    import torch.distributed as dist
    T, k, E = cfg.T, cfg.top_k, cfg.E
    dev = x.device
    out_dtype = x.dtype
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    P_local = torch.empty(E, dtype=torch.float32, device=dev)
    api.moe_route(cfg, x, W_router, logit_bias, noise, idx, gates, P_local, None, ws)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    api.moe_dispatch_count(cfg, idx, counts, ws)
    all_counts, P, T_global = exchange(counts, P_local, T, group)
    all_counts = all_counts.to(dev).contiguous()
    P = P.to(dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    dest = torch.empty((T, k), dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    drop = torch.empty((T, k), dtype=torch.uint8, device=dev)
    f = torch.empty(E, dtype=torch.float32, device=dev)
    aux = torch.empty(1, dtype=torch.float32, device=dev)
    x_perm = torch.empty((T * k, cfg.d), dtype=x.dtype, device=dev)
    api.moe_dispatch_shard(cfg, rank, dist.get_world_size(group), T_global, all_counts, x, idx, P,
                           counts, offsets, dest, perm, drop, f, aux, x_perm, ws)
    y_perm = torch.empty((T * k, cfg.d_out), dtype=torch.float32, device=dev)
    api.moe_expert_ffn(cfg, x_perm, offsets, W_in, W_up, W_out, y_perm, ws)
    output = torch.empty((T, cfg.d_out), dtype=out_dtype, device=dev)
    api.moe_combine(cfg, y_perm, dest, gates, output)
    return dict(output=output, expert_indices=idx, gates=gates, drop_mask=drop, counts=counts,
                f=f, aux_loss=aux)
