"""One batch split over ranks (GPUs) in contiguous token blocks.

Every token's route, expert work and combine are its own; two quantities
couple the tokens of a batch: the load-balancing loss (P_e and f_e are means
over the whole batch, "Mixture-of-Experts Routing - LLM Internals",
mlgrind.dev, Algorithm 4) and the capacity (a slot's position on its expert
counts every earlier slot of the batch, Algorithm 3 and Follow-up).  So each
rank writes one exchange record of 2E+1 int32 (moe_shard_record: its E slot
counts, its E probability means as fp32 bits, its token count), the ranks
all-gather the records once per forward, and ``moe_dispatch_shard`` takes
from them the earlier ranks' slots, the batch's f and the batch's P: it keeps
and drops exactly the slots the single-batch layer would, and every rank
gets the batch's aux loss.  All of that arithmetic runs in the library's
kernels; this module only moves the records.

``gather_records`` is the exchange over a torch.distributed group (NCCL on
GPUs, gloo on CPU); ``unpack_records`` reads records on the host (for tests
and diagnostics); ``ShardStep`` is one rank's whole layer with its buffers
allocated once, so that repeated steps allocate nothing and never wait on
the host.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import api


def record_ints(E: int) -> int:
    """Length of one rank's exchange record: E counts, E P bits, T."""
    return 2 * E + 1


def unpack_records(records) -> tuple:
    """(world, 2E+1) int32 records -> (counts (world, E) int32, P (world, E)
    fp32, tokens (world,) int64), on the host."""
    r = np.ascontiguousarray(np.asarray(records, dtype=np.int32))
    E = (r.shape[1] - 1) // 2
    return r[:, :E].copy(), r[:, E:2 * E].copy().view(np.float32), r[:, 2 * E].astype(np.int64)


def gather_records(record: torch.Tensor, out: Optional[torch.Tensor] = None, group=None):
    """all-gather of every rank's record over `group`, in rank order: returns
    (world, 2E+1) int32 on record's device (written into `out` if given)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if out is None:
        out = torch.empty((world, record.numel()), dtype=record.dtype, device=record.device)
    dist.all_gather_into_tensor(out.view(-1), record.contiguous(), group=group)
    return out


class ShardStep:
    """One rank's layer on its block of a batch split over ranks: route,
    record, all-gather of the records, sharded dispatch, experts and combine.
    The buffers are this object's; outputs are in ``self.out``."""

    def __init__(self, cfg, rank: int, world: int, T_global: int, device="cuda", group=None):
        from .layer import ForwardOutputs
        self.cfg, self.rank, self.world, self.T_global, self.group = cfg, rank, world, T_global, group
        T, k, E = cfg.T, cfg.top_k, cfg.E
        dev = torch.device(device)
        act = torch.bfloat16 if cfg.act_dtype == api.DTYPES["bf16"] else torch.float32
        i32 = dict(dtype=torch.int32, device=dev)
        self.ws = api.alloc_workspace(cfg, dev)
        self.P = torch.empty(E, dtype=torch.float32, device=dev)
        self.record = torch.empty(record_ints(E), **i32)
        self.records = torch.empty((world, record_ints(E)), **i32)
        self.offsets = torch.empty(E + 1, **i32)
        self.dest = torch.empty((T, k), **i32)
        self.perm = torch.empty(T * k, **i32)
        self.f = torch.empty(E, dtype=torch.float32, device=dev)
        self.x_perm = torch.empty((T * k, cfg.d), dtype=act, device=dev)
        # the experts and the combine in the form moe_forward uses for cfg
        self.fused = api.moe_forward_combine_fused(cfg)
        self.y_perm = None if self.fused else torch.empty((T * k, cfg.d_out),
                                                          dtype=torch.float32, device=dev)
        self.out = ForwardOutputs(
            output=torch.empty((T, cfg.d_out), dtype=act, device=dev),
            expert_indices=torch.empty((T, k), **i32),
            gates=torch.empty((T, k), dtype=torch.float32, device=dev),
            aux_loss=torch.empty((1,), dtype=torch.float32, device=dev),
            counts=torch.empty((E,), **i32),
            drop_mask=torch.empty((T, k), dtype=torch.uint8, device=dev))

    def route(self, x, W_router, logit_bias, noise):
        o = self.out
        api.moe_route(self.cfg, x, W_router, logit_bias, noise, o.expert_indices, o.gates, self.P,
                      None, self.ws)
        api.moe_shard_record(self.cfg, o.expert_indices, self.P, self.record, self.ws)

    def exchange(self, gather=None):
        """The records of every rank into self.records: over the group, or
        through `gather(record, records)` when given."""
        if gather is not None:
            gather(self.record, self.records)
        else:
            gather_records(self.record, self.records, self.group)

    def finish(self, x, W_in, W_up, W_out):
        o, cfg = self.out, self.cfg
        api.moe_dispatch_shard(cfg, self.rank, self.world, self.T_global, self.records, x,
                               o.expert_indices, None, o.counts, self.offsets, self.dest,
                               self.perm, o.drop_mask, self.f, o.aux_loss, self.x_perm, self.ws)
        if self.fused:
            api.moe_expert_ffn_combine(cfg, self.x_perm, self.offsets, self.perm, self.dest,
                                       o.gates, W_in, W_up, W_out, o.output, self.ws)
        else:
            api.moe_expert_ffn(cfg, self.x_perm, self.offsets, W_in, W_up, W_out, self.y_perm,
                               self.ws)
            api.moe_combine(cfg, self.y_perm, self.dest, o.gates, o.output)

    def __call__(self, x, W_router, logit_bias, noise, W_in, W_up, W_out, gather=None):
        self.route(x, W_router, logit_bias, noise)
        self.exchange(gather)
        self.finish(x, W_in, W_up, W_out)
        return self.out

    def device_status(self) -> int:
        return api.moe_device_status(self.ws)


def shard_forward(cfg, rank: int, x, W_router, logit_bias, noise, W_in, W_up, W_out,
                  T_global: int, group=None) -> dict:
    """This rank's layer on its block of the batch (one ShardStep call over
    `group`).  Returns a dict of the outputs (output, expert_indices, gates,
    drop_mask, counts (this rank's), f and aux_loss (the batch's))."""
    import torch.distributed as dist
    step = ShardStep(cfg, rank, dist.get_world_size(group), T_global, x.device, group)
    o = step(x, W_router, logit_bias, noise, W_in, W_up, W_out)
    return dict(output=o.output, expert_indices=o.expert_indices, gates=o.gates,
                drop_mask=o.drop_mask, counts=o.counts, f=step.f, aux_loss=o.aux_loss)
