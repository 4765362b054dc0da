"""Caller-side buffers for ``moe_forward``, allocated with torch.

:class:`MoeForward` owns the workspace and the output tensors of one layer
shape and calls the C entry point; torch only allocates memory and provides
the stream.  Inputs stay wherever the caller keeps them (device tensors).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

from . import api


@dataclass
class ForwardOutputs:
    output: "object"          # (T, d_out) act dtype
    expert_indices: "object"  # (T, k) int32
    gates: "object"           # (T, k) fp32
    aux_loss: "object"        # (1,) fp32
    counts: "object"          # (E,) int32
    drop_mask: "object"       # (T, k) uint8


class MoeForward:
    def __init__(self, cfg: api.MoeConfig, device="cuda"):
        import torch
        self.cfg = cfg
        self.device = torch.device(device)
        act = torch.bfloat16 if cfg.act_dtype == api.DTYPES["bf16"] else torch.float32
        T, k = cfg.T, cfg.top_k
        self.ws = api.alloc_workspace(cfg, self.device)
        self.out = ForwardOutputs(
            output=torch.empty((T, cfg.d_out), dtype=act, device=self.device),
            expert_indices=torch.empty((T, k), dtype=torch.int32, device=self.device),
            gates=torch.empty((T, k), dtype=torch.float32, device=self.device),
            aux_loss=torch.empty((1,), dtype=torch.float32, device=self.device),
            counts=torch.empty((cfg.E,), dtype=torch.int32, device=self.device),
            drop_mask=torch.empty((T, k), dtype=torch.uint8, device=self.device),
        )

    def __call__(self, x, W_router, logit_bias, noise, W_in, W_up, W_out,
                 stream=None) -> ForwardOutputs:
        o = self.out
        api.moe_forward(self.cfg, x, W_router, logit_bias, noise, W_in, W_up, W_out, o.output,
                        o.expert_indices, o.gates, o.aux_loss, o.counts, o.drop_mask, self.ws,
                        stream)
        return o

    def device_status(self, stream=None) -> int:
        return api.moe_device_status(self.ws, stream)
