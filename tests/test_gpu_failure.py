"""Failure detection on the GPU without a fault: every pipeline wait in the
library is bounded, records an error code and lets the kernel return.
moe_check_wait_timeout runs one such wait on an mbarrier that nothing
completes; the host must then read code 20 from the workspace, and the same
context and workspace must still run a correct forward pass."""
import time

import numpy as np
import pytest
import torch

from gpu_util import ambiguous_tokens, bf16_to_f64, cfg_of, dev, host
from mixture_experts_top_b200 import api
from mixture_experts_top_b200.layer import MoeForward
from oracle import moe_oracle as O
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_and_the_context_stays_usable():
    w = WORKLOADS["mixtral"].replace(T=300, d=256, d_hidden=384, d_out=256)
    layer = MoeForward(cfg_of(w))
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    api.moe_check_wait_timeout(layer.ws, 20000)          # 20 ms
    code = api.moe_device_status(layer.ws)                # synchronises
    elapsed = time.perf_counter() - t0
    assert code == 20
    assert elapsed >= 0.02
    assert api.moe_device_status(layer.ws) == 0           # read once, then cleared

    inp = make_inputs(w, seed=4)
    out = layer(dev(inp["x"]), dev(inp["W_router"]), None, None, dev(inp["W_in"]),
                dev(inp["W_up"]), dev(inp["W_out"]))
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    ref = O.moe_forward(inp["x"], inp["W_router"], {k: inp[k] for k in ("W_in", "W_up", "W_out")},
                        top_k=w.top_k, kind=w.kind, dtype=w.dtype, d_out=w.d_out)
    ok = ~ambiguous_tokens(ref["logits"], w.top_k)
    assert np.array_equal(host(out.expert_indices)[ok], ref["expert_indices"][ok])
    got = bf16_to_f64(host(out.output))[ok]
    want = ref["output"][ok]
    assert np.sqrt(np.mean((got - want) ** 2)) <= 2e-2 * np.sqrt(np.mean(want ** 2))
