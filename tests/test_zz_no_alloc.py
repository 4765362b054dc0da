"""moe_route_noalloc: the router for callers that cannot allocate device
memory (for instance a plugin inside a host program whose memory pool owns
the GPU, or a service that allows no allocation once it is serving).

It must give the same results as moe_route, which takes a workspace, on two
calls in a row of different shapes (the second call reuses the library's
fixed scratch left over from the first), and it must refuse a call whose
scratch would not fit.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import REL_ROUTE, dev, host, rel_close
from mixture_experts_top_b200 import api
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _outputs(cfg):
    T, k, E = cfg.T, cfg.top_k, cfg.E
    return (torch.full((T, k), -1, dtype=torch.int32, device="cuda"),
            torch.full((T, k), -1.0, dtype=torch.float32, device="cuda"),
            torch.full((E,), -1.0, dtype=torch.float32, device="cuda"),
            torch.full((T, E), -1.0, dtype=torch.float32, device="cuda"))


def test_route_noalloc_matches_route_on_two_calls_in_a_row():
    cases = [WORKLOADS["fine_grained"].with_tokens(3000), WORKLOADS["mixtral"].with_tokens(1000)]
    results = []
    for w in cases:
        inp = make_inputs(w, seed=21, with_experts=False)
        cfg = api.make_config(w.T, w.d, w.d_hidden, w.d_out, w.E, w.top_k, w.kind, w.dtype,
                              w.capacity_factor)
        x, Wr, b, n = dev(inp["x"]), dev(inp["W_router"]), dev(inp["logit_bias"]), dev(inp["noise"])
        idx0, g0, P0, L0 = _outputs(cfg)
        api.moe_route_noalloc(cfg, x, Wr, b, n, idx0, g0, P0, L0)
        ws = api.alloc_workspace(cfg)
        idx1, g1, P1, L1 = _outputs(cfg)
        api.moe_route(cfg, x, Wr, b, n, idx1, g1, P1, L1, ws)
        torch.cuda.synchronize()
        results.append((host(idx0), host(g0), host(P0), host(L0),
                        host(idx1), host(g1), host(P1), host(L1)))
    for idx0, g0, P0, L0, idx1, g1, P1, L1 in results:
        assert np.array_equal(idx0, idx1)
        assert np.array_equal(L0, L1)
        assert rel_close(g0, g1, REL_ROUTE)
        assert rel_close(P0, P1, REL_ROUTE)


def test_route_noalloc_rejects_calls_beyond_its_scratch():
    # ceil(T/32) * E = 1025 * 64 floats > 65536
    cfg = api.make_config(1025 * 32, 64, 64, 64, 64, 2, "swiglu", "bf16")
    lib = api.load_library()
    buf = torch.empty(16, device="cuda")
    p = buf.data_ptr()
    st = lib.moe_route_noalloc(ctypes.byref(cfg), p, p, None, None, p, p, p, None, None)
    assert st == api.MOE_ERR_UNSUPPORTED
    assert "scratch" in lib.moe_last_error_message().decode()
