"""moe_route_noalloc: the router for callers that cannot allocate device
memory (for instance a plugin inside a host program whose memory pool owns
the GPU, or a service that allows no allocation once it is serving).

It must give the same results as moe_route, which takes a workspace, on two
calls in a row of different shapes (the second call reuses the library's
fixed scratch left over from the first), and it must refuse a call whose
scratch would not fit.  This file is collected last on purpose.

moe_route computes bf16 logits on the tensor cores and moe_route_noalloc on
the fp32 pipes: both are fp32 dot products of the same inputs in different
summation orders, so they are compared with the router tests' rules: logits
within the sum of both fp32 accumulation bounds, identical indices except on
tokens whose logits leave a gap below the margin, gates and P within 1e-5.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import REL_ROUTE, ambiguous_tokens, dev, host, rel_close
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
        xf = (inp["x"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        scale = np.abs(xf) @ np.abs(inp["W_router"].astype(np.float64))
        results.append((w, scale, host(idx0), host(g0), host(P0), host(L0),
                        host(idx1), host(g1), host(P1), host(L1)))
    for w, scale, idx0, g0, P0, L0, idx1, g1, P1, L1 in results:
        bound = 4 * w.d * 2.0 ** -24 * scale + 2.0 ** -22 * (np.abs(L1.astype(np.float64)) + 1.0)
        assert np.all(np.abs(L0.astype(np.float64) - L1) <= bound)
        amb = ambiguous_tokens(L1, w.top_k)
        assert amb.mean() < 0.01
        ok = ~amb
        assert np.array_equal(idx0[ok], idx1[ok])
        assert rel_close(g0[ok], g1[ok], REL_ROUTE)
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


def test_route_noalloc_fills_its_scratch_exactly():
    # ceil(T/32) * E = 1024 * 64 = 65536 floats: the whole fixed array, its
    # last row of column sums included.
    w = WORKLOADS["fine_grained"].with_tokens(32768)
    assert -(-w.T // 32) * w.E == 65536
    inp = make_inputs(w, seed=23, with_experts=False)
    cfg = api.make_config(w.T, w.d, w.d_hidden, w.d_out, w.E, w.top_k, w.kind, w.dtype,
                          w.capacity_factor)
    x, Wr, b, n = dev(inp["x"]), dev(inp["W_router"]), dev(inp["logit_bias"]), dev(inp["noise"])
    idx0, g0, P0, L0 = _outputs(cfg)
    api.moe_route_noalloc(cfg, x, Wr, b, n, idx0, g0, P0, L0)
    ws = api.alloc_workspace(cfg)
    idx1, g1, P1, L1 = _outputs(cfg)
    api.moe_route(cfg, x, Wr, b, n, idx1, g1, P1, L1, ws)
    torch.cuda.synchronize()
    L1h = host(L1)
    ok = ~ambiguous_tokens(L1h, w.top_k)
    assert ok.mean() > 0.99
    assert np.array_equal(host(idx0)[ok], host(idx1)[ok])
    assert rel_close(host(g0)[ok], host(g1)[ok], REL_ROUTE)
    assert rel_close(host(P0), host(P1), REL_ROUTE)
    # the last CTA's row: tokens of the final 32-token tile were routed
    assert np.all(host(idx0)[-32:] >= 0)


def test_route_noalloc_against_the_oracle():
    # fp32 tokens (the pages' small linear-expert case): logits within an fp32
    # accumulation bound of the oracle's, indices identical outside near-ties,
    # gates and P within 1e-5, on two calls in a row.
    from oracle import moe_oracle as O
    for w in (WORKLOADS["tiny_linear"], WORKLOADS["tiny_linear"].with_tokens(1000)):
        inp = make_inputs(w, seed=29, with_experts=False)
        cfg = api.make_config(w.T, w.d, w.d_hidden, w.d_out, w.E, w.top_k, w.kind, w.dtype,
                              w.capacity_factor)
        idx, g, P, L = _outputs(cfg)
        api.moe_route_noalloc(cfg, dev(inp["x"]), dev(inp["W_router"]), None, None, idx, g, P, L)
        torch.cuda.synchronize()
        ref = O.moe_route(inp["x"], inp["W_router"], w.top_k, w.dtype)
        scale = np.abs(inp["x"].astype(np.float64)) @ np.abs(inp["W_router"].astype(np.float64))
        bound = 2 * w.d * 2.0 ** -24 * scale + 2.0 ** -23 * np.abs(ref["logits"])
        assert np.all(np.abs(host(L).astype(np.float64) - ref["logits"]) <= bound)
        ok = ~ambiguous_tokens(ref["logits"], w.top_k)
        assert np.array_equal(host(idx)[ok], ref["expert_indices"][ok])
        assert rel_close(host(g)[ok], ref["gates"][ok], REL_ROUTE)
        assert rel_close(host(P), ref["P"], REL_ROUTE)
