"""The noisy gate's noise drawn on the GPU (moe_gate_noise) against the
oracle's Philox4x64-10 + Box-Muller draws (oracle.gate_noise, pinned in
test_oracle_noise.py).

The draws z are fp64 on both sides; the noise logits l = x @ W_noise are
fp32 dot products accumulated in different orders, so the noise may differ
by |z| * softplus'(l) * |dl| (softplus' <= 1) with |dl| within the router's
fp32 accumulation bound, plus one fp32 rounding.  With exact-logit inputs it
must match bit for bit, and a block of the batch drawn with its token_base
must match the whole batch's rows.
"""
import math

import numpy as np
import pytest
import torch

from gpu_util import ambiguous_tokens, cfg_of, dev, host
from mixture_experts_top_b200 import api
from oracle import moe_oracle as O
from workloads import WORKLOADS, make_exact_router_inputs, make_inputs

pytestmark = pytest.mark.gpu


def gpu_noise(cfg, x, W_noise, seed, offset, token_base=0):
    ws = api.alloc_workspace(cfg)
    out = torch.full((cfg.T, cfg.E), float("nan"), dtype=torch.float32, device="cuda")
    api.moe_gate_noise(cfg, dev(x), dev(W_noise), seed, offset, token_base, out, ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 0
    return host(out)


def _w_noise(d, E, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((d, E)) / math.sqrt(d)).astype(np.float32)


@pytest.mark.parametrize("T,d,E", [(1024, 256, 64), (300, 200, 6), (4096, 768, 64)])
def test_noise_matches_oracle(T, d, E):
    w = WORKLOADS["switch_relu"].replace(T=T, d=d, E=E, d_hidden=64, d_out=64)
    x = make_inputs(w, seed=5, with_experts=False)["x"]
    Wn = _w_noise(d, E, 6)
    seed, offset = 0x1234_5678_9ABC, 17
    g = gpu_noise(cfg_of(w), x, Wn, seed, offset)
    o = O.gate_noise(x, Wn, "bf16", seed, offset)
    xf = O.widen(x, "bf16")
    lbound = 2 * d * 2.0 ** -24 * (np.abs(xf) @ np.abs(Wn.astype(np.float64)))
    L = (xf @ Wn.astype(np.float64)).astype(np.float32).astype(np.float64)
    z = o.astype(np.float64) / O.softplus(L)
    bound = np.abs(z) * lbound + 2.0 ** -22 * np.abs(o.astype(np.float64)) + 1e-30
    assert np.isfinite(g).all()
    assert np.all(np.abs(g.astype(np.float64) - o) <= bound)
    assert abs(float(np.mean(z))) < 0.05 and abs(float(np.var(z)) - 1.0) < 0.1


def test_noise_exact_logits_bit_identical_and_token_base():
    T, d, E = 500, 128, 32
    w = WORKLOADS["switch_relu"].replace(T=T, d=d, E=E, d_hidden=64, d_out=64)
    ex = make_exact_router_inputs(T, d, E, "bf16", seed=2)
    x, Wn = ex["x"], ex["W_router"]                # exact fp32 noise logits
    g = gpu_noise(cfg_of(w), x, Wn, 99, 3)
    assert np.array_equal(g, O.gate_noise(x, Wn, "bf16", 99, 3))
    part = gpu_noise(cfg_of(w, T=180), x[320:], Wn, 99, 3, token_base=320)
    assert np.array_equal(part, g[320:])
    assert not np.array_equal(gpu_noise(cfg_of(w), x, Wn, 99, 4), g)   # another offset


def test_noisy_forward_routes_like_the_oracle():
    w = WORKLOADS["switch_relu"].replace(T=1024, d=256, d_hidden=512, d_out=256)
    inp = make_inputs(w, seed=8)
    Wn = _w_noise(w.d, w.E, 9)
    cfg = cfg_of(w)
    noise = torch.from_numpy(gpu_noise(cfg, inp["x"], Wn, 7, 0)).cuda()
    ws = api.alloc_workspace(cfg)
    idx = torch.empty((w.T, w.top_k), dtype=torch.int32, device="cuda")
    gates = torch.empty((w.T, w.top_k), dtype=torch.float32, device="cuda")
    P = torch.empty(w.E, dtype=torch.float32, device="cuda")
    api.moe_route(cfg, dev(inp["x"]), dev(inp["W_router"]), None, noise, idx, gates, P, None, ws)
    torch.cuda.synchronize()
    o = O.moe_route(inp["x"], inp["W_router"], w.top_k, "bf16", None,
                    O.gate_noise(inp["x"], Wn, "bf16", 7, 0))
    amb = ambiguous_tokens(o["logits"], w.top_k)
    assert amb.mean() < 0.01
    assert np.array_equal(host(idx)[~amb], o["expert_indices"][~amb])


def test_noise_refuses_fp32_activations():
    cfg = api.make_config(64, 32, 0, 32, 8, 2, "linear", "f32")
    ws = api.alloc_workspace(cfg)
    out = torch.empty((64, 8), dtype=torch.float32, device="cuda")
    x = torch.zeros((64, 32), dtype=torch.float32, device="cuda")
    W = torch.zeros((32, 8), dtype=torch.float32, device="cuda")
    with pytest.raises(api.MoeError) as e:
        api.moe_gate_noise(cfg, x, W, 1, 0, 0, out, ws)
    assert e.value.status == api.MOE_ERR_UNSUPPORTED


def _route_outputs(cfg, T, E, k):
    return (torch.full((T, k), -1, dtype=torch.int32, device="cuda"),
            torch.full((T, k), -1.0, dtype=torch.float32, device="cuda"),
            torch.full((E,), -1.0, dtype=torch.float32, device="cuda"),
            torch.full((T, E), -1.0, dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("T,d,E,k,bias", [(4096, 768, 64, 1, False), (1000, 256, 8, 2, True),
                                          (777, 512, 32, 4, True), (130, 200, 20, 3, False)])
def test_fused_noisy_route_equals_noise_then_route(T, d, E, k, bias):
    """moe_route_noisy (the noise formed inside the router from its own
    contraction) gives the bits of moe_gate_noise followed by moe_route:
    indices, gates, P, logits and the noise itself."""
    w = WORKLOADS["switch_relu"].replace(T=T, d=d, E=E, top_k=k, d_hidden=64, d_out=64)
    inp = make_inputs(w, seed=12, with_experts=False)
    Wn = _w_noise(d, E, 13)
    b = (np.random.default_rng(14).standard_normal(E).astype(np.float32) if bias else None)
    cfg = cfg_of(w)
    ws = api.alloc_workspace(cfg)
    seed, offset, base = 0xBEEF, 5, 1234
    noise = torch.empty((T, E), dtype=torch.float32, device="cuda")
    api.moe_gate_noise(cfg, dev(inp["x"]), dev(Wn), seed, offset, base, noise, ws)
    ref = _route_outputs(cfg, T, E, k)
    api.moe_route(cfg, dev(inp["x"]), dev(inp["W_router"]), dev(b), noise, *ref, ws)
    got = _route_outputs(cfg, T, E, k)
    noise_out = torch.empty((T, E), dtype=torch.float32, device="cuda")
    api.moe_route_noisy(cfg, dev(inp["x"]), dev(inp["W_router"]), dev(b), dev(Wn), seed, offset,
                        base, *got, noise_out, ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 0
    assert np.array_equal(host(noise_out), host(noise))
    for g, r in zip(got, ref):
        assert np.array_equal(host(g), host(r))


def test_fused_noisy_route_against_the_oracle():
    """The fused path's routing against the oracle's router fed the oracle's
    own draws (the same generator, written from its definition)."""
    w = WORKLOADS["switch_relu"].replace(T=1024, d=256, d_hidden=512, d_out=256)
    inp = make_inputs(w, seed=8, with_experts=False)
    Wn = _w_noise(w.d, w.E, 9)
    cfg = cfg_of(w)
    ws = api.alloc_workspace(cfg)
    idx, gates, P, L = _route_outputs(cfg, w.T, w.E, w.top_k)
    api.moe_route_noisy(cfg, dev(inp["x"]), dev(inp["W_router"]), None, dev(Wn), 7, 0, 0, idx,
                        gates, P, L, None, ws)
    torch.cuda.synchronize()
    o = O.moe_route(inp["x"], inp["W_router"], w.top_k, "bf16", None,
                    O.gate_noise(inp["x"], Wn, "bf16", 7, 0))
    amb = ambiguous_tokens(o["logits"], w.top_k)
    assert amb.mean() < 0.01
    assert np.array_equal(host(idx)[~amb], o["expert_indices"][~amb])
    assert np.all(np.abs(host(P).astype(np.float64) - o["P"]) <= 1e-5 * np.abs(o["P"]) + 1e-9)


def test_fused_noisy_route_exact_logits_bit_exact():
    """Exact-logit inputs: the fused router's logits and noise equal the
    oracle's bit for bit."""
    T, d, E = 300, 128, 16
    w = WORKLOADS["switch_relu"].replace(T=T, d=d, E=E, top_k=2, d_hidden=64, d_out=64)
    ex = make_exact_router_inputs(T, d, E, "bf16", seed=4)
    Wn = make_exact_router_inputs(T, d, E, "bf16", seed=5)["W_router"]
    cfg = cfg_of(w)
    ws = api.alloc_workspace(cfg)
    idx, gates, P, L = _route_outputs(cfg, T, E, 2)
    noise = torch.empty((T, E), dtype=torch.float32, device="cuda")
    api.moe_route_noisy(cfg, dev(ex["x"]), dev(ex["W_router"]), None, dev(Wn), 3, 1, 0, idx, gates,
                        P, L, noise, ws)
    torch.cuda.synchronize()
    on = O.gate_noise(ex["x"], Wn, "bf16", 3, 1)
    assert np.array_equal(host(noise), on)
    o = O.moe_route(ex["x"], ex["W_router"], 2, "bf16", None, on)
    assert np.array_equal(host(L), o["logits"])
    assert np.array_equal(host(idx), o["expert_indices"])
