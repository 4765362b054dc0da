"""GPU router (moe_route) against the CPU oracle.

Exact-logit inputs make the fp32 logits independent of the summation order,
so the GPU's logits, indices (heavy ties: lower index wins) and the oracle's
must agree bit for bit.  Random N(0,1) inputs check the tolerances.
"""
import numpy as np
import pytest
import torch

from gpu_util import (REL_ROUTE, ambiguous_tokens, cfg_of, dev, host, rel_close)
from mixture_experts_top_b200 import api
from oracle import moe_oracle as O
from workloads import WORKLOADS, Workload, make_exact_router_inputs, make_inputs

pytestmark = pytest.mark.gpu


def run_route(cfg, x, Wr, bias=None, noise=None):
    T, E, k = cfg.T, cfg.E, cfg.top_k
    ws = api.alloc_workspace(cfg)
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    gates = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    P = torch.empty(E, dtype=torch.float32, device="cuda")
    L = torch.empty((T, E), dtype=torch.float32, device="cuda")
    api.moe_route(cfg, dev(x), dev(Wr), dev(bias), dev(noise), idx, gates, P, L, ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 0
    return dict(idx=host(idx), gates=host(gates), P=host(P), L=host(L))


def _wl(T, d, E, k, dtype):
    return Workload("r", T=T, d=d, d_hidden=64, d_out=64, E=E, top_k=k,
                    kind="linear" if dtype == "f32" else "swiglu", dtype=dtype, capacity_factor=0)


EXACT_CASES = [
    # T (ragged vs the 64-token CTA), d (ragged vs the 64-wide k chunk), E, k, dtype
    (64, 32, 8, 2, "f32"),
    (1000, 256, 8, 2, "bf16"),
    (257, 200, 6, 3, "bf16"),      # E not a multiple of 4 (scalar W loads)
    (130, 64, 16, 1, "f32"),
    (333, 512, 32, 4, "bf16"),
    (700, 2048, 64, 6, "bf16"),
    (200, 96, 100, 8, "bf16"),
    (77, 128, 256, 8, "f32"),
    (1, 8, 1, 1, "bf16"),
    (5, 16, 4, 4, "f32"),          # k = E
    (20000, 256, 16, 2, "bf16"),   # > 2 tiles per SM: one CTA per token tile, no split of d
]


@pytest.mark.parametrize("T,d,E,k,dtype", EXACT_CASES)
@pytest.mark.parametrize("extras", ["none", "bias", "bias+noise"])
def test_route_exact_logits_bit_exact(T, d, E, k, dtype, extras):
    rng = np.random.default_rng(T + d + E)
    bias = noise = None
    if "bias" in extras:
        bias = (rng.integers(-8, 9, size=E) / 4.0).astype(np.float32)
    if "noise" in extras:
        noise = rng.standard_normal((T, E)).astype(np.float32)
    inp = make_exact_router_inputs(T, d, E, dtype, seed=T, bias=bias)
    cfg = cfg_of(_wl(T, d, E, k, dtype))
    g = run_route(cfg, inp["x"], inp["W_router"], bias, noise)
    o = O.moe_route(inp["x"], inp["W_router"], k, dtype, bias, noise)
    assert np.array_equal(g["L"], o["logits"]), "fp32 logits must be bit-identical"
    assert np.array_equal(g["idx"], o["expert_indices"])
    assert rel_close(g["gates"], o["gates"], REL_ROUTE)
    assert rel_close(g["P"], o["P"], REL_ROUTE)


@pytest.mark.parametrize("T,d,E,k", [(300, 64, 8, 2), (129, 200, 64, 6), (64, 4096, 32, 4)])
def test_route_full_precision_router_weights(T, d, E, k):
    """bf16 tokens that are one-hot (one entry +-2^j, the rest 0) make every
    logit one fp32 router weight times a power of two, exactly: the logits
    must equal the oracle's bit for bit, whatever the 24-bit mantissas of
    W_router.  This checks that no bit of the fp32 weights is lost by the
    bf16 tensor-core router, which splits each weight into three bf16 terms."""
    rng = np.random.default_rng(T * 7 + E)
    xf = np.zeros((T, d), np.float32)
    t = np.arange(T)
    xf[t, rng.integers(0, d, size=T)] = (rng.choice([-1.0, 1.0], size=T) *
                                          2.0 ** rng.integers(-3, 4, size=T)).astype(np.float32)
    x = (xf.view(np.uint32) >> 16).astype(np.uint16)        # exact in bf16
    Wr = rng.standard_normal((d, E)).astype(np.float32) * np.float32(0.37)
    bias = rng.standard_normal(E).astype(np.float32)
    cfg = cfg_of(_wl(T, d, E, k, "bf16"))
    g = run_route(cfg, x, Wr, bias)
    o = O.moe_route(x, Wr, k, "bf16", bias, None)
    assert np.array_equal(g["L"], o["logits"]), "fp32 logits must be bit-identical"
    assert np.array_equal(g["idx"], o["expert_indices"])
    assert rel_close(g["gates"], o["gates"], REL_ROUTE)
    assert rel_close(g["P"], o["P"], REL_ROUTE)


@pytest.mark.parametrize("name", ["tiny_linear", "switch_relu", "mixtral", "fine_grained", "decode"])
def test_route_workloads_random(name):
    w = WORKLOADS[name]
    T = min(w.T, 4096)
    w = w.with_tokens(T)
    inp = make_inputs(w, seed=1, with_experts=False)
    cfg = cfg_of(w)
    g = run_route(cfg, inp["x"], inp["W_router"], inp["logit_bias"], inp["noise"])
    o = O.moe_route(inp["x"], inp["W_router"], w.top_k, w.dtype, inp["logit_bias"], inp["noise"])
    amb = ambiguous_tokens(o["logits"], w.top_k)
    assert amb.mean() < 0.01
    ok = ~amb
    assert np.array_equal(g["idx"][ok], o["expert_indices"][ok])
    assert rel_close(g["gates"][ok], o["gates"][ok], REL_ROUTE)
    assert rel_close(g["P"], o["P"], REL_ROUTE)
    # fp32 accumulation bound on the logits: 2 d eps sum |x_i W_ie| (+ rounding of bias/noise)
    xf = O.widen(inp["x"], w.dtype)
    bound = 2 * w.d * 2.0 ** -24 * (np.abs(xf) @ np.abs(inp["W_router"].astype(np.float64)))
    bound += 2.0 ** -23 * (np.abs(o["logits"].astype(np.float64)) + 1.0)
    assert np.all(np.abs(g["L"].astype(np.float64) - o["logits"]) <= bound)
    # the GPU's own top-k decision, re-taken by the oracle on the GPU's logits,
    # is the same (both in fp32): indices are a pure function of the logits.
    assert np.array_equal(O.top_k(g["L"], w.top_k), g["idx"])


def test_route_zero_router_gives_uniform_gates():
    """W_router = 0: every logit ties, experts 0..k-1 win, gates are 1/k."""
    for k in (1, 2, 3, 8):
        w = _wl(100, 64, 8, k, "bf16")
        inp = make_inputs(w, seed=2, with_experts=False)
        g = run_route(cfg_of(w), inp["x"], np.zeros((64, 8), np.float32))
        assert (g["idx"] == np.arange(k)[None, :]).all()
        assert np.array_equal(g["gates"], np.full((100, k), np.float32(1.0) / np.float32(k)))
        assert np.array_equal(g["P"], np.full(8, 0.125, np.float32))


def test_route_empty_batch():
    w = _wl(0, 64, 8, 2, "bf16")
    cfg = cfg_of(w)
    ws = api.alloc_workspace(cfg)
    P = torch.full((8,), 5.0, device="cuda")
    api.moe_route(cfg, None, dev(np.zeros((64, 8), np.float32)), None, None, None, None, P, None, ws)
    torch.cuda.synchronize()
    assert (host(P) == 0).all()


def test_route_is_deterministic():
    w = _wl(3000, 512, 64, 6, "bf16")
    inp = make_inputs(w, seed=3, with_experts=False)
    a = run_route(cfg_of(w), inp["x"], inp["W_router"])
    b = run_route(cfg_of(w), inp["x"], inp["W_router"])
    for key in a:
        assert np.array_equal(a[key], b[key])
