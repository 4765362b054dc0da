"""GPU combine (moe_combine) against the oracle's combine on the same fp32
expert rows, destinations and gates.  The kernel's fp32 multiply-add chain is
within k * 2^-24 * sum |g y| of the exact sum, then rounds once to bf16."""
import numpy as np
import pytest
import torch

from gpu_util import bf16_to_f64, bf16_ulp, dev, host
from mixture_experts_top_b200 import api
from oracle import moe_oracle as O
from workloads.generate import f32_to_bf16_bits

pytestmark = pytest.mark.gpu


def run_combine(cfg, y_perm, dest, gates):
    act = torch.bfloat16 if cfg.act_dtype == 1 else torch.float32
    out = torch.full((cfg.T, cfg.d_out), 99.0, dtype=act, device="cuda")
    api.moe_combine(cfg, dev(y_perm), dev(dest.astype(np.int32)), dev(gates.astype(np.float32)), out)
    torch.cuda.synchronize()
    return host(out)


def _case(T, k, d_out, drop_frac, rng):
    R = T * k
    perm = rng.permutation(R)
    dest = perm.reshape(T, k).astype(np.int32)
    dest[rng.random((T, k)) < drop_frac] = -1
    g = rng.random((T, k)).astype(np.float32)
    g /= g.sum(axis=1, keepdims=True)
    return dest, g.astype(np.float32)


@pytest.mark.parametrize("T,k,d_out,drop", [(1, 1, 8, 0.0), (100, 2, 4096, 0.0), (999, 6, 2048, 0.3),
                                            (64, 8, 768, 0.5), (300, 1, 264, 0.2)])
def test_combine_bf16(T, k, d_out, drop):
    rng = np.random.default_rng(T + k)
    dest, gates = _case(T, k, d_out, drop, rng)
    y_perm = rng.standard_normal((T * k, d_out)).astype(np.float32)
    cfg = api.make_config(T, 64, 64, d_out, 8, k, "relu", "bf16")
    got = bf16_to_f64(run_combine(cfg, y_perm, dest, gates))
    ref = O.combine(y_perm.astype(np.float64), dest, gates)
    chain = 2 * k * 2.0 ** -24 * O.combine(np.abs(y_perm.astype(np.float64)), dest, gates)
    assert np.all(np.abs(got - ref) <= bf16_ulp(ref) + chain)
    dropped_all = (dest < 0).all(axis=1)
    assert (got[dropped_all] == 0).all()


def test_combine_f32():
    rng = np.random.default_rng(3)
    T, k, d_out = 64, 2, 32
    dest, gates = _case(T, k, d_out, 0.1, rng)
    y_perm = rng.standard_normal((T * k, d_out)).astype(np.float32)
    cfg = api.make_config(T, 32, 0, d_out, 8, k, "linear", "f32")
    got = run_combine(cfg, y_perm, dest, gates).astype(np.float64)
    ref = O.combine(y_perm.astype(np.float64), dest, gates)
    chain = 2 * k * 2.0 ** -24 * O.combine(np.abs(y_perm.astype(np.float64)), dest, gates)
    assert np.all(np.abs(got - ref) <= 1e-6 * np.abs(ref) + chain)


def test_combine_top1_gate_one_copies_row():
    """top_k = 1 with gate 1.0: the output row is the expert row rounded
    once to bf16 (bit for bit)."""
    rng = np.random.default_rng(4)
    T, d_out = 50, 512
    dest = rng.permutation(T).reshape(T, 1).astype(np.int32)
    y_perm = rng.standard_normal((T, d_out)).astype(np.float32)
    cfg = api.make_config(T, 64, 64, d_out, 4, 1, "relu", "bf16")
    got = run_combine(cfg, y_perm, dest, np.ones((T, 1), np.float32))
    assert np.array_equal(got, f32_to_bf16_bits(y_perm[dest[:, 0]]))


@pytest.mark.parametrize("name,k,cf", [("switch_relu", 1, 1.25), ("mixtral", 1, 0.5),
                                       ("mixtral", 1, 0.0), ("switch_relu", 2, 1.0),
                                       ("mixtral", 2, 0.25), ("mixtral", 2, 0.0),
                                       ("fine_grained", 6, 1.0), ("fine_grained", 8, 0.5),
                                       ("mixtral_pairs", 2, 0.0), ("mixtral_pairs", 3, 0.5)])
def test_expert_ffn_combine_equals_ffn_then_combine(name, k, cf):
    """moe_expert_ffn_combine runs the combine in the down projection's
    epilogue: at top_k = 1 gate * row goes straight to the token's row (no
    y_perm); at top_k > 1 the last of a token's kept rows to finish a column
    block sums the token's rows in slot order.  Either way it must give the
    bits of moe_expert_ffn followed by moe_combine, drops included (tokens
    with every slot dropped get a zero row), on the single-CTA and the
    CTA-pair GEMM (mixtral_pairs: 1024 rows per expert or more)."""
    from gpu_util import cfg_of
    from workloads import WORKLOADS, make_inputs
    base = {"switch_relu": WORKLOADS["switch_relu"].replace(T=1500, d=256, d_hidden=512,
                                                            d_out=256),
            "mixtral": WORKLOADS["mixtral"].replace(T=900, d=256, d_hidden=384, d_out=264),
            "fine_grained": WORKLOADS["fine_grained"].replace(T=1100, d=256, d_hidden=352,
                                                              d_out=520),
            "mixtral_pairs": WORKLOADS["mixtral"].replace(T=4100, d=256, d_hidden=512,
                                                          d_out=776)}[name]
    w = base.replace(top_k=k, capacity_factor=cf)
    inp = make_inputs(w, seed=17)
    cfg = cfg_of(w)
    ws = api.alloc_workspace(cfg)
    T, E = w.T, w.E
    i32 = dict(dtype=torch.int32, device="cuda")
    x = dev(inp["x"])
    idx = torch.empty((T, k), **i32)
    gates = torch.empty((T, k), device="cuda")
    P = torch.empty(E, device="cuda")
    counts, offsets = torch.empty(E, **i32), torch.empty(E + 1, **i32)
    dest, perm = torch.empty((T, k), **i32), torch.empty(T * k, **i32)
    drop = torch.empty((T, k), dtype=torch.uint8, device="cuda")
    f, aux = torch.empty(E, device="cuda"), torch.empty(1, device="cuda")
    x_perm = torch.empty((T * k, w.d), dtype=torch.bfloat16, device="cuda")
    api.moe_route(cfg, x, dev(inp["W_router"]), dev(inp["logit_bias"]), dev(inp["noise"]), idx,
                  gates, P, None, ws)
    api.moe_dispatch(cfg, x, idx, P, counts, offsets, dest, perm, drop, f, aux, x_perm, ws)
    W = [dev(inp[key]) for key in ("W_in", "W_up", "W_out")]
    y_perm = torch.empty((T * k, w.d_out), device="cuda")
    api.moe_expert_ffn(cfg, x_perm, offsets, *W, y_perm, ws)
    ref = torch.full((T, w.d_out), 3.0, dtype=torch.bfloat16, device="cuda")
    api.moe_combine(cfg, y_perm, dest, gates, ref)
    got = torch.full((T, w.d_out), 3.0, dtype=torch.bfloat16, device="cuda")
    api.moe_expert_ffn_combine(cfg, x_perm, offsets, perm, dest, gates, *W, got, ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 0
    dropped = host(drop).all(axis=1)
    if cf > 0 and (k == 1 or cf <= 0.25):
        assert dropped.any()
    g, r = host(got), host(ref)
    assert np.array_equal(g, r)
    assert (bf16_to_f64(g[dropped]) == 0).all()
