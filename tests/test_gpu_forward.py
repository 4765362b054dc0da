"""End-to-end moe_forward against the CPU oracle.

Reduced variants of the five workloads (same E, top_k, expert kind, dtype,
capacity, bias and noise; smaller widths) are compared on every token; the
full-size workloads, run in the launch configuration the benchmark times,
are compared on every routing output and on a sample of output rows.
"""
import numpy as np
import pytest
import torch

from gpu_util import (REL_F32, REL_ROUTE, ambiguous_tokens, bf16_to_f64, cfg_of, dev, host,
                      layer_tolerance, rel_close)
from mixture_experts_top_b200.layer import MoeForward
from oracle import moe_oracle as O
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

REDUCED = {
    "tiny_linear": WORKLOADS["tiny_linear"],
    "switch_relu": WORKLOADS["switch_relu"].replace(T=1024, d=256, d_hidden=512, d_out=256),
    "mixtral": WORKLOADS["mixtral"].replace(T=600, d=512, d_hidden=1024, d_out=512),
    "fine_grained": WORKLOADS["fine_grained"].replace(T=1100, d=256, d_hidden=352, d_out=256),
    "decode": WORKLOADS["decode"].replace(d=512, d_hidden=1024, d_out=512),
    # top-2 with the combine in the down projection's epilogue (hidden width
    # 4096, 1024 grouped rows per expert), capacity drops included
    "mixtral_fused_combine": WORKLOADS["mixtral"].replace(T=2048, d=256, d_hidden=4096,
                                                          d_out=256, E=4, capacity_factor=0.9),
}


def gpu_forward(w, inp):
    layer = MoeForward(cfg_of(w))
    o = layer(dev(inp["x"]), dev(inp["W_router"]), dev(inp["logit_bias"]), dev(inp["noise"]),
              dev(inp["W_in"]), dev(inp["W_up"]), dev(inp["W_out"]))
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    return {k: host(getattr(o, k)) for k in ("output", "expert_indices", "gates", "aux_loss",
                                             "counts", "drop_mask")}


def oracle_routing(w, inp):
    r = O.moe_route(inp["x"], inp["W_router"], w.top_k, w.dtype, inp["logit_bias"], inp["noise"])
    d = O.dispatch(r["expert_indices"], w.E, w.capacity_factor)
    r.update(d)
    r["aux_loss"] = O.aux_loss(d["f"], r["P"])
    return r


def check_routing(w, g, o):
    """Indices, gates, counts, drops and aux; returns the tokens to compare."""
    amb = ambiguous_tokens(o["logits"], w.top_k)
    assert amb.mean() < 0.01
    agree = ~amb & (g["expert_indices"] == o["expert_indices"]).all(axis=1)
    assert np.array_equal(agree, ~amb), "indices differ on an unambiguous token"
    assert rel_close(g["gates"][agree], o["gates"][agree], REL_ROUTE)
    if amb.any():
        # a flipped near-tie moves counts by one and may shift later drops
        assert np.abs(g["counts"].astype(int) - o["counts"]).sum() <= 2 * int(amb.sum())
        same_drop = (g["drop_mask"] == o["drop_mask"]).all(axis=1)
        return agree & same_drop
    assert np.array_equal(g["counts"], o["counts"])
    assert np.array_equal(g["drop_mask"], o["drop_mask"])
    assert abs(float(g["aux_loss"][0]) - o["aux_loss"]) <= REL_ROUTE * o["aux_loss"]
    return agree


def check_rows(w, got_rows, ref_rows, expert_rows):
    """Layer output rows; bf16 bound derived from the expert-output bound."""
    if w.dtype == "f32":
        assert np.abs(got_rows - ref_rows).max() <= REL_F32 * np.abs(ref_rows).max()
    else:
        got = bf16_to_f64(got_rows)
        rms_y = float(np.sqrt(np.mean(np.asarray(expert_rows) ** 2)))
        assert np.isfinite(got).all()
        err = np.abs(got - ref_rows)
        assert np.all(err <= layer_tolerance(ref_rows, rms_y)), err.max()


@pytest.mark.parametrize("name", list(REDUCED))
def test_forward_reduced_all_tokens(name):
    w = REDUCED[name]
    if name == "mixtral_fused_combine":
        from mixture_experts_top_b200 import api
        assert api.moe_forward_combine_fused(cfg_of(w))
    inp = make_inputs(w, seed=11)
    g = gpu_forward(w, inp)
    weights = {k: inp[k] for k in ("W_in", "W_up", "W_out")}
    o = O.moe_forward(inp["x"], inp["W_router"], weights, top_k=w.top_k, kind=w.kind,
                      dtype=w.dtype, d_out=w.d_out, capacity_factor=w.capacity_factor,
                      logit_bias=inp["logit_bias"], noise=inp["noise"])
    tok = check_routing(w, g, o)
    check_rows(w, g["output"][tok], o["output"][tok], o["Y"])
    if w.capacity_factor > 0:
        assert o["drop_mask"].sum() > 0 or name == "switch_relu"
        # fully dropped tokens output exactly zero
        dead = (o["drop_mask"] == 1).all(axis=1) & tok
        if w.dtype == "bf16":
            assert (bf16_to_f64(g["output"][dead]) == 0).all()


def full_size_sample(w, tok, o, n_total=256):
    """At least n_total comparable tokens (all of them if fewer): for every
    expert a share of the tokens it kept, then tokens that had a slot
    dropped, then random ones."""
    rng = np.random.default_rng(1)
    per = -(-n_total // w.E)
    picks = []
    kept = (o["drop_mask"] == 0)
    for e in range(w.E):
        on_e = np.flatnonzero(tok & ((o["expert_indices"] == e) & kept).any(axis=1))
        if len(on_e):
            picks.append(rng.choice(on_e, size=min(per, len(on_e)), replace=False))
    dropped = np.flatnonzero(tok & (o["drop_mask"] == 1).any(axis=1))
    picks.append(dropped[:16])
    sample = np.unique(np.concatenate(picks)) if picks else np.zeros(0, np.int64)
    rest = np.setdiff1d(np.flatnonzero(tok), sample)
    need = max(0, n_total - len(sample))
    if need and len(rest):
        sample = np.union1d(sample, rng.choice(rest, size=min(need, len(rest)), replace=False))
    return sample


@pytest.mark.slow
@pytest.mark.parametrize("name", ["decode", "switch_relu", "fine_grained", "mixtral"])
def test_forward_full_size_sampled(name):
    w = WORKLOADS[name]
    inp = make_inputs(w, seed=0)
    g = gpu_forward(w, inp)
    o = oracle_routing(w, inp)
    tok = check_routing(w, g, o)
    sample = full_size_sample(w, tok, o)
    assert len(sample) >= min(256, int(tok.sum()))
    weights = {k: inp[k] for k in ("W_in", "W_up", "W_out")}
    ref, rows = O.sampled_outputs(sample, inp["x"], w.dtype, w.kind, weights,
                                  o["expert_indices"], o["gates"], o["dest"], return_rows=True)
    check_rows(w, g["output"][sample], ref, rows)


def test_forward_repeat_is_bit_identical():
    """Noise off, two runs: identical outputs (no atomics, fixed orders)."""
    w = REDUCED["fine_grained"]
    inp = make_inputs(w, seed=5)
    a = gpu_forward(w, inp)
    b = gpu_forward(w, inp)
    for key in a:
        assert np.array_equal(a[key], b[key]), key


def test_forward_top1_gate_one():
    """top_k = 1: every gate is exactly 1 (MLG Edge cases)."""
    w = REDUCED["switch_relu"].replace(capacity_factor=0.0, noise=False)
    g = gpu_forward(w, make_inputs(w, seed=2))
    assert (g["gates"] == 1.0).all()


def test_forward_zero_router_aux_is_one():
    """W_router = 0: aux_loss = 1.0 exactly (MLG Examples)."""
    w = REDUCED["mixtral"].replace(T=512)
    inp = make_inputs(w, seed=3)
    inp["W_router"] = np.zeros_like(inp["W_router"])
    g = gpu_forward(w, inp)
    assert float(g["aux_loss"][0]) == 1.0
    assert (g["expert_indices"] == np.array([0, 1])).all()


def test_forward_collapse_aux_near_E():
    """A +30 bias on one expert sends every token there: aux -> E."""
    w = REDUCED["fine_grained"].replace(capacity_factor=0.0, top_k=1, T=640)
    inp = make_inputs(w, seed=4)
    bias = np.zeros(w.E, np.float32)
    bias[9] = 30.0
    inp["logit_bias"] = bias
    g = gpu_forward(w, inp)
    assert (g["expert_indices"][:, 0] == 9).all()
    assert w.E - 1e-3 < float(g["aux_loss"][0]) <= w.E * (1 + 1e-6)


def test_tiny_linear_zero_router_aux_is_exactly_one():
    """The pages' small linear case with W_router = 0: every logit ties, so
    indices are [0, 1] (lower index wins), gates are 1/2, and aux = 1.0
    exactly (MLG Examples); the output is the oracle's within 1e-4."""
    w = WORKLOADS["tiny_linear"]
    inp = make_inputs(w, seed=0)
    inp["W_router"] = np.zeros_like(inp["W_router"])
    g = gpu_forward(w, inp)
    assert float(g["aux_loss"][0]) == 1.0
    assert (g["expert_indices"] == np.array([0, 1])).all()
    assert (g["gates"] == 0.5).all()
    o = O.moe_forward(inp["x"], inp["W_router"], {"W_in": inp["W_in"]}, top_k=2, kind="linear",
                      dtype="f32", d_out=w.d_out)
    assert o["aux_loss"] == 1.0
    check_rows(w, g["output"], o["output"], o["Y"])


def test_tiny_linear_top1_output_is_the_expert_matmul():
    """The pages' small linear case with top_k = 1: every gate is exactly 1
    and each token's output is x_t @ W_e of its expert, checked against a
    plain einsum of the fp32 inputs in fp64 and against the oracle."""
    w = WORKLOADS["tiny_linear"].replace(top_k=1)
    inp = make_inputs(w, seed=0)
    g = gpu_forward(w, inp)
    assert (g["gates"] == 1.0).all()
    o = O.moe_forward(inp["x"], inp["W_router"], {"W_in": inp["W_in"]}, top_k=1, kind="linear",
                      dtype="f32", d_out=w.d_out)
    amb = ambiguous_tokens(o["logits"], 1)
    assert not amb.any()
    assert np.array_equal(g["expert_indices"], o["expert_indices"])
    e = g["expert_indices"][:, 0]
    ref = np.einsum("td,tdo->to", inp["x"].astype(np.float64),
                    inp["W_in"].astype(np.float64)[e])
    assert np.abs(g["output"] - ref).max() <= REL_F32 * np.abs(ref).max()
    check_rows(w, g["output"], o["output"], o["Y"])


def test_forward_empty_batch():
    w = REDUCED["mixtral"].replace(T=0)
    inp = make_inputs(w.replace(T=1), seed=0)
    layer = MoeForward(cfg_of(w))
    layer.out.aux_loss.fill_(7.0)
    layer(None, dev(inp["W_router"]), None, None, dev(inp["W_in"]), dev(inp["W_up"]),
          dev(inp["W_out"]))
    torch.cuda.synchronize()
    assert float(layer.out.aux_loss[0]) == 0.0
