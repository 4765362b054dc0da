"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test names the passage (page title and section) or the closed form it
checks.  None of them compares the oracle with itself: values come from the
pages' printed output, from closed forms, from invariants, from library
routines (numpy einsum, torch's bf16 rounding) or from the independent dense
formulation ``moe_forward_brute_force``.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import moe_oracle as O
from workloads import WORKLOADS, make_inputs, make_exact_router_inputs


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# --- router ----------------------------------------------------------------

def test_pfd_token0_worked_example(golden_dir):
    """PFD 'The router': probs of token 0 -> top-2 [6, 3], gates [0.627, 0.373]."""
    g = _load(golden_dir, "pfd_token0_routing.json")
    L = np.log(np.array([g["probs"]], dtype=np.float64)).astype(np.float32)
    idx = O.top_k(L, g["top_k"])
    assert idx[0].tolist() == g["expected_indices"]
    probs = O.softmax_rows(L)
    top = probs[0, idx[0]]
    np.testing.assert_allclose(np.round(top, 3), g["expected_top_probs"], atol=1e-12)
    # The printed probabilities are rounded to 3 decimals (they add up to
    # 1.002), so the top-2 sum is only fixed to within that rounding.
    assert abs(float(top.sum()) - g["expected_top_prob_sum"]) < 2e-3
    gates = O.renormalised_gates(L, idx)
    np.testing.assert_allclose(np.round(gates[0].astype(np.float64), 3), g["expected_gates"], atol=1e-12)


def test_pfd_routing_table_rows_consistent(golden_dir):
    """PFD 'The router': every printed routing-table row has gates summing to 1
    and the printed per-expert counts add up to tokens * k."""
    g = _load(golden_dir, "pfd_token0_routing.json")
    for row in g["printed_routing_table_first_rows"]:
        assert abs(row[2] + row[4] - 1.0) <= 1e-3
    assert sum(g["printed_counts"]) == g["printed_total_assignments"] == g["tokens"] * g["top_k"]


def test_gates_closed_form():
    """softmax over chosen logits: logits ln4, ln2, 0, -5 with k=2 -> gates 2/3, 1/3."""
    L = np.array([[math.log(4.0), math.log(2.0), 0.0, -5.0]], dtype=np.float32)
    idx = O.top_k(L, 2)
    assert idx.tolist() == [[0, 1]]
    g = O.renormalised_gates(L, idx)
    np.testing.assert_allclose(g[0], [2.0 / 3.0, 1.0 / 3.0], rtol=1e-6)


def test_aux_closed_form_two_tokens():
    """Two tokens, two experts, top-1, both choosing expert 1 with probs
    (1/4, 3/4): f = (0, 1), P = (1/4, 3/4), aux = 2 * 3/4 = 1.5."""
    x = np.ones((2, 1), dtype=np.float32)
    W = np.array([[0.0, math.log(3.0)]], dtype=np.float32)
    r = O.moe_route(x, W, 1, "f32")
    assert r["expert_indices"].tolist() == [[1], [1]]
    np.testing.assert_allclose(r["P"], [0.25, 0.75], rtol=1e-7)
    d = O.dispatch(r["expert_indices"], 2, 0.0)
    np.testing.assert_allclose(d["f"], [0.0, 1.0])
    assert abs(O.aux_loss(d["f"], r["P"]) - 1.5) < 1e-6


@pytest.mark.parametrize("T,d,E,k", [(6, 4, 4, 2), (64, 32, 8, 2), (64, 32, 8, 1), (16, 8, 64, 6)])
def test_zero_router_aux_is_exactly_one(T, d, E, k):
    """MLG 'Examples': W_router = 0 -> aux_loss = 1.0.  All logits tie, so the
    chosen experts are 0..k-1 (lower index wins) and each gate is 1/k."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((T, d)).astype(np.float32)
    W = np.zeros((d, E), dtype=np.float32)
    r = O.moe_route(x, W, k, "f32")
    assert (r["expert_indices"] == np.arange(k)[None, :]).all()
    np.testing.assert_allclose(r["gates"], 1.0 / k, rtol=1e-7)
    d_ = O.dispatch(r["expert_indices"], E, 0.0)
    assert O.aux_loss(d_["f"], r["P"]) == 1.0


def test_mlg_collapse_aux_is_E(golden_dir):
    """MLG 'Examples': x = ones(6,4), router strongly prefers expert 0,
    top_k = 1, E = 4 -> aux_loss = 4.0 (f_0 = 1, P_0 close to 1)."""
    g = _load(golden_dir, "mlg_examples.json")["collapse"]
    x = np.ones((g["T"], g["d"]), dtype=np.float32)
    W = np.zeros((g["d"], g["E"]), dtype=np.float32)
    W[:, 0] = 10.0
    r = O.moe_route(x, W, g["top_k"], "f32")
    d_ = O.dispatch(r["expert_indices"], g["E"], 0.0)
    aux = O.aux_loss(d_["f"], r["P"])
    assert aux <= g["aux_loss"] and abs(aux - g["aux_loss"]) < 1e-12


def test_collapse_by_bias_tends_to_E():
    """PFD 'Hot shards': a large logit bias on E3 sends all 64 tokens there;
    the Switch loss climbs towards N = 8 (printed 7.956 for bias +8 on that
    page's weights).  With bias +30 it must lie in (8 - 1e-6, 8]."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 16)).astype(np.float32)
    W = (rng.standard_normal((16, 8)) / 4.0).astype(np.float32)
    bias = np.zeros(8, dtype=np.float32)
    bias[3] = 30.0
    r = O.moe_route(x, W, 1, "f32", logit_bias=bias)
    d_ = O.dispatch(r["expert_indices"], 8, 0.0)
    assert d_["counts"].tolist() == [0, 0, 0, 64, 0, 0, 0, 0]
    aux = O.aux_loss(d_["f"], r["P"])
    assert 8.0 - 1e-6 < aux <= 8.0


def test_tie_break_lower_index_wins():
    """MLG 'Edge cases': stable sort of -logits.  Equal logits keep index
    order, and -0.0 equals +0.0."""
    L = np.array([[1.0, 3.0, 3.0, 2.0],
                  [-0.0, 0.0, -1.0, -0.0],
                  [5.0, 5.0, 5.0, 5.0]], dtype=np.float32)
    assert O.top_k(L, 2).tolist() == [[1, 2], [0, 1], [0, 1]]
    assert O.top_k(L, 3).tolist() == [[1, 2, 3], [0, 1, 3], [0, 1, 2]]


@pytest.mark.parametrize("E", [64, 256])
def test_tie_break_with_many_ties(E):
    """MLG 'Edge cases' with heavy ties at large E: the order must equal a
    sort on the key (-logit, expert index)."""
    rng = np.random.default_rng(E)
    L = rng.integers(0, 3, size=(64, E)).astype(np.float32)
    L[::2] *= -1.0                                   # mixes -0.0 and +0.0 in
    idx = O.top_k(L, 8)
    for t in range(64):
        ref = sorted(range(E), key=lambda e: (-float(L[t, e]), e))[:8]
        assert idx[t].tolist() == ref


def test_topk_is_sorted_and_distinct():
    """NumPy tutorial 'Running and Testing It': every top-k mask row has
    exactly k ones; MLG: indices sorted by descending logit."""
    rng = np.random.default_rng(11)
    L = rng.standard_normal((200, 16)).astype(np.float32)
    idx = O.top_k(L, 5)
    for t in range(200):
        assert len(set(idx[t].tolist())) == 5
        vals = L[t, idx[t]]
        assert (np.diff(vals) <= 0).all()
        assert vals[-1] >= np.sort(L[t])[::-1][5]


def test_gate_rows_sum_to_one_and_match_softmax_then_renormalise():
    """MLG 'Expected Return Format': gate rows sum to 1.  PFD 'The one
    formula': softmax first and renormalise after gives the same numbers as
    softmax over the kept logits."""
    rng = np.random.default_rng(5)
    L = (3.0 * rng.standard_normal((300, 32))).astype(np.float32)
    for k in (1, 2, 4, 8):
        idx = O.top_k(L, k)
        g = O.renormalised_gates(L, idx).astype(np.float64)
        np.testing.assert_allclose(g.sum(axis=1), 1.0, atol=1e-6)
        p = O.softmax_rows(L)
        pk = np.take_along_axis(p, idx.astype(np.int64), 1)
        np.testing.assert_allclose(g, pk / pk.sum(axis=1, keepdims=True), rtol=1e-6)


def test_router_logits_rounding_and_bias_noise_order():
    """Logits are the fp64 dot product rounded once to fp32, then the bias and
    the noise are added in fp32, in that order (PFD 'The code', ``router``)."""
    x = np.array([[1.0, 2.0 ** -30]], dtype=np.float32)
    W = np.array([[1.0], [1.0]], dtype=np.float32)
    L = O.router_logits(x, W, "f32")
    assert L.dtype == np.float32 and L[0, 0] == np.float32(1.0 + 2.0 ** -30)  # == 1.0 in fp32
    bias = np.array([2.0 ** -24], dtype=np.float32)
    noise = np.array([[2.0 ** -24]], dtype=np.float32)
    # (1 + 2^-24) rounds to 1 (tie to even), twice: result stays 1.0.
    assert O.router_logits(x, W, "f32", bias, noise)[0, 0] == np.float32(1.0)
    # Summed first in fp64 the two would give 1 + 2^-23, a different fp32 value.
    assert np.float32(1.0 + 2.0 ** -23) != np.float32(1.0)


# --- dispatch and capacity ---------------------------------------------------

def test_capacity_rounding():
    assert O.capacity(0.0, 64, 1, 8) is None
    assert O.capacity(-1.0, 64, 1, 8) is None
    assert O.capacity(1.25, 10, 1, 4) == 4          # 3.125 rounds up
    assert O.capacity(1.25, 4096, 1, 64) == 80       # switch_relu workload
    assert O.capacity(1.0, 16384, 6, 64) == 1536     # fine_grained workload


def _logits_for_counts(counts, T, E, rng):
    """Top-1 logits whose argmax gives each expert counts[e] tokens, shuffled."""
    experts = np.repeat(np.arange(E), counts)
    rng.shuffle(experts)
    L = rng.standard_normal((T, E)).astype(np.float32)
    L[np.arange(T), experts] = 10.0
    return L


def test_pfd_capacity_drop_table(golden_dir):
    """PFD 'Switch': 64 tokens, 8 experts, top-1; capacity 8/10/16 for
    factors 1.0/1.25/2.0 drops 15/7/0 tokens on the random-init router and
    56/54/48 on the collapsed one."""
    g = _load(golden_dir, "pfd_capacity_table.json")
    rng = np.random.default_rng(0)
    for name, router in g["routers"].items():
        L = _logits_for_counts(router["counts"], g["tokens"], g["experts"], rng)
        idx = O.top_k(L, g["top_k"])
        for factor, dropped in router["dropped"].items():
            cap = O.capacity(float(factor), g["tokens"], g["top_k"], g["experts"])
            assert cap == g["capacity"][factor]
            d = O.dispatch(idx, g["experts"], float(factor))
            assert d["counts"].tolist() == router["counts"], name
            assert int(d["drop_mask"].sum()) == dropped, (name, factor)
            assert d["kept"].tolist() == np.minimum(router["counts"], cap).tolist()


@pytest.mark.parametrize("cf", [0.0, 0.5, 1.0, 1.25])
def test_dispatch_invariants(cf):
    """Counts sum to T*k (PFD 'The router': 32 = 16 tokens x k=2); kept =
    min(count, cap); grouped rows are a permutation of [0, R); each expert's
    segment lists tokens in increasing order (first come, first served); a
    slot is dropped iff earlier tokens already filled the expert."""
    rng = np.random.default_rng(int(cf * 100) + 1)
    T, E, k = 300, 12, 3
    L = rng.standard_normal((T, E)).astype(np.float32)
    L[:, 2] += 1.0                                    # one busier expert
    idx = O.top_k(L, k)
    d = O.dispatch(idx, E, cf)
    assert d["counts"].sum() == T * k
    assert d["counts"].tolist() == np.bincount(idx.ravel(), minlength=E).tolist()
    cap = O.capacity(cf, T, k, E)
    kept = d["counts"] if cap is None else np.minimum(d["counts"], cap)
    assert d["kept"].tolist() == kept.tolist()
    R = int(kept.sum())
    assert d["offsets"][-1] == R
    rows = d["dest"][d["dest"] >= 0]
    assert sorted(rows.tolist()) == list(range(R))
    for e in range(E):
        seg = d["perm_token"][d["offsets"][e]:d["offsets"][e + 1]]
        assert (np.diff(seg) > 0).all()
        # first come first served: kept tokens are the earliest ones on e
        on_e = [t for t in range(T) if e in idx[t]]
        assert seg.tolist() == on_e[:len(seg)]
    for t in range(T):
        for j in range(k):
            if d["dest"][t, j] >= 0:
                assert d["perm_token"][d["dest"][t, j]] == t
    np.testing.assert_array_equal(d["f"], d["counts"] / float(T * k))


# --- experts and combine -----------------------------------------------------

def _tiny(kind, dtype, T=40, d=16, h=24, d_out=16, E=6, k=2, seed=0):
    from workloads import Workload
    w = Workload("t", T=T, d=d, d_hidden=h if kind != "linear" else 0, d_out=d_out, E=E,
                 top_k=k, kind=kind, dtype=dtype, capacity_factor=0.0)
    return w, make_inputs(w, seed)


@pytest.mark.parametrize("kind,dtype", [("linear", "f32"), ("relu", "bf16"), ("swiglu", "bf16"),
                                        ("relu", "f32"), ("swiglu", "f32")])
@pytest.mark.parametrize("cf", [0.0, 0.75, 1.0])
@pytest.mark.parametrize("k", [1, 2, 3])
def test_matches_brute_force(kind, dtype, cf, k):
    """The looped, routed oracle equals the independent dense formulation."""
    w, inp = _tiny(kind, dtype, k=k, seed=k + int(cf * 10))
    rng = np.random.default_rng(99)
    bias = rng.standard_normal(w.E).astype(np.float32)
    noise = (0.3 * rng.standard_normal((w.T, w.E))).astype(np.float32)
    weights = {key: inp[key] for key in ("W_in", "W_up", "W_out")}
    a = O.moe_forward(inp["x"], inp["W_router"], weights, top_k=k, kind=kind, dtype=dtype,
                      d_out=w.d_out, capacity_factor=cf, logit_bias=bias, noise=noise)
    b = O.moe_forward_brute_force(inp["x"], inp["W_router"], weights, top_k=k, kind=kind,
                                  dtype=dtype, capacity_factor=cf, logit_bias=bias, noise=noise)
    assert (a["expert_indices"] == b["expert_indices"]).all()
    np.testing.assert_allclose(a["gates"], b["gates"], rtol=1e-6, atol=1e-7)
    # The oracle combines with fp32 gates (the layer's gate output), the dense
    # form with fp64 gates: they differ by the fp32 rounding of a gate.
    scale = float(np.abs(b["output"]).max())
    np.testing.assert_allclose(a["output"], b["output"], rtol=0, atol=2e-7 * scale)
    assert abs(a["aux_loss"] - b["aux_loss"]) <= 1e-12 * max(1.0, abs(b["aux_loss"]))
    assert a["counts"].tolist() == b["counts"].tolist()
    assert int(a["drop_mask"].sum()) == w.T * k - int(b["keep"].sum())


def test_top1_gate_is_one_and_output_is_that_experts_output():
    """MLG 'Edge cases': top_k = 1 (Switch) -> the gate is 1 and the output
    is the chosen expert's output, here checked against numpy einsum."""
    w, inp = _tiny("linear", "f32", k=1)
    weights = {key: inp[key] for key in ("W_in", "W_up", "W_out")}
    r = O.moe_forward(inp["x"], inp["W_router"], weights, top_k=1, kind="linear", dtype="f32",
                      d_out=w.d_out)
    assert (r["gates"] == np.float32(1.0)).all()
    X = inp["x"].astype(np.float64)
    W = inp["W_in"].astype(np.float64)
    e = r["expert_indices"][:, 0]
    ref = np.einsum("td,tdo->to", X, W[e])
    np.testing.assert_allclose(r["output"], ref, rtol=1e-12, atol=1e-12)


def test_linear_layer_matches_einsum_definition():
    """MLG 'Algorithm' 3: y_t = sum_j gates[t,j] * x_t @ W_{idx[t,j]}, written
    with numpy einsum over a gathered weight tensor, on the tiny_linear shape."""
    w = WORKLOADS["tiny_linear"]
    inp = make_inputs(w, seed=0)
    weights = {key: inp[key] for key in ("W_in", "W_up", "W_out")}
    r = O.moe_forward(inp["x"], inp["W_router"], weights, top_k=w.top_k, kind="linear",
                      dtype="f32", d_out=w.d_out)
    X = inp["x"].astype(np.float64)
    W = inp["W_in"].astype(np.float64)
    idx = r["expert_indices"]
    g = r["gates"].astype(np.float64)
    ref = np.einsum("tj,td,tjdo->to", g, X, W[idx])
    np.testing.assert_allclose(r["output"], ref, rtol=1e-12, atol=1e-12)


def test_token_output_matches_layer():
    """The one-token path used for sampled full-size checks agrees with the
    layer (with drops)."""
    w, inp = _tiny("swiglu", "bf16", k=2, seed=4)
    weights = {key: inp[key] for key in ("W_in", "W_up", "W_out")}
    r = O.moe_forward(inp["x"], inp["W_router"], weights, top_k=2, kind="swiglu", dtype="bf16",
                      d_out=w.d_out, capacity_factor=0.8)
    assert r["drop_mask"].sum() > 0
    for t in range(w.T):
        y = O.token_output(t, inp["x"], "bf16", "swiglu", weights, r["expert_indices"], r["gates"],
                           r["dest"])
        np.testing.assert_allclose(y, r["output"][t], rtol=1e-12, atol=1e-12)


def test_sampled_outputs_match_layer():
    """The expert-by-expert sampled path agrees with the layer's rows."""
    w, inp = _tiny("relu", "bf16", k=3, seed=5)
    weights = {key: inp[key] for key in ("W_in", "W_up", "W_out")}
    r = O.moe_forward(inp["x"], inp["W_router"], weights, top_k=3, kind="relu", dtype="bf16",
                      d_out=w.d_out, capacity_factor=0.9)
    tokens = [0, 7, 7, 13, 39]
    y = O.sampled_outputs(tokens, inp["x"], "bf16", "relu", weights, r["expert_indices"],
                          r["gates"], r["dest"])
    np.testing.assert_allclose(y, r["output"][tokens], rtol=1e-12, atol=1e-12)


def test_idle_expert_weights_do_not_change_output():
    """PFD 'Hot shards': an expert that receives no token can have any
    weights; the output does not change (bit for bit)."""
    w, inp = _tiny("relu", "bf16", E=6, k=1, seed=2)
    bias = np.zeros(w.E, dtype=np.float32)
    bias[5] = -50.0                                   # expert 5 never chosen
    weights = {key: inp[key] for key in ("W_in", "W_up", "W_out")}
    a = O.moe_forward(inp["x"], inp["W_router"], weights, top_k=1, kind="relu", dtype="bf16",
                      d_out=w.d_out, logit_bias=bias)
    assert a["counts"][5] == 0
    W_in = inp["W_in"].copy()
    W_in[5] = np.uint16(0x3F80)                       # 1.0 everywhere
    b = O.moe_forward(inp["x"], inp["W_router"], dict(weights, W_in=W_in), top_k=1, kind="relu",
                      dtype="bf16", d_out=w.d_out, logit_bias=bias)
    assert np.array_equal(a["output"], b["output"])


def test_dropped_everywhere_gives_zero_and_gates_not_renormalised():
    """PFD 'Switch': a dropped token gets 0 from the experts; MLG: gates still
    sum to 1 (they are reported before capacity)."""
    w, inp = _tiny("relu", "f32", T=32, E=4, k=1, seed=8)
    bias = np.array([40.0, 0, 0, 0], dtype=np.float32)          # everyone on expert 0
    weights = {key: inp[key] for key in ("W_in", "W_up", "W_out")}
    r = O.moe_forward(inp["x"], inp["W_router"], weights, top_k=1, kind="relu", dtype="f32",
                      d_out=w.d_out, capacity_factor=0.5, logit_bias=bias)
    cap = O.capacity(0.5, 32, 1, 4)
    assert cap == 4 and r["kept"].tolist() == [4, 0, 0, 0]
    assert (r["output"][4:] == 0).all() and (np.abs(r["output"][:4]).sum(axis=1) > 0).all()
    np.testing.assert_allclose(r["gates"].sum(axis=1), 1.0)


def test_repeated_runs_are_bit_identical():
    """PFD 'The router': noise off, two runs give identical outputs."""
    w, inp = _tiny("swiglu", "bf16", seed=6)
    weights = {key: inp[key] for key in ("W_in", "W_up", "W_out")}
    kw = dict(top_k=2, kind="swiglu", dtype="bf16", d_out=w.d_out, capacity_factor=1.0)
    a = O.moe_forward(inp["x"], inp["W_router"], weights, **kw)
    b = O.moe_forward(inp["x"], inp["W_router"], weights, **kw)
    assert np.array_equal(a["output"], b["output"]) and a["aux_loss"] == b["aux_loss"]


def test_mlg_shape_example(golden_dir):
    """MLG 'Examples': x (6,4), W_router (4,4), expert_weights (4,4,3), top_k=2."""
    g = _load(golden_dir, "mlg_examples.json")["shape_example"]
    rng = np.random.default_rng(1)
    x = rng.standard_normal(g["x"]).astype(np.float32)
    W = rng.standard_normal(g["W_router"]).astype(np.float32)
    We = rng.standard_normal(g["expert_weights"]).astype(np.float32)
    r = O.moe_forward(x, W, {"W_in": We}, top_k=g["top_k"], kind="linear", dtype="f32",
                      d_out=g["expert_weights"][2])
    assert list(r["output"].shape) == g["output"]
    assert list(r["expert_indices"].shape) == g["expert_indices"]
    assert list(r["gates"].shape) == g["gates"]
    assert isinstance(r["aux_loss"], float)


def test_swiglu_closed_form_single_element():
    """SwiGLU on 1x1 matrices: (silu(a x) * (b x)) * c with silu(z) = z/(1+e^-z)."""
    x = np.array([[2.0]])
    y = O.expert_forward("swiglu", x, np.array([[0.5]]), np.array([[3.0]]), np.array([[-1.0]]))
    z = 1.0
    assert abs(y[0, 0] - (z / (1.0 + math.exp(-z))) * 6.0 * -1.0) < 1e-15
    y = O.expert_forward("relu", x, np.array([[-0.5, 0.5]]), None, np.array([[1.0], [10.0]]))
    assert y[0, 0] == 10.0


# --- dtype helpers -----------------------------------------------------------

def test_f64_to_bf16_matches_torch_on_fp32_values():
    """For values exactly representable in fp32, one rounding to bf16 must
    equal torch's fp32 -> bf16 conversion (round to nearest, ties to even)."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 8, 20000),
                        [0.0, -0.0, 1.0, -1.0, 1.00390625, 1.01171875, 3.0e38 / 4]]).astype(np.float32)
    ours = O.f64_to_bf16_bits(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_f64_to_bf16_single_rounding():
    """A value just above a bf16 halfway point in fp64 rounds up, although
    rounding through fp32 first would land on the tie and round to even."""
    v = 1.0 + 2.0 ** -8 + 2.0 ** -40              # halfway between 1 and 1+2^-7, nudged up
    assert O.f64_to_bf16_bits(np.array([v]))[0] == 0x3F81
    assert O.f64_to_bf16_bits(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80


def test_exact_router_inputs_are_exact():
    """The exact-logit generator: fp32 logits under different summation
    orders agree bit for bit with the fp64 sum."""
    inp = make_exact_router_inputs(64, 512, 16, "f32", seed=2)
    x, W = inp["x"].astype(np.float32), inp["W_router"]
    L64 = O.router_logits(inp["x"], W, "f32")
    L32 = np.zeros((64, 16), dtype=np.float32)
    for i in range(512):                              # naive fp32 order
        L32 = (L32 + x[:, i:i + 1] * W[i:i + 1, :]).astype(np.float32)
    assert np.array_equal(L64, L32)
