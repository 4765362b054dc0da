"""The experts' backward on the GPU (moe_expert_ffn_backward,
moe_permute_backward) against the oracle (expert_backward, moe_backward;
pinned by finite differences of the fp64 layer in test_oracle_backward.py).

The grouped rows (x_perm, offsets, dest) come from the GPU forward and a
seeded dy_perm is fed to both sides, so the per-expert comparison is about
the experts' backward alone; the whole-layer test composes every GPU piece
and compares with the oracle's moe_backward.

Bounds:
* linear experts (fp32 throughout): max |gpu - oracle| <= 1e-4 max |oracle|
  per tensor, the fp32 rule of the forward;
* bf16 experts: the inputs are exact bf16 and the GPU accumulates in fp32,
  but it rounds two intermediates to bf16 on the way (dY, the tensor-core
  operand of dH; then dA, dB and H, the operands of dX and of the weight
  gradients), each a relative error of at most u = 2^-9.  Through a
  contraction those errors are uncorrelated, so a tensor's normwise relative
  error is about sqrt(2) u / sqrt(3) = 1.6e-3 and at most 2u = 3.9e-3 to
  first order; the bound is ||gpu - oracle||_F <= 1e-2 ||oracle||_F per
  tensor (dx_perm of all rows, each expert's dW block), and elementwise
  |gpu - oracle| <= 0.1 RMS(oracle) + 2e-2 |oracle| (the second term for
  heavy-tailed elements far above the RMS, whose rounding error scales with
  their own size), which no misplaced tile or row passes.  (The forward's elementwise 2e-2 RMS rule covers one rounding;
  here the tails of two chained roundings reach 2-3 % of RMS at 10^5-10^6
  elements.)
* an expert without rows: its dW blocks are exactly zero;
* rows of dx_perm at and beyond offsets[E]: untouched.
"""
import numpy as np
import pytest
import torch

from gpu_util import REL_F32, cfg_of, dev, host
from mixture_experts_top_b200 import api
from oracle import moe_oracle as O
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "mixtral": WORKLOADS["mixtral"].replace(T=600, d=512, d_hidden=1024, d_out=512),
    # DH = 352 is not a multiple of 64: padded hidden columns
    "fine_grained": WORKLOADS["fine_grained"].replace(T=1100, d=256, d_hidden=352, d_out=256),
    "switch_relu": WORKLOADS["switch_relu"].replace(T=1024, d=256, d_hidden=512, d_out=256),
    "tiny_linear": WORKLOADS["tiny_linear"],
    # d and d_out not multiples of the 256-column tile, rows of one expert
    # spanning several 256-row tiles
    "ragged": WORKLOADS["mixtral"].replace(T=700, d=200, d_hidden=136, d_out=72, E=5, top_k=2),
}


def _route_dispatch(w, inp, cfg, ws):
    T, k, E = w.T, w.top_k, w.E
    i32 = dict(dtype=torch.int32, device="cuda")
    x = dev(inp["x"])
    t = dict(idx=torch.empty((T, k), **i32), gates=torch.empty((T, k), device="cuda"),
             P=torch.empty(E, device="cuda"), L=torch.empty((T, E), device="cuda"),
             counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
             dest=torch.empty((T, k), **i32), perm=torch.empty(T * k, **i32),
             drop=torch.empty((T, k), dtype=torch.uint8, device="cuda"),
             f=torch.empty(E, device="cuda"), aux=torch.empty(1, device="cuda"),
             x_perm=torch.empty((T * k, w.d), dtype=x.dtype, device="cuda"))
    api.moe_route(cfg, x, dev(inp["W_router"]), dev(inp["logit_bias"]), dev(inp["noise"]),
                  t["idx"], t["gates"], t["P"], t["L"], ws)
    api.moe_dispatch(cfg, x, t["idx"], t["P"], t["counts"], t["offsets"], t["dest"], t["perm"],
                     t["drop"], t["f"], t["aux"], t["x_perm"], ws)
    return x, t


def _grads(w, T):
    """Output buffers of moe_expert_ffn_backward, filled with a sentinel."""
    f32 = dict(dtype=torch.float32, device="cuda")
    R = T * w.top_k
    out = dict(dx_perm=torch.full((R, w.d), 7.0, **f32))
    if w.kind == "linear":
        out.update(dW_in=torch.full((w.E, w.d, w.d_out), 7.0, **f32), dW_up=None, dW_out=None)
    else:
        out.update(dW_in=torch.full((w.E, w.d, w.d_hidden), 7.0, **f32),
                   dW_up=(torch.full((w.E, w.d, w.d_hidden), 7.0, **f32)
                          if w.kind == "swiglu" else None),
                   dW_out=torch.full((w.E, w.d_hidden, w.d_out), 7.0, **f32))
    return out


NORM_BWD = 1e-2     # normwise relative bound of the bf16 backward (module docstring)
MAX_BWD = 0.1       # elementwise bound, in units of RMS(oracle) ...
REL_BWD = 2e-2      # ... plus this fraction of |oracle|


def _check(w, got, ref, name="", elementwise=True, norm_tol=NORM_BWD):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.isfinite(got).all(), name
    if w.kind == "linear":
        assert np.abs(got - ref).max() <= REL_F32 * max(np.abs(ref).max(), 1e-30), name
    else:
        nref = float(np.linalg.norm(ref))
        rms = nref / np.sqrt(max(ref.size, 1))
        nerr = float(np.linalg.norm(got - ref))
        assert nerr <= norm_tol * max(nref, 1e-30), (name, nerr / max(nref, 1e-30), "normwise")
        if elementwise:
            excess = np.abs(got - ref) - (MAX_BWD * rms + REL_BWD * np.abs(ref))
            assert excess.max() <= 0, (name, float(np.abs(got - ref).max() / max(rms, 1e-30)),
                                       "elementwise")


@pytest.mark.parametrize("name", list(CASES))
def test_expert_backward_against_oracle(name):
    w = CASES[name]
    inp = make_inputs(w, seed=31)
    cfg = cfg_of(w)
    ws = api.alloc_workspace(cfg)
    x, t = _route_dispatch(w, inp, cfg, ws)
    R = int(host(t["offsets"])[-1])
    rng = np.random.default_rng(32)
    dy = np.zeros((w.T * w.top_k, w.d_out), np.float32)
    dy[:R] = rng.standard_normal((R, w.d_out)).astype(np.float32)
    g = _grads(w, w.T)
    bws = api.alloc_backward_workspace(cfg)
    W = {key: dev(inp[key]) for key in ("W_in", "W_up", "W_out")}
    api.moe_expert_ffn_backward(cfg, t["x_perm"], t["offsets"], W["W_in"], W["W_up"], W["W_out"],
                                dev(dy), g["dx_perm"], g["dW_in"], g["dW_up"], g["dW_out"], bws)
    torch.cuda.synchronize()
    assert api.moe_device_status(bws) == 0 and api.moe_device_status(ws) == 0
    offs = host(t["offsets"])
    xp = host(t["x_perm"])
    weights = {key: inp[key] for key in ("W_in", "W_up", "W_out")}
    dx_ref = np.zeros((R, w.d))
    keys = [("W_in", "dW_in"), ("W_up", "dW_up"), ("W_out", "dW_out")]
    dW_ref = {gk: np.zeros(np.asarray(inp[k]).shape) for k, gk in keys if inp[k] is not None}
    idle = []
    for e in range(w.E):
        lo, hi = int(offs[e]), int(offs[e + 1])
        if hi == lo:
            idle.append(e)
            continue
        r = O.expert_backward(w.kind, O.widen(xp[lo:hi], w.dtype),
                              *O.expert_weights(weights, e, w.dtype), dy[lo:hi])
        dx_ref[lo:hi] = r["dx"]
        for gk in dW_ref:
            dW_ref[gk][e] = r[gk]
    _check(w, host(g["dx_perm"])[:R], dx_ref, "dx_perm")
    assert (host(g["dx_perm"])[R:] == 7.0).all(), "rows beyond offsets[E] were written"
    for gk, ref in dW_ref.items():
        got = host(g[gk])
        for e in range(w.E):
            if e in idle:
                assert (got[e] == 0).all(), (gk, e)
            else:
                _check(w, got[e], ref[e], f"{gk}[{e}]")


def test_expert_backward_idle_experts_and_repeat():
    """A +30 bias on one expert routes every top-1 slot there: the other
    experts get exactly zero weight gradients; two calls on one workspace
    give identical bits (no atomics)."""
    w = CASES["fine_grained"].replace(top_k=1, capacity_factor=0.0, n_hot=0, T=300)
    inp = make_inputs(w, seed=33)
    bias = np.zeros(w.E, np.float32)
    bias[5] = 30.0
    inp["logit_bias"] = bias
    cfg = cfg_of(w)
    ws = api.alloc_workspace(cfg)
    _, t = _route_dispatch(w, inp, cfg, ws)
    assert (host(t["idx"])[:, 0] == 5).all()
    dy = dev(np.random.default_rng(1).standard_normal((w.T, w.d_out)).astype(np.float32))
    W = {key: dev(inp[key]) for key in ("W_in", "W_up", "W_out")}
    bws = api.alloc_backward_workspace(cfg)
    runs = []
    for _ in range(2):
        g = _grads(w, w.T)
        api.moe_expert_ffn_backward(cfg, t["x_perm"], t["offsets"], W["W_in"], W["W_up"],
                                    W["W_out"], dy, g["dx_perm"], g["dW_in"], g["dW_up"],
                                    g["dW_out"], bws)
        torch.cuda.synchronize()
        runs.append({k: host(v) for k, v in g.items() if v is not None})
    assert api.moe_device_status(bws) == 0
    # nothing but the error word is left in the control block
    ctrl = host(bws[:256]).view(np.uint32)
    assert (ctrl[1:] == 0).all(), ctrl[ctrl != 0]
    for key in runs[0]:
        assert np.array_equal(runs[0][key], runs[1][key]), key
        if key != "dx_perm":
            others = np.delete(runs[0][key], 5, axis=0)
            assert (others == 0).all(), key
            assert np.abs(runs[0][key][5]).max() > 0, key


def test_expert_backward_rejects_bad_offsets():
    """Offsets that are not a partition of the rows: recorded on the error
    word (code 2), nothing read or written outside the buffers."""
    w = CASES["mixtral"].replace(T=64)
    cfg = cfg_of(w)
    inp = make_inputs(w, seed=3)
    R = w.T * w.top_k
    offsets = torch.tensor([0, 10, 5, 30, 40, 50, 60, 70, R + 500], dtype=torch.int32,
                           device="cuda")
    x_perm = torch.zeros((R, w.d), dtype=torch.bfloat16, device="cuda")
    dy = torch.zeros((R, w.d_out), device="cuda")
    g = _grads(w, w.T)
    bws = api.alloc_backward_workspace(cfg)
    api.moe_expert_ffn_backward(cfg, x_perm, offsets, dev(inp["W_in"]), dev(inp["W_up"]),
                                dev(inp["W_out"]), dy, g["dx_perm"], g["dW_in"], g["dW_up"],
                                g["dW_out"], bws)
    torch.cuda.synchronize()
    assert api.moe_device_status(bws) == 2


def _layer_backward_gpu(w, inp, dy_tok, daux):
    """Every GPU piece in order: forward (route with logits, dispatch,
    experts, combine), combine backward, experts' backward, router backward,
    rows back to tokens."""
    cfg = cfg_of(w)
    ws = api.alloc_workspace(cfg)
    x, t = _route_dispatch(w, inp, cfg, ws)
    T, k, E = w.T, w.top_k, w.E
    W = {key: dev(inp[key]) for key in ("W_in", "W_up", "W_out")}
    y_perm = torch.zeros((T * k, w.d_out), device="cuda")
    api.moe_expert_ffn(cfg, t["x_perm"], t["offsets"], W["W_in"], W["W_up"], W["W_out"], y_perm,
                       ws)
    dyp = torch.zeros((T * k, w.d_out), device="cuda")
    dg = torch.empty((T, k), device="cuda")
    api.moe_combine_backward(cfg, dev(dy_tok), y_perm, t["dest"], t["gates"], dyp, dg)
    g = _grads(w, T)
    bws = api.alloc_backward_workspace(cfg)
    api.moe_expert_ffn_backward(cfg, t["x_perm"], t["offsets"], W["W_in"], W["W_up"], W["W_out"],
                                dyp, g["dx_perm"], g["dW_in"], g["dW_up"], g["dW_out"], bws)
    dx_r = torch.empty((T, w.d), device="cuda")
    dWr = torch.empty((w.d, E), device="cuda")
    db = torch.empty(E, device="cuda")
    api.moe_route_backward(cfg, x, dev(inp["W_router"]), t["L"], t["idx"], t["gates"], t["f"], dg,
                           torch.tensor([daux], dtype=torch.float32, device="cuda"), 0, dx_r,
                           dWr, db, None, ws)
    dx = torch.empty((T, w.d), device="cuda")
    api.moe_permute_backward(cfg, g["dx_perm"], t["dest"], dx_r, dx)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 0 and api.moe_device_status(bws) == 0
    out = dict(dx=host(dx), dW_router=host(dWr), dbias=host(db), idx=host(t["idx"]),
               L=host(t["L"]))
    for key in ("dW_in", "dW_up", "dW_out"):
        out[key] = None if g[key] is None else host(g[key])
    return out


@pytest.mark.parametrize("name", ["mixtral", "fine_grained", "switch_relu", "tiny_linear"])
def test_layer_backward_against_oracle(name):
    w = CASES[name]
    inp = make_inputs(w, seed=41)
    rng = np.random.default_rng(42)
    dy = rng.standard_normal((w.T, w.d_out)).astype(np.float32)
    if w.dtype == "bf16":
        from workloads import f32_to_bf16_bits
        dy_dev = f32_to_bf16_bits(dy)
        dy_ref = (dy_dev.astype(np.uint32) << 16).view(np.float32)
    else:
        dy_dev = dy_ref = dy
    got = _layer_backward_gpu(w, inp, dy_dev, 0.7)
    weights = {key: inp[key] for key in ("W_in", "W_up", "W_out")}
    ref = O.moe_backward(inp["x"], inp["W_router"], weights, top_k=w.top_k, kind=w.kind,
                         dtype=w.dtype, d_out=w.d_out, dy=dy_ref, daux=0.7,
                         capacity_factor=w.capacity_factor, logit_bias=inp["logit_bias"],
                         noise=inp["noise"])
    ref_idx = O.top_k(O.router_logits(inp["x"], inp["W_router"], w.dtype, inp["logit_bias"],
                                      inp["noise"]), w.top_k)
    # the routing decisions must agree, else the two layers differ by design
    # (the seeds are chosen with no near-tie that the fp32 logits could flip)
    assert np.array_equal(got["idx"], ref_idx)
    # The experts' weight gradients carry the experts' own rounding only (the
    # bounds above).  dx, dW_router and dbias also carry the forward's: the
    # gate gradients are <dy, Y> with the GPU's bf16-computed expert rows Y
    # (within 2e-2 RMS(Y) of the oracle's), and the gate softmax's backward
    # g (dg - sum g dg) subtracts nearly equal terms, so their error is
    # judged normwise, at twice the forward's relative bound.
    for key in ("dW_in", "dW_up", "dW_out"):
        if ref[key] is not None:
            _check(w, got[key], ref[key], key)
    for key in ("dx", "dW_router", "dbias"):
        _check(w, got[key], ref[key], key, elementwise=False, norm_tol=4e-2)


TRAIN_CASES = dict(CASES)
# 1024 grouped rows per expert on average: the forward runs on CTA pairs
TRAIN_CASES["mixtral_pairs"] = WORKLOADS["mixtral"].replace(T=4096, d=256, d_hidden=512,
                                                            d_out=256)


@pytest.mark.parametrize("name", ["mixtral", "fine_grained", "switch_relu", "ragged",
                                  "mixtral_pairs"])
def test_training_forward_and_saved_backward(name):
    """moe_expert_ffn_train writes the same expert rows as moe_expert_ffn
    (bit for bit) and keeps the pre-activations in the backward workspace;
    moe_expert_ffn_backward_saved then gives the recomputing backward's
    gradients up to the order in which the tensor cores summed A and B, and
    stays within the oracle bounds.  The backward workspace starts filled
    with NaN, so a pre-activation the forward did not write (a padding row,
    a padding hidden unit) would show."""
    w = TRAIN_CASES[name]
    inp = make_inputs(w, seed=41)
    cfg = cfg_of(w)
    ws = api.alloc_workspace(cfg)
    _, t = _route_dispatch(w, inp, cfg, ws)
    R = int(host(t["offsets"])[-1])
    W = {key: dev(inp[key]) for key in ("W_in", "W_up", "W_out")}
    f32 = dict(dtype=torch.float32, device="cuda")
    y_plain = torch.full((w.T * w.top_k, w.d_out), 3.0, **f32)
    y_train = torch.full((w.T * w.top_k, w.d_out), 3.0, **f32)
    api.moe_expert_ffn(cfg, t["x_perm"], t["offsets"], W["W_in"], W["W_up"], W["W_out"], y_plain,
                       ws)
    bws = api.alloc_backward_workspace(cfg)
    bws[256:].view(torch.uint8).fill_(0xFF)          # NaN everywhere but the error word
    api.moe_expert_ffn_train(cfg, t["x_perm"], t["offsets"], W["W_in"], W["W_up"], W["W_out"],
                             y_train, ws, bws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 0
    assert np.array_equal(host(y_plain), host(y_train))

    rng = np.random.default_rng(42)
    dy = np.zeros((w.T * w.top_k, w.d_out), np.float32)
    dy[:R] = rng.standard_normal((R, w.d_out)).astype(np.float32)
    g_saved, g_rec = _grads(w, w.T), _grads(w, w.T)
    api.moe_expert_ffn_backward_saved(cfg, t["x_perm"], t["offsets"], W["W_in"], W["W_up"],
                                      W["W_out"], dev(dy), g_saved["dx_perm"], g_saved["dW_in"],
                                      g_saved["dW_up"], g_saved["dW_out"], bws)
    bws2 = api.alloc_backward_workspace(cfg)
    api.moe_expert_ffn_backward(cfg, t["x_perm"], t["offsets"], W["W_in"], W["W_up"], W["W_out"],
                                dev(dy), g_rec["dx_perm"], g_rec["dW_in"], g_rec["dW_up"],
                                g_rec["dW_out"], bws2)
    torch.cuda.synchronize()
    assert api.moe_device_status(bws) == 0 and api.moe_device_status(bws2) == 0
    for key in ("dx_perm", "dW_in", "dW_up", "dW_out"):
        if g_saved[key] is None:
            continue
        a, b = host(g_saved[key]), host(g_rec[key])
        if key == "dx_perm":
            a, b = a[:R], b[:R]
        assert np.isfinite(a).all(), key
        nb = float(np.linalg.norm(b))
        assert float(np.linalg.norm(a - b)) <= 2e-3 * max(nb, 1e-30), key
    # and against the oracle, on the saved path
    offs = host(t["offsets"])
    xp = host(t["x_perm"])
    weights = {key: inp[key] for key in ("W_in", "W_up", "W_out")}
    dx_ref = np.zeros((R, w.d))
    for e in range(w.E):
        lo, hi = int(offs[e]), int(offs[e + 1])
        if hi > lo:
            r = O.expert_backward(w.kind, O.widen(xp[lo:hi], w.dtype),
                                  *O.expert_weights(weights, e, w.dtype), dy[lo:hi])
            dx_ref[lo:hi] = r["dx"]
    _check(w, host(g_saved["dx_perm"])[:R], dx_ref, "dx_perm (saved)")


def test_training_forward_and_saved_backward_empty_batch():
    """T = 0: the training forward writes nothing and the saved backward
    gives zero weight gradients, like the recomputing one."""
    w = CASES["mixtral"].replace(T=0)
    cfg = cfg_of(w)
    ws = api.alloc_workspace(cfg)
    bws = api.alloc_backward_workspace(cfg)
    W = {key: dev(v) for key, v in
         zip(("W_in", "W_up", "W_out"),
             (np.zeros((w.E, w.d, w.d_hidden), np.uint16), np.zeros((w.E, w.d, w.d_hidden), np.uint16),
              np.zeros((w.E, w.d_hidden, w.d_out), np.uint16)))}
    offsets = torch.zeros(w.E + 1, dtype=torch.int32, device="cuda")
    api.moe_expert_ffn_train(cfg, None, offsets, W["W_in"], W["W_up"], W["W_out"], None, ws, bws)
    g = _grads(w, 0)
    api.moe_expert_ffn_backward_saved(cfg, None, offsets, W["W_in"], W["W_up"], W["W_out"], None,
                                      None, g["dW_in"], g["dW_up"], g["dW_out"], bws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 0 and api.moe_device_status(bws) == 0
    for key in ("dW_in", "dW_up", "dW_out"):
        assert (host(g[key]) == 0).all(), key
