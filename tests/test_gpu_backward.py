"""Routing backward on the GPU (moe_combine_backward, moe_route_backward)
against the oracle's (combine_backward, route_backward; pinned by finite
differences in test_oracle_backward.py).

The forward intermediates (y_perm, dest, gates, logits, f) come from the
GPU forward and are fed to both sides, so the comparison is about the
backward alone.  Bounds (fp32 with fixed orders, fp64 references):
* dy_perm: one fp32 product per element, within one rounding;
* dgates: an fp32 dot over d_out: d_out 2^-23 sum |dy Y|;
* dlogits: a few roundings of each term: g (|dg| + sum_j |g_j dg_j|) and
  p (|a| + sum_e p_e |a_e|);
* dx, dW, dbias: fp32 sums of E / T terms of the GPU's own dlogits:
  n 2^-23 sum |terms|.
"""
import numpy as np
import pytest
import torch

from gpu_util import cfg_of, dev, host
from mixture_experts_top_b200 import api
from oracle import moe_oracle as O
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

EPS = 2.0 ** -23

CASES = {
    "fine_grained": WORKLOADS["fine_grained"].replace(T=1100, d=256, d_hidden=352, d_out=256),
    "mixtral": WORKLOADS["mixtral"].replace(T=600, d=512, d_hidden=1024, d_out=512),
    "switch_relu": WORKLOADS["switch_relu"].replace(T=1024, d=256, d_hidden=512, d_out=256),
    "tiny_linear": WORKLOADS["tiny_linear"],
    "wide": WORKLOADS["fine_grained"].replace(T=300, d=128, d_hidden=64, d_out=64, E=200, top_k=8,
                                             n_hot=0, capacity_factor=0.5),
}


def _forward(w, inp, cfg, ws):
    T, k, E = w.T, w.top_k, w.E
    i32 = dict(dtype=torch.int32, device="cuda")
    x = dev(inp["x"])
    t = dict(idx=torch.empty((T, k), **i32), gates=torch.empty((T, k), device="cuda"),
             P=torch.empty(E, device="cuda"), L=torch.empty((T, E), device="cuda"),
             counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
             dest=torch.empty((T, k), **i32), perm=torch.empty(T * k, **i32),
             drop=torch.empty((T, k), dtype=torch.uint8, device="cuda"),
             f=torch.empty(E, device="cuda"), aux=torch.empty(1, device="cuda"),
             x_perm=torch.empty((T * k, w.d), dtype=x.dtype, device="cuda"),
             y_perm=torch.zeros((T * k, w.d_out), device="cuda"))
    api.moe_route(cfg, x, dev(inp["W_router"]), dev(inp["logit_bias"]), dev(inp["noise"]),
                  t["idx"], t["gates"], t["P"], t["L"], ws)
    api.moe_dispatch(cfg, x, t["idx"], t["P"], t["counts"], t["offsets"], t["dest"], t["perm"],
                     t["drop"], t["f"], t["aux"], t["x_perm"], ws)
    api.moe_expert_ffn(cfg, t["x_perm"], t["offsets"], dev(inp["W_in"]), dev(inp["W_up"]),
                       dev(inp["W_out"]), t["y_perm"], ws)
    return x, t


@pytest.mark.parametrize("name,T_batch", [("fine_grained", 0), ("mixtral", 0),
                                          ("switch_relu", 0), ("tiny_linear", 0),
                                          ("wide", 0), ("mixtral", 1800)])
def test_routing_backward(name, T_batch):
    w = CASES[name]
    inp = make_inputs(w, seed=21)
    cfg = cfg_of(w)
    ws = api.alloc_workspace(cfg)
    x, t = _forward(w, inp, cfg, ws)
    T, k, E = w.T, w.top_k, w.E
    rng = np.random.default_rng(5)
    dyf = rng.standard_normal((T, w.d_out)).astype(np.float32)
    dy = O.f64_to_bf16_bits(dyf.astype(np.float64)) if w.dtype == "bf16" else dyf
    daux = np.array([0.37], np.float32)
    dy_perm = torch.full((T * k, w.d_out), float("nan"), device="cuda")
    dg = torch.empty((T, k), device="cuda")
    api.moe_combine_backward(cfg, dev(dy), t["y_perm"], t["dest"], t["gates"], dy_perm, dg)
    dx = torch.empty((T, w.d), device="cuda")
    dW = torch.empty((w.d, E), device="cuda")
    db = torch.empty(E, device="cuda")
    dL = torch.empty((T, E), device="cuda")
    api.moe_route_backward(cfg, x, dev(inp["W_router"]), t["L"], t["idx"], t["gates"], t["f"], dg,
                           dev(daux), T_batch, dx, dW, db, dL, ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 0
    h = {key: host(v) for key, v in t.items()}
    g_dy_perm, g_dg, g_dx, g_dW, g_db, g_dL = map(host, (dy_perm, dg, dx, dW, db, dL))

    # combine backward
    Y = h["y_perm"].astype(np.float64)
    dy64 = O.widen(dy, w.dtype)
    dY_ref, dg_ref = O.combine_backward(Y, h["dest"], h["gates"], dy64)
    kept = h["dest"][h["dest"] >= 0]
    assert np.all(np.abs(g_dy_perm[kept] - dY_ref[kept]) <= EPS * np.abs(dY_ref[kept]) + 1e-30)
    unused = np.setdiff1d(np.arange(T * k), kept)
    assert np.isnan(g_dy_perm[unused]).all()
    bound = w.d_out * EPS * np.array([[np.abs(dy64[i]) @ np.abs(Y[r]) if r >= 0 else 0.0
                                       for r in h["dest"][i]] for i in range(T)]) + 1e-30
    assert np.all(np.abs(g_dg - dg_ref) <= bound)
    assert (g_dg[h["drop"] == 1] == 0).all()

    # router backward, on the GPU's own dgates
    r = O.route_backward(inp["x"], inp["W_router"], w.dtype, h["L"], h["idx"], h["gates"], h["f"],
                         g_dg, float(daux[0]), T_batch=T_batch or None)
    # each term's rounding scale: the sums s = sum_j g_j dg_j and p.a are
    # bounded by the sums of their terms' magnitudes (they may cancel)
    g64 = h["gates"].astype(np.float64)
    s_abs = np.sum(np.abs(g64 * g_dg), axis=1, keepdims=True)
    p = O.softmax_rows(h["L"].astype(np.float64))
    a = float(daux[0]) * E * h["f"].astype(np.float64) / (T_batch or T)
    scale = np.zeros((T, E))
    np.put_along_axis(scale, h["idx"].astype(np.int64),
                      g64 * (np.abs(g_dg) + s_abs), axis=1)
    scale += p * (np.abs(a)[None, :] + (p @ np.abs(a))[:, None])
    err = np.abs(g_dL - r["dlogits"])
    lim = 64 * EPS * scale + 1e-12
    bad = np.argwhere(err > lim)
    assert len(bad) == 0, [(int(i), int(e), float(g_dL[i, e]), float(r["dlogits"][i, e]),
                            float(scale[i, e]), bool(e in h["idx"][i]))
                           for i, e in bad[:6]] + [len(bad)]
    W64 = inp["W_router"].astype(np.float64)
    dL64 = g_dL.astype(np.float64)
    assert np.all(np.abs(g_dx - dL64 @ W64.T) <= E * EPS * (np.abs(dL64) @ np.abs(W64.T)) + 1e-30)
    xf = O.widen(inp["x"], w.dtype)
    assert np.all(np.abs(g_dW - xf.T @ dL64) <= T * EPS * (np.abs(xf.T) @ np.abs(dL64)) + 1e-30)
    assert np.all(np.abs(g_db - dL64.sum(0)) <= T * EPS * np.abs(dL64).sum(0) + 1e-30)
    # the gate part conserves each token's logit-gradient mass; aux part too
    assert np.all(np.abs(g_dL.sum(axis=1)) <= 64 * EPS * scale.sum(axis=1) + 1e-9)


def test_route_backward_empty_batch():
    w = CASES["mixtral"].replace(T=0)
    cfg = cfg_of(w)
    ws = api.alloc_workspace(cfg)
    dW = torch.full((w.d, w.E), 5.0, device="cuda")
    db = torch.full((w.E,), 5.0, device="cuda")
    W = torch.zeros((w.d, w.E), device="cuda")
    f = torch.zeros(w.E, device="cuda")
    daux = torch.ones(1, device="cuda")
    api.moe_route_backward(cfg, None, W, None, None, None, f, None, daux, 0, None, dW, db, None, ws)
    torch.cuda.synchronize()
    assert (host(dW) == 0).all() and (host(db) == 0).all()
