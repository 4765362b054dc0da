"""Pins of the oracle's routing backward (combine_backward, route_backward)
by central finite differences of the forward in fp64.

The forward used here is the layer's routing half with every step in fp64
and the top-k choice and the drops held fixed (they are piecewise constant;
the inputs keep every logit gap far above the step size):
    L = x W + bias,  p = softmax(L),  g = softmax over the chosen k,
    y = combine(Y, dest, g),  aux = E sum_e f_e mean_t p_te,
    loss = <dy, y> + daux * aux.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O


def _gates64(L, idx):
    Lk = np.take_along_axis(L, idx, axis=1)
    ez = np.exp(Lk - Lk.max(axis=1, keepdims=True))
    return ez / ez.sum(axis=1, keepdims=True)


def _case(T=7, d=5, E=6, k=3, cap_drop=True, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    W = rng.standard_normal((d, E))
    bias = rng.standard_normal(E)
    L = x @ W + bias
    idx = O.top_k(L.astype(np.float32), k)
    disp = O.dispatch(idx, E, 0.5 if cap_drop else 0.0)
    R = int(disp["offsets"][-1])
    Y = rng.standard_normal((R, 4))
    dy = rng.standard_normal((T, 4))
    f = disp["f"].astype(np.float64)
    return x, W, bias, idx, disp, Y, dy, f


def _loss(x, W, bias, idx, dest, Y, dy, f, daux):
    L = x @ W + bias
    g = _gates64(L, idx)
    y = O.combine(Y, dest, g)
    p = O.softmax_rows(L)
    aux = L.shape[1] * float(f @ p.mean(axis=0))
    return float(np.sum(dy * y)) + daux * aux


@pytest.mark.parametrize("drops", [False, True])
def test_backward_matches_finite_differences(drops):
    x, W, bias, idx, disp, Y, dy, f = _case(cap_drop=drops)
    if drops:
        assert (disp["drop_mask"] == 1).any()
    daux = 0.7
    L = x @ W + bias
    g = _gates64(L, idx)
    dY, dg = O.combine_backward(Y, disp["dest"], g, dy)
    r = O.route_backward(x, W, "f64", L, idx, g, f, dg, daux)
    h = 1e-6
    args = dict(x=x, W=W, bias=bias, Y=Y)
    grads = dict(x=r["dx"], W=r["dW"], bias=r["dbias"], Y=dY)
    for name, a in args.items():
        num = np.zeros_like(a)
        for i in np.ndindex(a.shape):
            ap, am = a.copy(), a.copy()
            ap[i] += h
            am[i] -= h
            kw = dict(args)
            kw[name] = ap
            lp = _loss(kw["x"], kw["W"], kw["bias"], idx, disp["dest"], kw["Y"], dy, f, daux)
            kw[name] = am
            lm = _loss(kw["x"], kw["W"], kw["bias"], idx, disp["dest"], kw["Y"], dy, f, daux)
            num[i] = (lp - lm) / (2 * h)
        assert np.allclose(grads[name], num, rtol=1e-6, atol=1e-8), name


def test_dropped_slots_and_zero_upstream():
    x, W, bias, idx, disp, Y, dy, f = _case(cap_drop=True, seed=3)
    L = x @ W + bias
    g = _gates64(L, idx)
    dY, dg = O.combine_backward(Y, disp["dest"], g, dy)
    assert (dg[disp["drop_mask"] == 1] == 0).all()
    r = O.route_backward(x, W, "f64", L, idx, g, f, np.zeros_like(dg), 0.0)
    assert not r["dlogits"].any() and not r["dW"].any()
    # the gate softmax conserves mass: every token's gate gradient sums to 0
    r = O.route_backward(x, W, "f64", L, idx, g, f, dg, 0.0)
    assert np.allclose(r["dlogits"].sum(axis=1), 0.0, atol=1e-12)


def test_aux_gradient_closed_form_uniform():
    """W = 0, no bias: p = 1/E everywhere; with f uniform (every a_e equal)
    the aux gradient vanishes; with f concentrated on expert 0 it is
    p (a - p.a): (E-1)/E^2 * daux * E / T on expert 0, -1/E^2 * daux * E / T
    elsewhere."""
    T, d, E, k = 4, 3, 5, 2
    x = np.ones((T, d))
    W = np.zeros((d, E))
    L = x @ W
    idx = O.top_k(L.astype(np.float32), k)
    g = _gates64(L, idx)
    r = O.route_backward(x, W, "f64", L, idx, g, np.full(E, 1.0 / E), np.zeros((T, k)), 2.0)
    assert np.allclose(r["dlogits"], 0.0, atol=1e-15)
    f = np.zeros(E)
    f[0] = 1.0
    r = O.route_backward(x, W, "f64", L, idx, g, f, np.zeros((T, k)), 2.0)
    a0 = 2.0 * E * 1.0 / T
    assert np.allclose(r["dlogits"][:, 0], (1 / E) * (a0 - a0 / E))
    assert np.allclose(r["dlogits"][:, 1:], (1 / E) * (0 - a0 / E))


def _layer_loss(x, W, bias, weights, kind, idx, disp, dy, f, daux):
    """The layer in fp64 with the routing decisions held fixed."""
    L = x @ W + bias
    g = _gates64(L, idx)
    E = W.shape[1]
    R = int(disp["offsets"][-1])
    Y = np.zeros((R, dy.shape[1]))
    for e in range(E):
        lo, hi = int(disp["offsets"][e]), int(disp["offsets"][e + 1])
        if hi > lo:
            Y[lo:hi] = O.expert_forward(kind, x[disp["perm_token"][lo:hi]],
                                        *O.expert_weights(weights, e, "f64"))
    y = O.combine(Y, disp["dest"], g)
    aux = E * float(f @ O.softmax_rows(L).mean(axis=0))
    return float(np.sum(dy * y)) + daux * aux


@pytest.mark.parametrize("kind", ["linear", "relu", "swiglu"])
@pytest.mark.parametrize("cf", [0.0, 0.75])
def test_layer_backward_matches_finite_differences(kind, cf):
    T, d, h, d_out, E, k = 6, 4, 5, 3, 4, 2
    rng = np.random.default_rng(7 + len(kind))
    x = rng.standard_normal((T, d))
    W = rng.standard_normal((d, E))
    bias = rng.standard_normal(E)
    L = x @ W + bias
    Ls = -np.sort(-L, axis=1)
    assert (Ls[:, :k] - Ls[:, 1:k + 1]).min() > 1e-3            # no near-tie in the top k
    weights = {"W_in": rng.standard_normal((E, d, d_out if kind == "linear" else h)),
               "W_up": rng.standard_normal((E, d, h)) if kind == "swiglu" else None,
               "W_out": rng.standard_normal((E, h, d_out)) if kind != "linear" else None}
    dy = rng.standard_normal((T, d_out))
    daux = 0.3
    got = O.moe_backward(x, W, weights, top_k=k, kind=kind, dtype="f64", d_out=d_out, dy=dy,
                         daux=daux, capacity_factor=cf, logit_bias=bias)
    idx = O.top_k(L.astype(np.float32), k)
    disp = O.dispatch(idx, E, cf)
    f = disp["f"].astype(np.float64)
    params = dict(x=x, W=W, bias=bias, **{key: v for key, v in weights.items() if v is not None})
    want = dict(x="dx", W="dW_router", bias="dbias", W_in="dW_in", W_up="dW_up", W_out="dW_out")
    hstep = 1e-6
    for name, a in params.items():
        num = np.zeros_like(a)
        for i in np.ndindex(a.shape):
            vals = []
            for sgn in (1, -1):
                p = {key: v.copy() for key, v in params.items()}
                p[name][i] += sgn * hstep
                wts = {key: p.get(key) for key in ("W_in", "W_up", "W_out")}
                vals.append(_layer_loss(p["x"], p["W"], p["bias"], wts, kind, idx, disp, dy, f,
                                        daux))
            num[i] = (vals[0] - vals[1]) / (2 * hstep)
        # the oracle's forward decides on fp32 logits and fp32 gates: ~1e-7 relative
        assert np.allclose(got[want[name]], num, rtol=2e-5, atol=2e-6), (kind, cf, name)
