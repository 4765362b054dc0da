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
