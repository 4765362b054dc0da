"""CPU oracle for the forward pass of a sparsely-gated Mixture-of-Experts layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code with
the CUDA library; both sides receive the same seeded input arrays from the
``workloads`` package and nothing else.

It is plain, slow and written to be checked by eye against the pages.  All
floating-point work is fp64 unless a step says otherwise; the router logits are
rounded to fp32 because the top-k decision is taken on fp32 logits on both
sides.  Pages cited (title, then section):

* [MLG] "Mixture-of-Experts Routing - LLM Internals" (mlgrind.dev):
  "Algorithm" steps 1-4, "Inputs", "Expected Return Format",
  "Edge cases and conventions", "Follow-up" (capacity).
* [PFD] "Mixture of Experts: the Sparsely-Gated Layer" (paperfordummies.in):
  "The one formula" (pipeline table), "The code" (``router``,
  ``moe_forward``, ``switch_balance_loss``), "Switch: top-1, one loss, and a
  rate limit" (capacity, first come first served, dropped tokens give 0).
* [EB] "Sparsely-gated Mixture of Experts (MoE)" (Eli Bendersky's website):
  "A Minimal Numpy Implementation" (ReLU feed-forward expert, Wh/Wo).
* Philox4x64-10: Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as
  easy as 1, 2, 3" (SC 2011), for the noisy gate's draws.

Readings taken where the pages are silent or disagree are listed in the
repository's design notes; the ones that shape code are repeated at the step.

Parity pins: every function here is pinned by ``tests/test_oracle_*.py``
against printed values of the pages, closed forms, invariants and an
independent brute-force formulation.  No function is parity-unpinned.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

KINDS = ("linear", "relu", "swiglu")


# ----------------------------------------------------------------------------
# noisy gating drawn from a counter-based generator
# ----------------------------------------------------------------------------
# [PFD The code, `router`] adds noise to the logits; the noisy top-k gate it
# names draws, per token and expert, a standard normal scaled by
# softplus(x @ W_noise).  The draw comes from Philox4x64-10 (Salmon, Moraes,
# Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011),
# implemented here from that definition with Python integers, and two of its
# words become one normal by the Box-Muller transform.

PHILOX_M = (0xD2E7470EE14C6C93, 0xCA5A826395121157)   # round multipliers, 4x64
PHILOX_W = (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)   # key increments (Weyl)
_U64 = (1 << 64) - 1


def philox4x64(counter, key, rounds: int = 10):
    """Philox4x64-`rounds` of a 4-word counter under a 2-word key."""
    x0, x1, x2, x3 = (int(v) & _U64 for v in counter)
    k0, k1 = (int(v) & _U64 for v in key)
    for r in range(rounds):
        if r > 0:
            k0 = (k0 + PHILOX_W[0]) & _U64
            k1 = (k1 + PHILOX_W[1]) & _U64
        p0 = PHILOX_M[0] * x0
        p1 = PHILOX_M[1] * x2
        x0, x1, x2, x3 = ((p1 >> 64) ^ x1 ^ k0, p1 & _U64, (p0 >> 64) ^ x3 ^ k1, p0 & _U64)
    return x0, x1, x2, x3


def gate_normal(seed: int, offset: int, t: int, e: int) -> float:
    """The standard normal of token t (its index in the whole batch) and
    expert e: Philox4x64-10 of the counter (t, e, offset, 0) under the key
    (seed, 0); its first two words w0, w1 give u = ((w >> 11) + 1/2) / 2^53
    in (0, 1), and z = sqrt(-2 ln u0) cos(2 pi u1), in fp64."""
    w = philox4x64((t, e, offset, 0), (seed, 0))
    u0 = ((w[0] >> 11) + 0.5) * 2.0 ** -53
    u1 = ((w[1] >> 11) + 0.5) * 2.0 ** -53
    return math.sqrt(-2.0 * math.log(u0)) * math.cos(2.0 * math.pi * u1)


def softplus(v: np.ndarray) -> np.ndarray:
    """log(1 + exp(v)), written as max(v, 0) + log1p(exp(-|v|)) (no overflow)."""
    v = np.asarray(v, np.float64)
    return np.maximum(v, 0.0) + np.log1p(np.exp(-np.abs(v)))


def gate_noise(x: np.ndarray, W_noise: np.ndarray, dtype: str, seed: int, offset: int,
               token_base: int = 0) -> np.ndarray:
    """(T, E) fp32 noise: z(t, e) * softplus(l_te) with l = x @ W_noise the
    fp32 noise logits (fp64 dot, rounded to fp32 like the router logits) and
    the product rounded to fp32 once.  Token t of this call is token
    token_base + t of the batch."""
    L = (widen(x, dtype) @ np.asarray(W_noise, np.float64)).astype(np.float32).astype(np.float64)
    T, E = L.shape
    z = np.array([[gate_normal(seed, offset, token_base + t, e) for e in range(E)]
                  for t in range(T)], np.float64).reshape(T, E)
    return (z * softplus(L)).astype(np.float32)


# ----------------------------------------------------------------------------
# dtype helpers (the oracle's own; it does not use the generator's helpers)
# ----------------------------------------------------------------------------

def widen(a: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array -> fp64.  bf16 arrives as uint16 bit patterns."""
    if dtype == "bf16":
        a = np.asarray(a, dtype=np.uint16)
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if dtype == "f64":
        return np.asarray(a, dtype=np.float64)
    return np.asarray(a, dtype=np.float32).astype(np.float64)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round fp64 straight to bf16 (nearest, ties to even), one rounding.

    Magnitudes below the smallest normal bf16 (about 1.2e-38) become signed
    zero; the layer's outputs never come near that range or near overflow.
    """
    v = np.ascontiguousarray(v, dtype=np.float64)
    u = v.view(np.uint64)
    sign = (u >> np.uint64(63)) & np.uint64(1)
    mag = u & np.uint64(0x7FFFFFFFFFFFFFFF)
    lsb = (mag >> np.uint64(45)) & np.uint64(1)
    r = (mag + np.uint64((1 << 44) - 1) + lsb) >> np.uint64(45)   # 11-bit exp, 7-bit mantissa
    exp = (r >> np.uint64(7)).astype(np.int64) - 1023 + 127
    mant = (r & np.uint64(0x7F)).astype(np.int64)
    bits = (exp << 7) | mant
    bits = np.where((mag == 0) | (exp <= 0), 0, bits)
    bits = bits | (sign.astype(np.int64) << 15)
    return bits.astype(np.uint16)


def round_output(y: np.ndarray, dtype: str) -> np.ndarray:
    """The layer output in its storage dtype (the activation dtype)."""
    if dtype == "bf16":
        return f64_to_bf16_bits(y)
    return np.asarray(y, dtype=np.float64).astype(np.float32)


# ----------------------------------------------------------------------------
# Router: logits, softmax, top-k, renormalised gates
# ----------------------------------------------------------------------------

def router_logits(x: np.ndarray, W_router: np.ndarray, dtype: str,
                  logit_bias: Optional[np.ndarray] = None,
                  noise: Optional[np.ndarray] = None) -> np.ndarray:
    """L = x @ W_router (+ bias) (+ noise), fp32.

    [MLG Algorithm 1] logits = x @ W_router.  [PFD The code, ``router``]
    adds the optional per-expert bias first and the noise second.  The dot
    product is summed in fp64 and rounded once to fp32; the bias and the noise
    are then each added in fp32, in that order.
    """
    xf = widen(x, dtype)
    L = (xf @ np.asarray(W_router, dtype=np.float64)).astype(np.float32)
    if logit_bias is not None:
        L = (L + np.asarray(logit_bias, dtype=np.float32)[None, :]).astype(np.float32)
    if noise is not None:
        L = (L + np.asarray(noise, dtype=np.float32)).astype(np.float32)
    return L


def softmax_rows(L: np.ndarray) -> np.ndarray:
    """Row softmax of the fp32 logits, in fp64, max subtracted first.

    [MLG Algorithm 1] probs = softmax(logits, axis=-1).
    """
    z = np.asarray(L, dtype=np.float64)
    z = z - z.max(axis=1, keepdims=True)
    ez = np.exp(z)
    return ez / ez.sum(axis=1, keepdims=True)


def top_k(L: np.ndarray, k: int) -> np.ndarray:
    """The k experts with the largest fp32 logits, by descending logit.

    [MLG Algorithm 2] sorted by descending logit; [MLG Edge cases] a stable
    sort of -logits: among equal logits the lower expert index comes first.
    Negation is exact in fp32 and -0 == +0 compares equal, so a stable
    ascending sort of -L realises exactly that order.
    """
    L = np.asarray(L, dtype=np.float32)
    if not 1 <= k <= L.shape[1]:
        raise ValueError("top_k must satisfy 1 <= top_k <= E")
    order = np.argsort(-L, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def renormalised_gates(L: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """gates[t, j] = softmax over the chosen k logits of token t, as fp32.

    [MLG Algorithm 2] gates = softmax(top-k logits), renormalised over the
    chosen k only.  Computed in fp64 as exp(L_j - L_0) / sum_i exp(L_i - L_0),
    L_0 being the largest chosen logit, then rounded to fp32.
    """
    Lk = np.take_along_axis(np.asarray(L, dtype=np.float64), idx.astype(np.int64), axis=1)
    ez = np.exp(Lk - Lk[:, :1])
    return (ez / ez.sum(axis=1, keepdims=True)).astype(np.float32)


def prob_mean(probs: np.ndarray) -> np.ndarray:
    """P_e = mean over tokens of probs[:, e], fp64.  [MLG Algorithm 4]."""
    return np.asarray(probs, dtype=np.float64).mean(axis=0)


# ----------------------------------------------------------------------------
# Dispatch: histogram, positions, capacity, offsets, permutation
# ----------------------------------------------------------------------------

def capacity(capacity_factor: float, T: int, k: int, E: int) -> Optional[int]:
    """Slots per expert, ceil(cf * T * k / E); None when cf <= 0 (no limit).

    [MLG Follow-up] capacity_factor * T * k / E slots; rounded up.  The
    product is formed in fp64 as ((cf * T) * k) / E with cf taken as the fp32
    value the caller passes.
    """
    cf = float(np.float32(capacity_factor))
    if cf <= 0.0:
        return None
    return int(math.ceil(((cf * float(T)) * float(k)) / float(E)))


def dispatch(idx: np.ndarray, E: int, capacity_factor: float) -> dict:
    """Group routing slots by expert in token order and apply the capacity.

    [MLG Algorithm 3] gather the tokens routed to each expert;
    [PFD The code, ``moe_forward``] tokens routed to expert i in token order,
    truncated to the capacity, first come first served, overflow dropped.

    Slots are visited in token order t = 0..T-1 and, within a token, in rank
    order j = 0..k-1 (a token never picks an expert twice, so the within-token
    order cannot change a decision).  A slot's position p is the number of
    earlier slots on the same expert; it is kept iff p < cap.

    Returns counts (routed, before drops), kept, offsets (exclusive scan of
    kept, E+1 entries), dest (T, k) row in the grouped layout or -1,
    perm_token (R,) token of each grouped row, drop_mask (T, k) uint8,
    f (E,) fp64 routing-slot fractions and cap.
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    cap = capacity(capacity_factor, T, k, E)
    counts = np.zeros(E, dtype=np.int64)
    pos = np.zeros((T, k), dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            pos[t, j] = counts[e]
            counts[e] += 1
    kept = counts.copy() if cap is None else np.minimum(counts, cap)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    dest = np.full((T, k), -1, dtype=np.int64)
    perm_token = np.full(int(offsets[-1]), -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            if cap is None or pos[t, j] < cap:
                dest[t, j] = offsets[e] + pos[t, j]
                perm_token[dest[t, j]] = t
    f = counts.astype(np.float64) / float(T * k)
    return dict(counts=counts.astype(np.int32), kept=kept.astype(np.int32),
                offsets=offsets.astype(np.int32), dest=dest.astype(np.int32),
                perm_token=perm_token.astype(np.int32),
                drop_mask=(dest < 0).astype(np.uint8), f=f, cap=cap)


def aux_loss(f: np.ndarray, P: np.ndarray) -> float:
    """Switch load-balancing loss E * sum_e f_e * P_e.  [MLG Algorithm 4].

    f counts routing slots before any capacity drop.
    """
    f = np.asarray(f, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    return float(len(f) * np.sum(f * P))


# ----------------------------------------------------------------------------
# Experts and combine
# ----------------------------------------------------------------------------

def silu(z: np.ndarray) -> np.ndarray:
    """z * sigmoid(z) = z / (1 + exp(-z)), fp64."""
    return z / (1.0 + np.exp(-z))


def expert_forward(kind: str, xe: np.ndarray, W_in: np.ndarray,
                   W_up: Optional[np.ndarray], W_out: Optional[np.ndarray]) -> np.ndarray:
    """One expert on the rows routed to it, fp64, no intermediate rounding.

    * linear: x @ W  [MLG Background, Inputs: expert_e(x) = x @ W_e]
    * relu:   relu(x @ W1) @ W2  [PFD The code, ``expert_forward``;
      EB A Minimal Numpy Implementation, ``feed_forward_relu``(Wh, Wo)]
    * swiglu: (silu(x @ W_gate) * (x @ W_up)) @ W_down.  The pages only name
      SwiGLU experts with three matrices each [MLG Background; PFD Eight
      times the parameters]; this is the plainest reading of those words.
    """
    if kind == "linear":
        return xe @ W_in
    if kind == "relu":
        return np.maximum(xe @ W_in, 0.0) @ W_out
    if kind == "swiglu":
        return (silu(xe @ W_in) * (xe @ W_up)) @ W_out
    raise ValueError(f"unknown expert kind {kind!r}")


def expert_weights(weights: dict, e: int, dtype: str):
    """Expert e's (W_in, W_up, W_out) widened to fp64 (None stays None)."""
    out = []
    for key in ("W_in", "W_up", "W_out"):
        w = weights.get(key)
        out.append(None if w is None else widen(w[e], dtype))
    return tuple(out)


def run_experts(kind: str, x: np.ndarray, dtype: str, disp: dict, weights: dict,
                d_out: int) -> np.ndarray:
    """Y (R, d_out) fp64: each expert run only on its kept rows, in grouped order.

    [MLG Constraints] run each expert on its routed tokens, never on all.
    """
    xf = widen(x, dtype)
    offsets, perm = disp["offsets"], disp["perm_token"]
    E = len(offsets) - 1
    Y = np.zeros((int(offsets[-1]), d_out), dtype=np.float64)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue                       # idle expert: no work [PFD The code]
        Y[lo:hi] = expert_forward(kind, xf[perm[lo:hi]], *expert_weights(weights, e, dtype))
    return Y


def combine(Y: np.ndarray, dest: np.ndarray, gates: np.ndarray) -> np.ndarray:
    """y_t = sum_j gates[t, j] * Y[dest[t, j]] over kept slots, fp64.

    [MLG Algorithm 3] y_t = sum_j gates[t,j] * expert_{idx[t,j]}(x_t);
    [PFD Switch] a dropped slot contributes 0 and the remaining gates are not
    renormalised, so a token whose every slot was dropped outputs 0.
    """
    Y = np.asarray(Y, dtype=np.float64)
    T, k = dest.shape
    y = np.zeros((T, Y.shape[1]), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            r = int(dest[t, j])
            if r >= 0:
                y[t] += float(gates[t, j]) * Y[r]
    return y


# ----------------------------------------------------------------------------
# Backward of the routing half (gradients of the combine and of the router)
# ----------------------------------------------------------------------------
# The pages train the layer but print no backward; these are the derivatives
# of the forward above, in fp64, pinned by finite differences of it.
# [MLG Algorithm 2-4; PFD The code, `switch_balance_loss`: f is a count and
# carries no gradient, P does]

def combine_backward(Y: np.ndarray, dest: np.ndarray, gates: np.ndarray, dy: np.ndarray):
    """Gradients of y_t = sum over kept j of gates[t,j] * Y[dest[t,j]].

    Returns dY (rows of Y; a row gets gates[t,j] * dy_t from its slot) and
    dgates[t, j] = <dy_t, Y[dest[t,j]]> (0 for a dropped slot)."""
    Y = np.asarray(Y, np.float64)
    dy = np.asarray(dy, np.float64)
    T, k = dest.shape
    dY = np.zeros_like(Y)
    dg = np.zeros((T, k), np.float64)
    for t in range(T):
        for j in range(k):
            r = int(dest[t, j])
            if r >= 0:
                dY[r] += float(gates[t, j]) * dy[t]
                dg[t, j] = float(dy[t] @ Y[r])
    return dY, dg


def expert_backward(kind: str, xe: np.ndarray, W_in: np.ndarray, W_up: Optional[np.ndarray],
                    W_out: Optional[np.ndarray], dY: np.ndarray) -> dict:
    """Gradients of one expert (expert_forward) on its rows, fp64.

    With A = x W_in (and B = x W_up for SwiGLU), H the hidden activation and
    dH = dY W_out^T:
    * linear: dx = dY W_in^T, dW_in = x^T dY
    * relu:   dA = dH * [A > 0]
    * swiglu: H = silu(A) * B; dA = dH * B * silu'(A), dB = dH * silu(A),
              silu'(a) = s (1 + a (1 - s)) with s = sigmoid(a)
    then dW_out = H^T dY, dW_in = x^T dA, dW_up = x^T dB, dx = dA W_in^T
    (+ dB W_up^T).  Returns dict(dx, dW_in, dW_up, dW_out)."""
    xe = np.asarray(xe, np.float64)
    dY = np.asarray(dY, np.float64)
    if kind == "linear":
        return dict(dx=dY @ W_in.T, dW_in=xe.T @ dY, dW_up=None, dW_out=None)
    A = xe @ W_in
    if kind == "relu":
        H = np.maximum(A, 0.0)
        dH = dY @ W_out.T
        dA = dH * (A > 0.0)
        return dict(dx=dA @ W_in.T, dW_in=xe.T @ dA, dW_up=None, dW_out=H.T @ dY)
    if kind == "swiglu":
        B = xe @ W_up
        sg = 1.0 / (1.0 + np.exp(-A))
        H = A * sg * B
        dH = dY @ W_out.T
        dA = dH * B * (sg * (1.0 + A * (1.0 - sg)))
        dB = dH * (A * sg)
        return dict(dx=dA @ W_in.T + dB @ W_up.T, dW_in=xe.T @ dA, dW_up=xe.T @ dB,
                    dW_out=H.T @ dY)
    raise ValueError(f"unknown expert kind {kind!r}")


def moe_backward(x, W_router, weights: dict, *, top_k: int, kind: str, dtype: str,
                 d_out: int, dy: np.ndarray, daux: float, capacity_factor: float = 0.0,
                 logit_bias=None, noise=None) -> dict:
    """The whole layer's backward in fp64, composed of the pieces above: the
    forward (moe_forward), the combine backward into each kept row, each
    expert's backward on its rows, the rows' input gradients added back to
    their tokens (dx_t = sum over kept j of dX[dest[t,j]]), and the router
    backward (gates and aux) added to dx.  Returns dict(dx, dW_router, dbias,
    dW_in, dW_up, dW_out) (weights' gradients stacked over experts)."""
    fw = moe_forward(x, W_router, weights, top_k=top_k, kind=kind, dtype=dtype, d_out=d_out,
                     capacity_factor=capacity_factor, logit_bias=logit_bias, noise=noise)
    dY, dg = combine_backward(fw["Y"], fw["dest"], fw["gates"].astype(np.float64), dy)
    xf = widen(x, dtype)
    T, d = xf.shape
    E = np.asarray(W_router).shape[1]
    dx = np.zeros((T, d), np.float64)
    grads = {key: None for key in ("W_in", "W_up", "W_out")}
    for key in grads:
        if weights.get(key) is not None:
            grads[key] = np.zeros(np.asarray(weights[key]).shape, np.float64)
    offs = fw["offsets"]
    perm = fw["perm_token"]
    for e in range(E):
        lo, hi = int(offs[e]), int(offs[e + 1])
        if hi <= lo:
            continue
        rows = perm[lo:hi]
        g = expert_backward(kind, xf[rows], *expert_weights(weights, e, dtype), dY[lo:hi])
        np.add.at(dx, rows, g["dx"])
        for key, gk in (("W_in", "dW_in"), ("W_up", "dW_up"), ("W_out", "dW_out")):
            if grads[key] is not None:
                grads[key][e] += g[gk]
    r = route_backward(x, W_router, dtype, fw["logits"], fw["expert_indices"],
                       fw["gates"].astype(np.float64), fw["f"], dg, daux)
    dx += r["dx"]
    return dict(dx=dx, dW_router=r["dW"], dbias=r["dbias"], dW_in=grads["W_in"],
                dW_up=grads["W_up"], dW_out=grads["W_out"])


def route_backward(x, W_router, dtype: str, logits, idx, gates, f, dgates, daux: float,
                   T_batch: Optional[int] = None):
    """Gradients of the router's outputs back to its inputs.

    gates (softmax over the chosen k): dL_m += g_m (dg_m - sum_j g_j dg_j)
    for each chosen m; the top-k choice itself has no gradient.  aux =
    E sum_e f_e P_e with P_e the batch mean of softmax(L)[:, e] (T_batch
    tokens, this call's T by default) and f constant: dL_te += p_te (a_e -
    sum_e' p_te' a_e') with a_e = daux E f_e / T_batch.  Then, for L = x @ W
    (+ bias + noise): dx = dL @ W^T, dW = x^T @ dL, dbias = sum_t dL.
    Returns dict(dlogits, dx, dW, dbias), fp64."""
    L = np.asarray(logits, np.float64)
    T, E = L.shape
    p = softmax_rows(L)
    g = np.asarray(gates, np.float64)
    dg = np.asarray(dgates, np.float64)
    dL = np.zeros((T, E), np.float64)
    for t in range(T):
        s = float(g[t] @ dg[t])
        for j in range(idx.shape[1]):
            dL[t, int(idx[t, j])] += g[t, j] * (dg[t, j] - s)
    Tb = T if T_batch is None else T_batch
    a = float(daux) * E * np.asarray(f, np.float64) / Tb
    dL += p * (a[None, :] - (p @ a)[:, None])
    W = np.asarray(W_router, np.float64)
    xf = widen(x, dtype)
    return dict(dlogits=dL, dx=dL @ W.T, dW=xf.T @ dL, dbias=dL.sum(axis=0))


# ----------------------------------------------------------------------------
# The whole layer
# ----------------------------------------------------------------------------

def moe_route(x, W_router, top_k_: int, dtype: str, logit_bias=None, noise=None) -> dict:
    """Router half of the layer: logits, probs, P, expert_indices, gates."""
    L = router_logits(x, W_router, dtype, logit_bias, noise)
    probs = softmax_rows(L)
    idx = top_k(L, top_k_)
    gates = renormalised_gates(L, idx)
    return dict(logits=L, probs=probs, P=prob_mean(probs), expert_indices=idx, gates=gates)


def moe_forward(x, W_router, weights: dict, *, top_k: int, kind: str, dtype: str,
                d_out: int, capacity_factor: float = 0.0, logit_bias=None, noise=None) -> dict:
    """The full forward pass, in the pages' order.

    Returns the [MLG Expected Return Format] dict (output, expert_indices,
    gates, aux_loss) plus the routing and dispatch intermediates.  ``output``
    is fp64 (``round_output`` gives the storage dtype).
    """
    r = moe_route(x, W_router, top_k, dtype, logit_bias, noise)
    E = np.asarray(W_router).shape[1]
    disp = dispatch(r["expert_indices"], E, capacity_factor)
    Y = run_experts(kind, x, dtype, disp, weights, d_out)
    y = combine(Y, disp["dest"], r["gates"])
    out = dict(r)
    out.update(disp)
    out.update(output=y, Y=Y, aux_loss=aux_loss(disp["f"], r["P"]))
    return out


def token_output(t: int, x, dtype: str, kind: str, weights: dict, expert_indices,
                 gates, dest, cache: Optional[dict] = None) -> np.ndarray:
    """Output row of one token, computed on its own (for sampled checks).

    Same definition as ``combine`` restricted to token t: the sum over its kept
    slots of gate times the chosen expert applied to x_t alone.
    """
    xt = widen(np.asarray(x)[t:t + 1], dtype)
    acc = None
    for j in range(expert_indices.shape[1]):
        if int(dest[t, j]) < 0:
            continue
        e = int(expert_indices[t, j])
        if cache is not None and e in cache:
            w = cache[e]
        else:
            w = expert_weights(weights, e, dtype)
            if cache is not None:
                cache[e] = w
        contrib = float(gates[t, j]) * expert_forward(kind, xt, *w)[0]
        acc = contrib if acc is None else acc + contrib
    if acc is None:
        d_out = expert_forward(kind, xt, *expert_weights(weights, int(expert_indices[t, 0]), dtype)).shape[1]
        acc = np.zeros(d_out)
    return acc


def sampled_outputs(tokens, x, dtype: str, kind: str, weights: dict, expert_indices, gates,
                    dest, return_rows: bool = False):
    """Output rows of the listed tokens only (for sampled full-size checks).

    The same definition as ``combine`` restricted to those tokens, evaluated
    expert by expert so that only one expert's weights are widened to fp64 at
    a time: for each expert, its kept slots among the sampled tokens are run
    through it together, then each token adds gate * row over its slots in
    increasing j.  With ``return_rows`` the kept slots' expert output rows
    are returned as well, stacked in (token, j) order.
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    xs = widen(np.asarray(x)[tokens], dtype)
    idx = np.asarray(expert_indices)[tokens]
    dst = np.asarray(dest)[tokens]
    g = np.asarray(gates)[tokens]
    n, k = idx.shape
    rows = {}
    for e in np.unique(idx[dst >= 0]):
        sel = [(i, j) for i in range(n) for j in range(k) if idx[i, j] == e and dst[i, j] >= 0]
        out = expert_forward(kind, xs[[i for i, _ in sel]], *expert_weights(weights, int(e), dtype))
        for r, key in enumerate(sel):
            rows[key] = out[r]
    d_out = next(iter(rows.values())).shape[0] if rows else 0
    y = np.zeros((n, d_out))
    for i in range(n):
        for j in range(k):
            if dst[i, j] >= 0:
                y[i] += float(g[i, j]) * rows[(i, j)]
    if return_rows:
        return y, np.array([rows[key] for key in sorted(rows)])
    return y


def moe_forward_brute_force(x, W_router, weights: dict, *, top_k: int, kind: str, dtype: str,
                            capacity_factor: float = 0.0, logit_bias=None, noise=None) -> dict:
    """Independent dense formulation, for tiny inputs only.

    Runs every expert on every token and masks with a dense (T, E) gate
    matrix -- the approach [MLG Constraints] says not to use for speed, and
    the one the NumPy tutorial's ``moe_forward`` uses.  It re-derives every
    step differently from ``moe_forward``: top-k by a per-row Python sort on
    (-logit, index) keys, gates by softmax-then-renormalise over the full
    probabilities [PFD The one formula: both orders give the same numbers],
    positions by a running one-hot count, drops by comparing that count with
    the capacity, and the loss from a dense routing mask.
    """
    xf = widen(x, dtype)
    L = router_logits(x, W_router, dtype, logit_bias, noise).astype(np.float64)
    T, E = L.shape
    probs = np.exp(L - L.max(axis=1, keepdims=True))
    probs /= probs.sum(axis=1, keepdims=True)
    idx = np.zeros((T, top_k), dtype=np.int32)
    G = np.zeros((T, E))
    for t in range(T):
        chosen = sorted(range(E), key=lambda e: (-float(np.float32(L[t, e])), e))[:top_k]
        idx[t] = chosen
        p = np.array([probs[t, e] for e in chosen])
        for j, e in enumerate(chosen):
            G[t, e] = p[j] / p.sum()
    mask = (G > 0).astype(np.float64)
    mask[np.arange(T)[:, None], idx] = 1.0        # a gate can underflow; the choice stands
    cap = capacity(capacity_factor, T, top_k, E)
    position = np.cumsum(mask, axis=0) - mask      # earlier tokens on the same expert
    keep = mask if cap is None else mask * (position < cap)
    outs =[expert_forward(kind, xf, *expert_weights(weights, e, dtype)) for e in range(E)]
    y = np.zeros_like(outs[0])
    for e in range(E):
        y += (G[:, e] * keep[:, e])[:, None] * outs[e]
    f = mask.sum(axis=0) / float(T * top_k)
    P = probs.mean(axis=0)
    return dict(output=y, expert_indices=idx, gates=np.take_along_axis(G, idx.astype(np.int64), 1),
                aux_loss=float(E * np.dot(f, P)), keep=keep, counts=mask.sum(axis=0).astype(np.int64))
