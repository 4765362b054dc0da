"""Seeded synthetic workloads for the sparsely-gated MoE forward pass.

The five workloads follow the shapes the pages use, from a tutorial-size router
with linear experts up to a Mixtral-shaped SwiGLU layer:

* ``tiny_linear``  - T=64, d=32, E=8, k=2, linear experts x @ W_e, fp32
  ("Mixture-of-Experts Routing - LLM Internals", mlgrind.dev: Inputs).
* ``switch_relu``  - Switch-style top-1 ReLU-MLP layer with noisy gating and a
  capacity factor of 1.25 ("Mixture of Experts: the Sparsely-Gated Layer",
  paperfordummies.in: "The code", "Switch: top-1, one loss, and a rate limit").
* ``mixtral``      - Mixtral-shaped SwiGLU layer, T=8192, D=4096, DH=14336,
  E=8, k=2 (same page, "Eight times the parameters, twice the compute").
* ``fine_grained`` - many small SwiGLU experts, E=64, k=6, capacity factor
  1.0, with a +3.0 logit bias on four hot experts (the bias argument of the
  same page's ``router``).
* ``decode``       - the Mixtral-shaped layer at T=64 tokens.

Every tensor is drawn from its own NumPy ``SeedSequence`` child so that any
one of them (for instance one expert's weights) can be regenerated on its own.
Values are drawn in fp32 and, for bf16 workloads, rounded to bf16 with
round-to-nearest-even.  bf16 tensors are returned as ``uint16`` bit patterns;
the CUDA side receives exactly these bytes and the oracle widens exactly these
bytes, so both see identical inputs.

The noisy-gating noise of ``switch_relu`` is part of the workload recipe: it is
made on the host, z * softplus(x @ W_noise) with z ~ N(0,1), and handed to both
sides as a finished (T, E) fp32 input.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

# Tags that select the SeedSequence child of each tensor.
_TAG_X, _TAG_WR, _TAG_BIAS, _TAG_WNOISE, _TAG_Z = 1, 2, 3, 4, 5
_TAG_W_IN, _TAG_W_UP, _TAG_W_OUT = 10, 11, 12


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    d_hidden: int          # expert hidden width (0 for linear experts)
    d_out: int
    E: int
    top_k: int
    kind: str              # "linear" | "relu" | "swiglu"
    dtype: str             # "f32" | "bf16" (activations and expert weights)
    capacity_factor: float  # <= 0 means no capacity limit
    noise: bool = False
    hot_bias: float = 0.0
    n_hot: int = 0

    def with_tokens(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_linear": Workload("tiny_linear", T=64, d=32, d_hidden=0, d_out=32, E=8, top_k=2,
                            kind="linear", dtype="f32", capacity_factor=0.0),
    "switch_relu": Workload("switch_relu", T=4096, d=768, d_hidden=3072, d_out=768, E=64,
                            top_k=1, kind="relu", dtype="bf16", capacity_factor=1.25,
                            noise=True),
    "mixtral": Workload("mixtral", T=8192, d=4096, d_hidden=14336, d_out=4096, E=8, top_k=2,
                        kind="swiglu", dtype="bf16", capacity_factor=0.0),
    "fine_grained": Workload("fine_grained", T=16384, d=2048, d_hidden=1408, d_out=2048, E=64,
                             top_k=6, kind="swiglu", dtype="bf16", capacity_factor=1.0,
                             hot_bias=3.0, n_hot=4),
    "decode": Workload("decode", T=64, d=4096, d_hidden=14336, d_out=4096, E=8, top_k=2,
                       kind="swiglu", dtype="bf16", capacity_factor=0.0),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return uint16 bits.

    Inputs are finite by construction, so no NaN handling is needed.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to fp32 exactly."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, tag: int, index: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, tag, index]))


def _normal(seed: int, tag: int, shape, scale: float, index: int = 0) -> np.ndarray:
    a = _rng(seed, tag, index).standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    return a


def _to_storage(a: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(a) if dtype == "bf16" else np.ascontiguousarray(a, dtype=np.float32)


def expert_weight_shapes(w: Workload):
    """Shapes of (W_in, W_up, W_out) per expert; None for an absent matrix."""
    if w.kind == "linear":
        return (w.d, w.d_out), None, None
    if w.kind == "relu":
        return (w.d, w.d_hidden), None, (w.d_hidden, w.d_out)
    if w.kind == "swiglu":
        return (w.d, w.d_hidden), (w.d, w.d_hidden), (w.d_hidden, w.d_out)
    raise ValueError(f"unknown expert kind {w.kind!r}")


def make_expert_weights(w: Workload, seed: int, e: int):
    """One expert's (W_in, W_up, W_out) in storage dtype, each ~N(0, 1/fan_in)."""
    out = []
    for tag, shape in zip((_TAG_W_IN, _TAG_W_UP, _TAG_W_OUT), expert_weight_shapes(w)):
        if shape is None:
            out.append(None)
            continue
        out.append(_to_storage(_normal(seed, tag, shape, 1.0 / np.sqrt(shape[0]), index=e), w.dtype))
    return tuple(out)


def make_inputs(w: Workload, seed: int = 0, with_experts: bool = True) -> dict:
    """All inputs of one forward pass of workload ``w``.

    Keys: x (T,d), W_router (d,E) fp32, logit_bias (E,) fp32 or None,
    noise (T,E) fp32 or None and the W_noise (d,E) fp32 it was made with,
    W_in / W_up / W_out (E, in, out) or None.
    Activations and expert weights are uint16 bf16 bits for bf16 workloads,
    fp32 otherwise.
    """
    x = _to_storage(_normal(seed, _TAG_X, (w.T, w.d), 1.0), w.dtype)
    W_router = _normal(seed, _TAG_WR, (w.d, w.E), 1.0 / np.sqrt(w.d))
    bias = None
    if w.n_hot > 0:
        bias = np.zeros(w.E, dtype=np.float32)
        hot = _rng(seed, _TAG_BIAS).choice(w.E, w.n_hot, replace=False)
        bias[hot] = np.float32(w.hot_bias)
    noise = None
    if w.noise:
        # Recipe of the workload: z * softplus(x @ W_noise), made on the host.
        W_noise = _normal(seed, _TAG_WNOISE, (w.d, w.E), 1.0 / np.sqrt(w.d))
        z = _normal(seed, _TAG_Z, (w.T, w.E), 1.0).astype(np.float64)
        xf = bf16_bits_to_f32(x) if w.dtype == "bf16" else x
        s = xf.astype(np.float64) @ W_noise.astype(np.float64)
        softplus = np.logaddexp(0.0, s)
        noise = (z * softplus).astype(np.float32)
    inputs = dict(x=x, W_router=W_router, logit_bias=bias, noise=noise,
                  W_noise=W_noise if w.noise else None,
                  W_in=None, W_up=None, W_out=None)
    if with_experts:
        per = [make_expert_weights(w, seed, e) for e in range(w.E)]
        for i, key in enumerate(("W_in", "W_up", "W_out")):
            if per[0][i] is not None:
                inputs[key] = np.stack([p[i] for p in per])
    return inputs


def make_exact_router_inputs(T: int, d: int, E: int, dtype: str, seed: int = 0,
                             bias: Optional[np.ndarray] = None) -> dict:
    """Router inputs whose logits are exact in fp32 under any summation order.

    x takes integer values in [-2, 2] and W_router multiples of 1/16 in
    [-1/4, 1/4]; every product is a multiple of 1/16 and every partial sum is
    bounded by d/2, so for d <= 2**19 each partial sum needs at most 24
    significant bits and is exact in fp32.  Ties between experts are frequent,
    which exercises the lower-index-wins rule.
    """
    if d > (1 << 19):
        raise ValueError("d too large for exact fp32 logits")
    r = _rng(seed, 100)
    xf = r.integers(-2, 3, size=(T, d)).astype(np.float32)
    Wr = (r.integers(-4, 5, size=(d, E)).astype(np.float32) / np.float32(16.0)).astype(np.float32)
    x = _to_storage(xf, dtype)
    return dict(x=x, W_router=Wr, logit_bias=bias, noise=None)
