"""Work accounting of the MoE forward pass: FLOPs, parameters, bytes.

Host-side arithmetic used by the benchmark's roofline figures.  The FLOP and
parameter formulas reproduce the counts printed in "Mixture of Experts: the
Sparsely-Gated Layer" (paperfordummies.in), section "Eight times the
parameters, twice the compute": a router of d*N multiply-adds plus k experts
of two d*h matrices (two FLOPs per multiply-add), and SwiGLU experts of
three d*h matrices.  Only work the method must do is counted: experts that
receive no token are not, padding never is.
"""
from __future__ import annotations

MATRICES = {"linear": 1, "relu": 2, "swiglu": 3}


def router_mlp_flops_per_token(d: int, h: int, n_experts: int, k: int) -> int:
    """2*d*N for the router plus k ReLU-MLP experts of 2 matrices (d x h)."""
    return 2 * d * n_experts + k * 2 * (2 * d * h)


def dense_ffn_params(d: int, h: int) -> int:
    return 2 * d * h


def moe_params(d: int, h: int, n_experts: int) -> int:
    """N two-matrix experts plus the d x N router."""
    return n_experts * dense_ffn_params(d, h) + d * n_experts


def swiglu_expert_params(d: int, h: int) -> int:
    return 3 * d * h


def expert_gemm_flops(rows: int, d: int, d_hidden: int, d_out: int, kind: str) -> int:
    """Tensor FLOPs of the expert projections over `rows` kept rows."""
    if kind == "linear":
        return 2 * rows * d * d_out
    if kind == "relu":
        return 2 * rows * (d * d_hidden + d_hidden * d_out)
    if kind == "swiglu":
        return 2 * rows * (2 * d * d_hidden + d_hidden * d_out)
    raise ValueError(kind)


def expert_weight_bytes(used_experts: int, d: int, d_hidden: int, d_out: int, kind: str,
                        elem: int) -> int:
    """Bytes of the weights of the experts that receive at least one row."""
    if kind == "linear":
        per = d * d_out
    elif kind == "relu":
        per = d * d_hidden + d_hidden * d_out
    else:
        per = 2 * d * d_hidden + d_hidden * d_out
    return used_experts * per * elem


def capacity_slots(capacity_factor: float, T: int, k: int, E: int):
    """ceil(((cf * T) * k) / E) slots per expert, or None without a limit."""
    import math
    cf = float(capacity_factor)
    return None if cf <= 0 else int(math.ceil(((cf * T) * k) / E))


def kept_rows(counts, capacity_factor: float, T: int, k: int) -> int:
    """Rows the experts process: per expert min(count, capacity), summed."""
    cap = capacity_slots(capacity_factor, T, k, len(counts))
    return int(sum(c if cap is None else min(int(c), cap) for c in counts))


def router_bytes(T: int, d: int, E: int, k: int, elem: int, noise: bool) -> int:
    """x read once, W_router read once, indices and gates written."""
    return T * d * elem + d * E * 4 + (T * E * 4 if noise else 0) + T * k * 8


def router_flops(T: int, d: int, E: int) -> int:
    return 2 * T * d * E


def permute_bytes(T: int, rows: int, d: int, elem: int) -> int:
    """x read once, each kept row written once."""
    return T * d * elem + rows * d * elem


def combine_bytes(T: int, rows: int, d_out: int, k: int, out_elem: int, row_elem: int = 4) -> int:
    """Each kept expert-output row (fp32) read once, dest+gates read, y written."""
    return rows * d_out * row_elem + T * k * 8 + T * d_out * out_elem


def gemm_roofline_seconds(flops: float, weight_bytes: float, act_bytes: float,
                          tflops: float, hbm_gbs: float) -> float:
    """max(tensor time, HBM time) for the expert projections."""
    return max(flops / (tflops * 1e12), (weight_bytes + act_bytes) / (hbm_gbs * 1e9))
