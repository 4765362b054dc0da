"""GPU experts (moe_expert_ffn: tcgen05 grouped GEMMs with fused ReLU or
SwiGLU, and the fp32 linear expert) against the CPU oracle on the same
grouped rows and weights.

Group sizes straddle the 128-row tile (0, 1, 127, 128, 129, ...), and the
widths cover ragged K (not a multiple of the 64-wide k block) and ragged N
(not a multiple of the 256/128-column output tile).
"""
import numpy as np
import pytest
import torch

from gpu_util import REL_F32, RMS_BF16, dev, host
from mixture_experts_top_b200 import api
from oracle import moe_oracle as O
from workloads import Workload, make_expert_weights
from workloads.generate import f32_to_bf16_bits

pytestmark = pytest.mark.gpu


def run_ffn(cfg, x_perm, offsets, W_in, W_up, W_out):
    R_max = cfg.T * cfg.top_k
    ws = api.alloc_workspace(cfg)
    y = torch.full((R_max, cfg.d_out), float("nan"), dtype=torch.float32, device="cuda")
    api.moe_expert_ffn(cfg, dev(x_perm), dev(offsets.astype(np.int32)), dev(W_in), dev(W_up),
                       dev(W_out), y, ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 0
    return host(y)


def make_case(kind, dtype, d, h, d_out, sizes, T_k, seed):
    E = len(sizes)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    assert offsets[-1] <= T_k
    w = Workload("ffn", T=T_k, d=d, d_hidden=h, d_out=d_out, E=E, top_k=1, kind=kind, dtype=dtype,
                 capacity_factor=0)
    rng = np.random.default_rng(seed)
    xf = rng.standard_normal((T_k, d)).astype(np.float32)
    x_perm = f32_to_bf16_bits(xf) if dtype == "bf16" else xf
    per = [make_expert_weights(w, seed, e) for e in range(E)]
    weights = {}
    for i, key in enumerate(("W_in", "W_up", "W_out")):
        weights[key] = None if per[0][i] is None else np.stack([p[i] for p in per])
    cfg = api.make_config(T_k, d, h, d_out, E, 1, kind, dtype)
    return cfg, x_perm, offsets, weights


def oracle_rows(kind, dtype, x_perm, offsets, weights):
    xf = O.widen(x_perm, dtype)
    out = []
    for e in range(len(offsets) - 1):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            out.append(O.expert_forward(kind, xf[lo:hi], *O.expert_weights(weights, e, dtype)))
    return np.concatenate(out) if out else np.zeros((0, 1))


def compare_bf16(y_gpu, ref, offsets):
    """bf16 experts: their fp32 output rows within 2e-2 * RMS of the oracle."""
    R = int(offsets[-1])
    got = y_gpu[:R].astype(np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert err.max() <= RMS_BF16 * rms, (err.max(), rms)
    # per expert as well, so that a small group cannot hide behind a big one
    for e in range(len(offsets) - 1):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            assert err[lo:hi].max() <= RMS_BF16 * rms


SIZES = [0, 1, 127, 128, 129, 300, 5, 0, 256]


@pytest.mark.parametrize("kind", ["relu", "swiglu"])
@pytest.mark.parametrize("d,h,d_out", [(256, 512, 256), (200, 384, 192), (64, 136, 72),
                                       (768, 3072, 768)])
def test_grouped_ffn_bf16(kind, d, h, d_out):
    sizes = SIZES
    cfg, x_perm, offsets, weights = make_case(kind, "bf16", d, h, d_out, sizes, sum(sizes) + 40,
                                              seed=d + h)
    y = run_ffn(cfg, x_perm, offsets, weights["W_in"], weights["W_up"], weights["W_out"])
    ref = oracle_rows(kind, "bf16", x_perm, offsets, weights)
    compare_bf16(y, ref, offsets)
    # rows beyond offsets[E] are untouched
    R = int(offsets[-1])
    assert np.isnan(y[R:]).all()


def test_grouped_ffn_many_experts_and_tiles():
    """64 experts, skewed ragged groups, several row and column tiles each."""
    rng = np.random.default_rng(12)
    sizes = list(rng.integers(0, 400, size=64))
    sizes[3] = 1536
    cfg, x_perm, offsets, weights = make_case("swiglu", "bf16", 512, 704, 512, sizes,
                                              sum(sizes), seed=3)
    y = run_ffn(cfg, x_perm, offsets, weights["W_in"], weights["W_up"], weights["W_out"])
    compare_bf16(y, oracle_rows("swiglu", "bf16", x_perm, offsets, weights), offsets)


def test_grouped_ffn_single_expert_exact_small_integers():
    """Small-integer inputs and weights make every product and sum exact in
    fp32 and every hidden value exact in bf16, so the fp32 output must equal
    the oracle's exact result bit for bit.  This pins the operand layouts."""
    d, h, d_out, R = 64, 256, 256, 200
    rng = np.random.default_rng(0)
    x = rng.integers(-2, 3, size=(R, d)).astype(np.float32)
    W1 = rng.integers(-1, 2, size=(1, d, h)).astype(np.float32)
    W2 = rng.integers(-1, 2, size=(1, h, d_out)).astype(np.float32) / 8
    cfg = api.make_config(R, d, h, d_out, 1, 1, "relu", "bf16")
    bits = lambda a: f32_to_bf16_bits(a)
    offsets = np.array([0, R], np.int32)
    y = run_ffn(cfg, bits(x), offsets, bits(W1), None, bits(W2))
    ref = O.expert_forward("relu", x.astype(np.float64), W1[0].astype(np.float64), None,
                           W2[0].astype(np.float64))
    assert np.array_equal(y[:R].astype(np.float64), ref)


def test_linear_expert_fp32():
    sizes = [0, 3, 60, 1, 64]
    cfg, x_perm, offsets, weights = make_case("linear", "f32", 32, 0, 32, sizes, 128, seed=9)
    y = run_ffn(cfg, x_perm, offsets, weights["W_in"], None, None)
    ref = oracle_rows("linear", "f32", x_perm, offsets, weights)
    R = int(offsets[-1])
    assert np.abs(y[:R] - ref).max() <= REL_F32 * np.abs(ref).max()


def test_bad_offsets_are_reported_not_used():
    cfg, x_perm, offsets, weights = make_case("relu", "bf16", 64, 128, 64, [10, 20], 40, seed=1)
    bad = np.array([0, 30, 20], np.int32)            # not monotone
    ws = api.alloc_workspace(cfg)
    y = torch.zeros((40, 64), dtype=torch.float32, device="cuda")
    api.moe_expert_ffn(cfg, dev(x_perm), dev(bad), dev(weights["W_in"]), None,
                       dev(weights["W_out"]), y, ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 2            # kDevBadOffsets
    assert (host(y) == 0).all()


# Groups averaging 1024 rows or more run on CTA pairs (cta_group::2, 256-row
# tiles); these shapes put the pair kernel through ragged groups, 1-row
# groups, and ragged K and N.
PAIR_CASES = [([1500, 700], 2200, 256, 384, 200),
              ([0, 1, 2049, 2050], 4100, 200, 256, 256),
              ([2048], 2048, 512, 1024, 512)]


@pytest.mark.parametrize("kind", ["relu", "swiglu"])
@pytest.mark.parametrize("sizes,T_k,d,h,d_out", PAIR_CASES)
def test_grouped_ffn_bf16_cta_pairs(kind, sizes, T_k, d, h, d_out):
    cfg, x_perm, offsets, weights = make_case(kind, "bf16", d, h, d_out, sizes, T_k, seed=T_k + d)
    assert cfg.T * cfg.top_k >= 1024 * cfg.E
    y = run_ffn(cfg, x_perm, offsets, weights["W_in"], weights["W_up"], weights["W_out"])
    compare_bf16(y, oracle_rows(kind, "bf16", x_perm, offsets, weights), offsets)
    assert np.isnan(y[int(offsets[-1]):]).all()


def test_grouped_ffn_cta_pairs_exact_small_integers():
    """The exact-arithmetic check of the operand layouts, on the pair kernel."""
    d, h, d_out, R = 128, 512, 256, 2100
    rng = np.random.default_rng(1)
    x = rng.integers(-2, 3, size=(R, d)).astype(np.float32)
    W1 = rng.integers(-1, 2, size=(1, d, h)).astype(np.float32)
    W2 = rng.integers(-1, 2, size=(1, h, d_out)).astype(np.float32) / 8
    cfg = api.make_config(R, d, h, d_out, 1, 1, "relu", "bf16")
    offsets = np.array([0, R], np.int32)
    y = run_ffn(cfg, f32_to_bf16_bits(x), offsets, f32_to_bf16_bits(W1), None,
                f32_to_bf16_bits(W2))
    ref = O.expert_forward("relu", x.astype(np.float64), W1[0].astype(np.float64), None,
                           W2[0].astype(np.float64))
    assert np.array_equal(y[:R].astype(np.float64), ref)


def test_cta_pairs_repeat_on_one_workspace_leaves_counters_at_zero():
    """The pair kernel hands tiles out from a counter in the workspace's
    control block; the last CTA of each launch puts it back to 0.  Three
    calls on one workspace (each two launches) give identical bits, and the
    control block's counters read 0 afterwards."""
    cfg, x_perm, offsets, weights = make_case("swiglu", "bf16", 256, 384, 256, [1500, 700], 2200,
                                              seed=9)
    ws = api.alloc_workspace(cfg)
    outs = []
    for _ in range(3):
        y = torch.full((cfg.T, cfg.d_out), float("nan"), dtype=torch.float32, device="cuda")
        api.moe_expert_ffn(cfg, dev(x_perm), dev(offsets), dev(weights["W_in"]),
                           dev(weights["W_up"]), dev(weights["W_out"]), y, ws)
        outs.append(y)
    torch.cuda.synchronize()
    ctrl = host(ws[:256]).view(np.uint32)
    assert api.moe_device_status(ws) == 0
    assert (ctrl[1:] == 0).all(), ctrl[ctrl != 0]
    ys = [host(y) for y in outs]
    assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[0], ys[2])
    compare_bf16(ys[0], oracle_rows("swiglu", "bf16", x_perm, offsets, weights), offsets)
