"""The permute fused into the experts' first projection
(moe_expert_ffn_gather): grouped row r is read as x[perm_token[r]] by TMA row
gathers instead of from a materialised x_perm.

The GEMM sees the same operand bytes either way, so its rows must be
bit-identical to moe_expert_ffn on x_perm = x[perm_token] (itself checked
against the oracle in test_gpu_experts.py), on the single-CTA and the
CTA-pair kernels, ragged groups included; one case is also checked against
the oracle directly.  moe_dispatch without x_perm must produce the same
routing tensors as with it.
"""
import numpy as np
import pytest
import torch

from gpu_util import REL_F32, RMS_BF16, dev, host
from mixture_experts_top_b200 import api
from oracle import moe_oracle as O
from workloads import WORKLOADS, Workload, make_expert_weights, make_inputs
from workloads.generate import f32_to_bf16_bits

pytestmark = pytest.mark.gpu


def make_case(kind, dtype, T, k, d, h, d_out, sizes, seed):
    E = len(sizes)
    R = int(sum(sizes))
    assert R <= T * k
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    rng = np.random.default_rng(seed)
    xf = rng.standard_normal((T, d)).astype(np.float32)
    x = f32_to_bf16_bits(xf) if dtype == "bf16" else xf
    perm = np.full(T * k, -99, np.int32)                  # beyond R: never read
    perm[:R] = rng.integers(0, T, size=R)
    w = Workload("g", T=T, d=d, d_hidden=h, d_out=d_out, E=E, top_k=k, kind=kind, dtype=dtype,
                 capacity_factor=0)
    per = [make_expert_weights(w, seed, e) for e in range(E)]
    weights = {}
    for i, key in enumerate(("W_in", "W_up", "W_out")):
        weights[key] = None if per[0][i] is None else np.stack([p[i] for p in per])
    cfg = api.make_config(T, d, h, d_out, E, k, kind, dtype)
    return cfg, x, perm, offsets, weights


def run_both(cfg, x, perm, offsets, weights):
    R_max = cfg.T * cfg.top_k
    ws = api.alloc_workspace(cfg)
    W = [dev(weights[key]) for key in ("W_in", "W_up", "W_out")]
    offs = dev(offsets)
    R = int(offsets[-1])
    x_perm = np.zeros((R_max,) + x.shape[1:], x.dtype)
    x_perm[:R] = x[perm[:R]]
    y0 = torch.full((R_max, cfg.d_out), float("nan"), dtype=torch.float32, device="cuda")
    y1 = torch.full((R_max, cfg.d_out), float("nan"), dtype=torch.float32, device="cuda")
    api.moe_expert_ffn(cfg, dev(x_perm), offs, *W, y0, ws)
    api.moe_expert_ffn_gather(cfg, dev(x), dev(perm), offs, *W, y1, ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 0
    return host(y0), host(y1), x_perm


CASES = [
    # kind, T, k, d, h, d_out, group sizes, CTA pairs (T k >= 1024 E) or single CTAs
    ("relu", 300, 2, 256, 512, 256, [0, 1, 127, 128, 129, 5, 0, 200], False),
    ("swiglu", 300, 2, 200, 384, 192, [0, 1, 127, 128, 129, 5, 0, 200], False),
    ("swiglu", 700, 6, 512, 704, 512, [330, 7, 1200, 0, 96, 260, 513, 40, 10, 999], False),
    ("relu", 1100, 2, 256, 384, 200, [1500, 700], True),
    ("swiglu", 2100, 2, 200, 256, 256, [0, 1, 2049, 2050], True),
    ("swiglu", 4096, 1, 512, 1024, 512, [4096], True),
]


@pytest.mark.parametrize("kind,T,k,d,h,d_out,sizes,pair", CASES)
def test_gather_is_bit_identical_to_grouped_rows(kind, T, k, d, h, d_out, sizes, pair):
    cfg, x, perm, offsets, weights = make_case(kind, "bf16", T, k, d, h, d_out, sizes,
                                               seed=T + d + len(sizes))
    assert pair == (cfg.T * cfg.top_k >= 1024 * cfg.E)
    y0, y1, _ = run_both(cfg, x, perm, offsets, weights)
    R = int(offsets[-1])
    assert np.array_equal(y0[:R], y1[:R])
    assert np.isnan(y1[R:]).all()                        # rows beyond offsets[E] untouched


def test_gather_against_oracle():
    cfg, x, perm, offsets, weights = make_case("swiglu", "bf16", 2100, 2, 200, 256, 256,
                                               [0, 1, 2049, 2050], seed=7)
    _, y1, x_perm = run_both(cfg, x, perm, offsets, weights)
    R = int(offsets[-1])
    xf = O.widen(x_perm, "bf16")
    ref = np.concatenate([O.expert_forward("swiglu", xf[offsets[e]:offsets[e + 1]],
                                           *O.expert_weights(weights, e, "bf16"))
                          for e in range(len(offsets) - 1) if offsets[e + 1] > offsets[e]])
    rms = float(np.sqrt(np.mean(ref ** 2)))
    assert np.abs(y1[:R].astype(np.float64) - ref).max() <= RMS_BF16 * rms


def test_gather_linear_fp32():
    cfg, x, perm, offsets, weights = make_case("linear", "f32", 64, 2, 32, 0, 32,
                                               [0, 3, 60, 1, 64], seed=9)
    y0, y1, x_perm = run_both(cfg, x, perm, offsets, weights)
    R = int(offsets[-1])
    assert np.array_equal(y0[:R], y1[:R])
    ref = np.concatenate([O.expert_forward("linear", x_perm[offsets[e]:offsets[e + 1]].astype(np.float64),
                                           weights["W_in"][e].astype(np.float64), None, None)
                          for e in range(len(offsets) - 1) if offsets[e + 1] > offsets[e]])
    assert np.abs(y1[:R] - ref).max() <= REL_F32 * np.abs(ref).max()


@pytest.mark.parametrize("kind,dtype", [("swiglu", "bf16"), ("linear", "f32")])
def test_gather_reports_bad_row_index(kind, dtype):
    """An index outside [0, T) is recorded (code 3), never used to address x."""
    cfg, x, perm, offsets, weights = make_case(kind, dtype, 100, 2, 64, 128 if kind != "linear"
                                               else 0, 64, [50, 60], seed=4)
    perm[7] = 100                                        # == T
    perm[70] = -1
    ws = api.alloc_workspace(cfg)
    y = torch.zeros((200, 64), dtype=torch.float32, device="cuda")
    api.moe_expert_ffn_gather(cfg, dev(x), dev(perm), dev(offsets), dev(weights["W_in"]),
                              dev(weights["W_up"]), dev(weights["W_out"]), y, ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 3


def test_dispatch_without_x_perm_gives_the_same_routing():
    w = WORKLOADS["fine_grained"].replace(T=1100, d=256, d_hidden=352, d_out=256)
    inp = make_inputs(w, seed=2, with_experts=False)
    cfg = api.make_config(w.T, w.d, w.d_hidden, w.d_out, w.E, w.top_k, w.kind, w.dtype,
                          w.capacity_factor)
    T, k, E = w.T, w.top_k, w.E
    ws = api.alloc_workspace(cfg)
    x = dev(inp["x"])
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    g = torch.empty((T, k), dtype=torch.float32, device="cuda")
    P = torch.empty(E, dtype=torch.float32, device="cuda")
    api.moe_route(cfg, x, dev(inp["W_router"]), dev(inp["logit_bias"]), None, idx, g, P, None, ws)
    outs = []
    for with_rows in (True, False):
        t = dict(counts=torch.empty(E, dtype=torch.int32, device="cuda"),
                 offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"),
                 dest=torch.empty((T, k), dtype=torch.int32, device="cuda"),
                 perm=torch.full((T * k,), -5, dtype=torch.int32, device="cuda"),
                 drop=torch.empty((T, k), dtype=torch.uint8, device="cuda"),
                 f=torch.empty(E, dtype=torch.float32, device="cuda"),
                 aux=torch.empty(1, dtype=torch.float32, device="cuda"))
        xp = torch.empty((T * k, w.d), dtype=torch.bfloat16, device="cuda") if with_rows else None
        api.moe_dispatch(cfg, x, idx, P, t["counts"], t["offsets"], t["dest"], t["perm"],
                         t["drop"], t["f"], t["aux"], xp, ws)
        torch.cuda.synchronize()
        outs.append({key: host(v) for key, v in t.items()})
    assert api.moe_device_status(ws) == 0
    for key in outs[0]:
        assert np.array_equal(outs[0][key], outs[1][key]), key
