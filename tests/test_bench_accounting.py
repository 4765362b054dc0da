"""bench.py's host-side accounting, on CPU: launches per step and the
experts' algorithmic bytes follow the form moe_forward uses for the experts
and the combine (the library's own host-only query), and the roofline picks
its bound from them."""
import pytest

import bench
from mixture_experts_top_b200 import accounting as A
from workloads import WORKLOADS

PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}


@pytest.mark.parametrize("name,fused,launches", [
    ("mixtral", True, 6),        # split, router, count, scatter, up, down (+ top-2 combine)
    ("decode", False, 7),        # ... + the combine kernel
    ("fine_grained", False, 7),
    ("switch_relu", True, 6),    # top-1 combine in the down projection
    ("tiny_linear", False, 6),   # one fp32 linear-expert launch + the combine kernel
])
def test_launches_follow_the_combine_form(name, fused, launches):
    w = WORKLOADS[name]
    assert bench.fused_combine(w) is fused
    assert bench.launches_per_step(w, None) == launches


def test_gemm_bytes_count_the_combine_output_where_fused():
    w = WORKLOADS["mixtral"]
    rows, used = w.T * w.top_k, w.E
    g = bench.gemm_roofline(w, rows, used, 4.0, PEAKS, "fallback", "burst")
    weights = A.expert_weight_bytes(used, w.d, w.d_hidden, w.d_out, w.kind, 2)
    expect = (weights + rows * w.d * 2 + 2 * rows * w.d_hidden * 2
              + rows * w.d_out * 4 + w.T * w.d_out * 2)
    assert g["algorithmic_bytes"] == expect
    assert g["bound"] == "tensor"
    assert g["frac"] == pytest.approx(g["achieved"] / 1590.0)


def test_gemm_bytes_without_the_fused_combine():
    w = WORKLOADS["decode"]
    rows, used = w.T * w.top_k, w.E
    g = bench.gemm_roofline(w, rows, used, 0.45, PEAKS, "fallback", "burst")
    weights = A.expert_weight_bytes(used, w.d, w.d_hidden, w.d_out, w.kind, 2)
    expect = weights + rows * w.d * 2 + 2 * rows * w.d_hidden * 2 + rows * w.d_out * 4
    assert g["algorithmic_bytes"] == expect
    assert g["bound"] == "hbm"             # decode streams its weights


def test_top1_fused_writes_only_the_output():
    w = WORKLOADS["switch_relu"]
    rows, used = 4000, w.E
    g = bench.gemm_roofline(w, rows, used, 0.12, PEAKS, "fallback", "burst")
    weights = A.expert_weight_bytes(used, w.d, w.d_hidden, w.d_out, w.kind, 2)
    expect = weights + rows * w.d * 2 + 2 * rows * w.d_hidden * 2 + w.T * w.d_out * 2
    assert g["algorithmic_bytes"] == expect
