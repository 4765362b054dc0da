"""The work accounting used by the benchmark reproduces the pages' counts.

"Mixture of Experts: the Sparsely-Gated Layer" (paperfordummies.in), section
"Eight times the parameters, twice the compute": FLOPs per token for k = 1,
2, 4, 8 and parameter counts for d=1024, h=4096, N=8, and the Mixtral 8x7B
expert-weight counts.
"""
import json
import os

from mixture_experts_top_b200 import accounting as A


def test_pfd_flops_and_params(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pfd_accounting.json")))["relu_mlp"]
    d, h, N = g["d_model"], g["ffn_hidden"], g["experts"]
    assert A.dense_ffn_params(d, h) == g["dense_ffn_params"]
    assert A.moe_params(d, h, N) == g["moe_params"]
    for k, flops in g["flops_per_token"].items():
        assert A.router_mlp_flops_per_token(d, h, N, int(k)) == flops
    # The expert part alone matches the GEMM count used for the roofline.
    assert A.expert_gemm_flops(1, d, h, d, "relu") * 2 + 2 * d * N == g["flops_per_token"]["2"]


def test_pfd_mixtral_expert_params(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pfd_accounting.json")))["mixtral"]
    one = A.swiglu_expert_params(g["d_model"], g["ffn_hidden"])
    assert one == g["one_expert_params"]
    assert one * g["experts"] * g["layers"] == g["all_expert_params"]
    assert one * g["top_k"] * g["layers"] == g["active_expert_params"]
    # bytes of one layer's bf16 expert weights (all 8 used)
    assert A.expert_weight_bytes(8, 4096, 14336, 4096, "swiglu", 2) == 8 * one * 2


def test_kept_rows_apply_the_capacity():
    """The capacity table of 'Switch: top-1, one loss, and a rate limit':
    64 tokens, 8 experts, top-1, counts 12,6,1,10,8,11,14,2 -> 15/7/0 dropped."""
    counts = [12, 6, 1, 10, 8, 11, 14, 2]
    for cf, dropped in ((1.0, 15), (1.25, 7), (2.0, 0)):
        assert A.kept_rows(counts, cf, 64, 1) == 64 - dropped
    assert A.kept_rows(counts, 0.0, 64, 1) == 64
