"""Helpers for the GPU parity tests: host <-> device marshalling and the
comparison rules.

Tolerances (stated once, used by every GPU test):
* integer and byte outputs (indices, counts, offsets, dest, perm_token, drop
  mask, gathered rows): bit-exact;
* gates, P and aux: within 1e-5 relative;
* fp32 linear-expert output: max |gpu - oracle| <= 1e-4 * max |oracle|;
* bf16 experts' output (the fp32 rows of moe_expert_ffn): max |gpu - oracle|
  <= 2e-2 * RMS(oracle), the oracle in fp64 on the same bf16-rounded inputs;
* layer output of bf16 experts: the combine adds the k expert rows with gates
  summing to 1 and rounds once to bf16, so the expert bound carries over as
  max |gpu - oracle| <= 2e-2 * RMS(oracle expert rows) + one bf16 ulp;
* combine alone (same fp32 expert rows in): the fp32 multiply-add chain is
  within k * 2^-24 * sum |g y| of the exact sum, then one rounding to bf16:
  |gpu - oracle| <= one bf16 ulp + 2 k 2^-24 sum_j |g_j y_j| (fp32 output:
  1e-6 relative + the same chain bound).
Index agreement between the GPU and the oracle on random inputs excludes
tokens whose oracle logits have a gap below 1e-5 between any two
consecutive positions of the first k+1 in sorted order.
"""
import numpy as np
import torch

from mixture_experts_top_b200 import api

MARGIN = 1e-5
REL_ROUTE = 1e-5
REL_F32 = 1e-4
RMS_BF16 = 2e-2


def dev(a):
    """numpy -> CUDA tensor (uint16 arrays are bf16 bit patterns)."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def host(t):
    """CUDA tensor -> numpy (bf16 -> uint16 bit patterns)."""
    t = t.detach()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def cfg_of(w, T=None):
    return api.make_config(w.T if T is None else T, w.d, w.d_hidden, w.d_out, w.E, w.top_k,
                           w.kind, w.dtype, w.capacity_factor)


def ambiguous_tokens(L, k):
    """Tokens whose top-(k) set or order is decided by a gap below MARGIN."""
    Ls = -np.sort(-np.asarray(L, np.float64), axis=1)
    upto = min(k + 1, Ls.shape[1])
    gaps = Ls[:, :upto - 1] - Ls[:, 1:upto]
    if gaps.shape[1] == 0:
        return np.zeros(Ls.shape[0], bool)
    return gaps.min(axis=1) < MARGIN


def rel_close(a, b, rel):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.all(np.abs(a - b) <= rel * np.maximum(np.abs(b), 1e-30))


def layer_tolerance(ref_rows, rms_expert_rows):
    """Per-element bound on the bf16 layer output (see the module docstring)."""
    return RMS_BF16 * rms_expert_rows + bf16_ulp(ref_rows)


def bf16_ulp(v):
    """One bf16 ulp at |v| (2^(e-7) for the binade of v)."""
    v = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.maximum(v, 1e-38)))
    return 2.0 ** (e - 7)
