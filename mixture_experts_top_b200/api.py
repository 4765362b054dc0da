"""Python binding of ``libmoe_b200.so`` (the C ABI in ``include/moe.h``).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  torch tensors supply device pointers and torch supplies the current
CUDA stream; nothing here computes any part of the layer, and there is no
fallback: if the library is missing or a call fails, an exception is raised.

Function names match the C entry points.  Each takes a :class:`MoeConfig`
and torch tensors (``None`` where the C side accepts NULL) and raises
:class:`MoeError` on a non-OK status.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

LIB_NAME = "libmoe_b200.so"
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), LIB_NAME)

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, \
    MOE_ERR_DEVICE_CHECK = range(6)
EXPERT_KINDS = {"linear": 0, "relu": 1, "swiglu": 2}
DTYPES = {"f32": 0, "bf16": 1}

# Every symbol the header declares, with its ctypes signature.
_c_p = ctypes.c_void_p
_SIGNATURES = {
    "moe_workspace_size": (ctypes.c_size_t, [_c_p]),
    "moe_workspace_init": (ctypes.c_int, [_c_p, ctypes.c_size_t, _c_p]),
    "moe_device_status": (ctypes.c_int, [_c_p, ctypes.c_size_t, _c_p, _c_p]),
    "moe_route": (ctypes.c_int, [_c_p] * 10 + [ctypes.c_size_t, _c_p]),
    "moe_route_noalloc": (ctypes.c_int, [_c_p] * 10),
    "moe_route_noisy": (ctypes.c_int, [_c_p] * 5 + [ctypes.c_uint64, ctypes.c_uint64,
                                                    ctypes.c_int64] + [_c_p] * 6
                        + [ctypes.c_size_t, _c_p]),
    "moe_check_wait_timeout": (ctypes.c_int, [_c_p, ctypes.c_size_t, ctypes.c_uint32, _c_p]),
    "moe_expert_backward_workspace_size": (ctypes.c_size_t, [_c_p]),
    "moe_expert_ffn_backward": (ctypes.c_int, [_c_p] * 12 + [ctypes.c_size_t, _c_p]),
    "moe_expert_ffn_backward_saved": (ctypes.c_int, [_c_p] * 12 + [ctypes.c_size_t, _c_p]),
    "moe_expert_ffn_train": (ctypes.c_int, [_c_p] * 8 + [ctypes.c_size_t, _c_p, ctypes.c_size_t,
                                                          _c_p]),
    "moe_permute_backward": (ctypes.c_int, [_c_p] * 6),
    "moe_combine_backward": (ctypes.c_int, [_c_p] * 8),
    "moe_route_backward": (ctypes.c_int, [_c_p] * 9 + [ctypes.c_int32] + [_c_p] * 5 +
                           [ctypes.c_size_t, _c_p]),
    "moe_gate_noise": (ctypes.c_int, [_c_p] * 3 + [ctypes.c_uint64, ctypes.c_uint64,
                                                   ctypes.c_int64, _c_p, _c_p, ctypes.c_size_t,
                                                   _c_p]),
    "moe_dispatch": (ctypes.c_int, [_c_p] * 13 + [ctypes.c_size_t, _c_p]),
    "moe_dispatch_count": (ctypes.c_int, [_c_p] * 4 + [ctypes.c_size_t, _c_p]),
    "moe_shard_record": (ctypes.c_int, [_c_p] * 5 + [ctypes.c_size_t, _c_p]),
    "moe_dispatch_shard": (ctypes.c_int, [_c_p] * 14 + [ctypes.c_size_t, _c_p]),
    "moe_expert_ffn": (ctypes.c_int, [_c_p] * 8 + [ctypes.c_size_t, _c_p]),
    "moe_expert_ffn_gather": (ctypes.c_int, [_c_p] * 9 + [ctypes.c_size_t, _c_p]),
    "moe_combine": (ctypes.c_int, [_c_p] * 6),
    "moe_expert_ffn_combine": (ctypes.c_int, [_c_p] * 11 + [ctypes.c_size_t, _c_p]),
    "moe_forward_combine_fused": (ctypes.c_int, [_c_p, _c_p]),
    "moe_forward": (ctypes.c_int, [_c_p] * 15 + [ctypes.c_size_t, _c_p]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_last_error_message": (ctypes.c_char_p, []),
}


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: status {status} ({message})")
        self.status = status


class MoeConfig(ctypes.Structure):
    """Mirror of ``moe_config_t``."""
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("d_hidden", ctypes.c_int32),
                ("d_out", ctypes.c_int32), ("E", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("expert_kind", ctypes.c_int32), ("act_dtype", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float)]


class MoeShard(ctypes.Structure):
    """Mirror of ``moe_shard_t``: this rank of a batch split over ranks and
    every rank's exchange record (world, 2E+1) int32."""
    _fields_ = [("rank", ctypes.c_int32), ("world", ctypes.c_int32), ("T_global", ctypes.c_int32),
                ("records", ctypes.c_void_p)]


def make_config(T: int, d: int, d_hidden: int, d_out: int, E: int, top_k: int, kind: str,
                dtype: str, capacity_factor: float = 0.0) -> MoeConfig:
    return MoeConfig(T, d, d_hidden, d_out, E, top_k, EXPERT_KINDS[kind], DTYPES[dtype],
                     float(capacity_factor))


def router_tc_width_supported(cfg: "MoeConfig") -> bool:
    """Whether the tensor-core router (and moe_gate_noise) serves `cfg`:
    bf16 activations and at most 64 experts."""
    return cfg.act_dtype == DTYPES["bf16"] and cfg.E <= 64


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"{LIB_NAME} not found at {path}: build it with "
                               "`python -m mixture_experts_top_b200.build` (needs nvcc)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def exported_symbols() -> list:
    return list(_SIGNATURES)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor arguments must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        lib = load_library()
        msg = lib.moe_last_error_message().decode() or lib.moe_status_string(status).decode()
        raise MoeError(status, where, msg)


def moe_workspace_size(cfg: MoeConfig) -> int:
    n = load_library().moe_workspace_size(ctypes.byref(cfg))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_workspace_size",
                       load_library().moe_last_error_message().decode())
    return n


def moe_workspace_init(ws, stream=None) -> None:
    _check(load_library().moe_workspace_init(_ptr(ws), ws.numel(), _stream(stream)),
           "moe_workspace_init")


def moe_device_status(ws, stream=None) -> int:
    code = ctypes.c_int32(0)
    st = load_library().moe_device_status(_ptr(ws), ws.numel(), ctypes.byref(code), _stream(stream))
    if st not in (MOE_OK, MOE_ERR_DEVICE_CHECK):
        _check(st, "moe_device_status")
    return int(code.value)


def alloc_workspace(cfg: MoeConfig, device="cuda", stream=None):
    """Caller-owned workspace as a torch uint8 tensor, error word cleared."""
    import torch
    ws = torch.empty(moe_workspace_size(cfg), dtype=torch.uint8, device=device)
    moe_workspace_init(ws, stream)
    return ws


def moe_route(cfg, x, W_router, logit_bias, noise, expert_indices, gates, prob_mean, logits_out,
              ws, stream=None) -> None:
    _check(load_library().moe_route(
        ctypes.byref(cfg), _ptr(x), _ptr(W_router), _ptr(logit_bias), _ptr(noise),
        _ptr(expert_indices), _ptr(gates), _ptr(prob_mean), _ptr(logits_out), _ptr(ws),
        ws.numel(), _stream(stream)), "moe_route")


def moe_route_noisy(cfg, x, W_router, logit_bias, W_noise, seed, offset, token_base,
                    expert_indices, gates, prob_mean, logits_out, noise_out, ws,
                    stream=None) -> None:
    _check(load_library().moe_route_noisy(
        ctypes.byref(cfg), _ptr(x), _ptr(W_router), _ptr(logit_bias), _ptr(W_noise), int(seed),
        int(offset), int(token_base), _ptr(expert_indices), _ptr(gates), _ptr(prob_mean),
        _ptr(logits_out), _ptr(noise_out), _ptr(ws), ws.numel(), _stream(stream)),
        "moe_route_noisy")


def moe_route_noalloc(cfg, x, W_router, logit_bias, noise, expert_indices, gates, prob_mean,
                      logits_out, stream=None) -> None:
    """moe_route for callers that cannot allocate: no workspace argument;
    the library's fixed scratch array is used (see include/moe.h)."""
    _check(load_library().moe_route_noalloc(
        ctypes.byref(cfg), _ptr(x), _ptr(W_router), _ptr(logit_bias), _ptr(noise),
        _ptr(expert_indices), _ptr(gates), _ptr(prob_mean), _ptr(logits_out), _stream(stream)),
        "moe_route_noalloc")


def moe_combine_backward(cfg, dy, y_perm, dest, gates, dy_perm, dgates, stream=None) -> None:
    _check(load_library().moe_combine_backward(
        ctypes.byref(cfg), _ptr(dy), _ptr(y_perm), _ptr(dest), _ptr(gates), _ptr(dy_perm),
        _ptr(dgates), _stream(stream)), "moe_combine_backward")


def moe_route_backward(cfg, x, W_router, logits, expert_indices, gates, f, dgates, daux, T_batch,
                       dx, dW_router, dbias, dlogits, ws, stream=None) -> None:
    _check(load_library().moe_route_backward(
        ctypes.byref(cfg), _ptr(x), _ptr(W_router), _ptr(logits), _ptr(expert_indices),
        _ptr(gates), _ptr(f), _ptr(dgates), _ptr(daux), int(T_batch), _ptr(dx), _ptr(dW_router),
        _ptr(dbias), _ptr(dlogits), _ptr(ws), ws.numel(), _stream(stream)), "moe_route_backward")


def moe_expert_backward_workspace_size(cfg: MoeConfig) -> int:
    n = load_library().moe_expert_backward_workspace_size(ctypes.byref(cfg))
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_expert_backward_workspace_size",
                       load_library().moe_last_error_message().decode())
    return n


def alloc_backward_workspace(cfg: MoeConfig, device="cuda", stream=None):
    """Caller-owned workspace of moe_expert_ffn_backward, error word cleared."""
    import torch
    ws = torch.empty(moe_expert_backward_workspace_size(cfg), dtype=torch.uint8, device=device)
    moe_workspace_init(ws, stream)
    return ws


def moe_expert_ffn_backward(cfg, x_perm, offsets, W_in, W_up, W_out, dy_perm, dx_perm, dW_in,
                            dW_up, dW_out, ws, stream=None) -> None:
    _check(load_library().moe_expert_ffn_backward(
        ctypes.byref(cfg), _ptr(x_perm), _ptr(offsets), _ptr(W_in), _ptr(W_up), _ptr(W_out),
        _ptr(dy_perm), _ptr(dx_perm), _ptr(dW_in), _ptr(dW_up), _ptr(dW_out), _ptr(ws),
        ws.numel(), _stream(stream)), "moe_expert_ffn_backward")


def moe_permute_backward(cfg, dx_perm, dest, dx_add, dx, stream=None) -> None:
    _check(load_library().moe_permute_backward(
        ctypes.byref(cfg), _ptr(dx_perm), _ptr(dest), _ptr(dx_add), _ptr(dx), _stream(stream)),
        "moe_permute_backward")


def moe_check_wait_timeout(ws, limit_us: int, stream=None) -> None:
    _check(load_library().moe_check_wait_timeout(_ptr(ws), ws.numel(), int(limit_us),
                                                  _stream(stream)), "moe_check_wait_timeout")


def moe_gate_noise(cfg, x, W_noise, seed, offset, token_base, noise_out, ws, stream=None) -> None:
    _check(load_library().moe_gate_noise(
        ctypes.byref(cfg), _ptr(x), _ptr(W_noise), int(seed), int(offset), int(token_base),
        _ptr(noise_out), _ptr(ws), ws.numel(), _stream(stream)), "moe_gate_noise")


def moe_dispatch(cfg, x, expert_indices, prob_mean, counts, offsets, dest, perm_token, drop_mask,
                 f, aux_loss, x_perm, ws, stream=None) -> None:
    _check(load_library().moe_dispatch(
        ctypes.byref(cfg), _ptr(x), _ptr(expert_indices), _ptr(prob_mean), _ptr(counts),
        _ptr(offsets), _ptr(dest), _ptr(perm_token), _ptr(drop_mask), _ptr(f), _ptr(aux_loss),
        _ptr(x_perm), _ptr(ws), ws.numel(), _stream(stream)), "moe_dispatch")


def moe_dispatch_count(cfg, expert_indices, counts, ws, stream=None) -> None:
    _check(load_library().moe_dispatch_count(
        ctypes.byref(cfg), _ptr(expert_indices), _ptr(counts), _ptr(ws), ws.numel(),
        _stream(stream)), "moe_dispatch_count")


def moe_shard_record(cfg, expert_indices, prob_mean, record, ws, stream=None) -> None:
    _check(load_library().moe_shard_record(
        ctypes.byref(cfg), _ptr(expert_indices), _ptr(prob_mean), _ptr(record), _ptr(ws),
        ws.numel(), _stream(stream)), "moe_shard_record")


def moe_dispatch_shard(cfg, rank, world, T_global, records, x, expert_indices, prob_mean,
                       counts, offsets, dest, perm_token, drop_mask, f, aux_loss, x_perm, ws,
                       stream=None) -> None:
    shard = MoeShard(rank, world, T_global, _ptr(records))
    _check(load_library().moe_dispatch_shard(
        ctypes.byref(cfg), ctypes.byref(shard), _ptr(x), _ptr(expert_indices), _ptr(prob_mean),
        _ptr(counts), _ptr(offsets), _ptr(dest), _ptr(perm_token), _ptr(drop_mask), _ptr(f),
        _ptr(aux_loss), _ptr(x_perm), _ptr(ws), ws.numel(), _stream(stream)),
        "moe_dispatch_shard")


def moe_expert_ffn_backward_saved(cfg, x_perm, offsets, W_in, W_up, W_out, dy_perm, dx_perm,
                                  dW_in, dW_up, dW_out, ws, stream=None) -> None:
    """moe_expert_ffn_backward with the pre-activations that
    moe_expert_ffn_train left in `ws`."""
    _check(load_library().moe_expert_ffn_backward_saved(
        ctypes.byref(cfg), _ptr(x_perm), _ptr(offsets), _ptr(W_in), _ptr(W_up), _ptr(W_out),
        _ptr(dy_perm), _ptr(dx_perm), _ptr(dW_in), _ptr(dW_up), _ptr(dW_out), _ptr(ws),
        ws.numel(), _stream(stream)), "moe_expert_ffn_backward_saved")


def moe_expert_ffn_train(cfg, x_perm, offsets, W_in, W_up, W_out, y_perm, ws, bwd_ws,
                         stream=None) -> None:
    """moe_expert_ffn that also keeps the pre-activations in bwd_ws (the
    experts' backward workspace)."""
    _check(load_library().moe_expert_ffn_train(
        ctypes.byref(cfg), _ptr(x_perm), _ptr(offsets), _ptr(W_in), _ptr(W_up), _ptr(W_out),
        _ptr(y_perm), _ptr(ws), ws.numel(), _ptr(bwd_ws), bwd_ws.numel(), _stream(stream)),
        "moe_expert_ffn_train")


def moe_expert_ffn(cfg, x_perm, offsets, W_in, W_up, W_out, y_perm, ws, stream=None) -> None:
    _check(load_library().moe_expert_ffn(
        ctypes.byref(cfg), _ptr(x_perm), _ptr(offsets), _ptr(W_in), _ptr(W_up), _ptr(W_out),
        _ptr(y_perm), _ptr(ws), ws.numel(), _stream(stream)), "moe_expert_ffn")


def moe_expert_ffn_gather(cfg, x, perm_token, offsets, W_in, W_up, W_out, y_perm, ws,
                          stream=None) -> None:
    _check(load_library().moe_expert_ffn_gather(
        ctypes.byref(cfg), _ptr(x), _ptr(perm_token), _ptr(offsets), _ptr(W_in), _ptr(W_up),
        _ptr(W_out), _ptr(y_perm), _ptr(ws), ws.numel(), _stream(stream)), "moe_expert_ffn_gather")


def moe_expert_ffn_combine(cfg, x_perm, offsets, perm_token, dest, gates, W_in, W_up, W_out,
                           output, ws, stream=None) -> None:
    _check(load_library().moe_expert_ffn_combine(
        ctypes.byref(cfg), _ptr(x_perm), _ptr(offsets), _ptr(perm_token), _ptr(dest), _ptr(gates),
        _ptr(W_in), _ptr(W_up), _ptr(W_out), _ptr(output), _ptr(ws), ws.numel(), _stream(stream)),
        "moe_expert_ffn_combine")


def moe_forward_combine_fused(cfg) -> bool:
    """Whether moe_forward runs the combine in the down projection's epilogue
    (moe_expert_ffn_combine) for cfg, rather than moe_expert_ffn then
    moe_combine.  Host-only."""
    out = ctypes.c_int32(0)
    _check(load_library().moe_forward_combine_fused(ctypes.byref(cfg), ctypes.byref(out)),
           "moe_forward_combine_fused")
    return bool(out.value)


def moe_combine(cfg, y_perm, dest, gates, output, stream=None) -> None:
    _check(load_library().moe_combine(
        ctypes.byref(cfg), _ptr(y_perm), _ptr(dest), _ptr(gates), _ptr(output), _stream(stream)),
        "moe_combine")


def moe_forward(cfg, x, W_router, logit_bias, noise, W_in, W_up, W_out, output, expert_indices,
                gates, aux_loss, counts, drop_mask, ws, stream=None) -> None:
    _check(load_library().moe_forward(
        ctypes.byref(cfg), _ptr(x), _ptr(W_router), _ptr(logit_bias), _ptr(noise), _ptr(W_in),
        _ptr(W_up), _ptr(W_out), _ptr(output), _ptr(expert_indices), _ptr(gates), _ptr(aux_loss),
        _ptr(counts), _ptr(drop_mask), _ptr(ws), ws.numel(), _stream(stream)), "moe_forward")
