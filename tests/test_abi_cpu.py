"""The C-ABI library loads, exports every declared entry point, and rejects
bad arguments on the host -- all without a GPU (no call here reaches CUDA:
each one fails an argument check first)."""
import ctypes
import os
import re

import pytest

from mixture_experts_top_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(moe_lib):
    names = declared_functions()
    assert len(names) == 27
    for n in names:
        assert hasattr(moe_lib, n), n
    assert sorted(api.exported_symbols()) == names


def _cfg(**kw):
    base = dict(T=64, d=32, d_hidden=0, d_out=32, E=8, top_k=2, kind="linear", dtype="f32",
                capacity_factor=0.0)
    base.update(kw)
    return api.make_config(**base)


FAKE = 0x7F0000000000          # 256-aligned, never dereferenced


@pytest.mark.parametrize("name,fused", [("mixtral", True), ("decode", False),
                                        ("fine_grained", False), ("switch_relu", True),
                                        ("tiny_linear", False)])
def test_forward_combine_form(name, fused):
    """moe_forward's form of the experts and the combine (host-only query):
    in the down projection's epilogue at top-1 and where long tiles hide the
    top-k epilogue's reads (Mixtral: d_hidden 14336, 16384 grouped rows), as
    two calls otherwise (64 tokens; d_hidden 1408; fp32 linear experts)."""
    from workloads import WORKLOADS
    w = WORKLOADS[name]
    cfg = api.make_config(w.T, w.d, w.d_hidden, w.d_out, w.E, w.top_k, w.kind, w.dtype,
                          w.capacity_factor)
    assert api.moe_forward_combine_fused(cfg) is fused
    with pytest.raises(RuntimeError):
        api.moe_forward_combine_fused(_cfg(top_k=0))


@pytest.mark.parametrize("kw,status", [
    (dict(top_k=0), api.MOE_ERR_INVALID_ARG),
    (dict(top_k=9, E=16), api.MOE_ERR_UNSUPPORTED),
    (dict(top_k=9), api.MOE_ERR_INVALID_ARG),            # k > E
    (dict(E=0), api.MOE_ERR_INVALID_ARG),
    (dict(E=257, top_k=2), api.MOE_ERR_UNSUPPORTED),
    (dict(T=-1), api.MOE_ERR_INVALID_ARG),
    (dict(d=12), api.MOE_ERR_UNSUPPORTED),
    (dict(d_out=4), api.MOE_ERR_UNSUPPORTED),
    (dict(dtype="bf16"), api.MOE_ERR_UNSUPPORTED),       # linear experts are fp32 only
    (dict(kind="swiglu", d_hidden=64), api.MOE_ERR_UNSUPPORTED),  # SwiGLU is bf16 only
    (dict(kind="relu", dtype="bf16", d_hidden=12), api.MOE_ERR_UNSUPPORTED),
    (dict(capacity_factor=float("nan")), api.MOE_ERR_INVALID_ARG),
    (dict(T=1 << 29, top_k=4), api.MOE_ERR_UNSUPPORTED),  # T*k >= 2^31
])
def test_config_checks(moe_lib, kw, status):
    cfg = _cfg(**kw)
    assert moe_lib.moe_workspace_size(ctypes.byref(cfg)) == 0
    st = moe_lib.moe_forward(ctypes.byref(cfg), *([FAKE] * 7), FAKE, FAKE, FAKE, FAKE, None,
                             None, FAKE, 1 << 40, None)
    assert st == status, moe_lib.moe_last_error_message()


def test_unknown_enum_values(moe_lib):
    cfg = _cfg()
    cfg.expert_kind = 7
    assert moe_lib.moe_workspace_size(ctypes.byref(cfg)) == 0
    cfg = _cfg()
    cfg.act_dtype = 5
    assert moe_lib.moe_workspace_size(ctypes.byref(cfg)) == 0


def test_null_config(moe_lib):
    assert moe_lib.moe_workspace_size(None) == 0
    assert moe_lib.moe_combine(None, FAKE, FAKE, FAKE, FAKE, None) == api.MOE_ERR_INVALID_ARG


def test_workspace_size_grows_with_tokens(moe_lib):
    small = moe_lib.moe_workspace_size(ctypes.byref(_cfg(T=64)))
    big = moe_lib.moe_workspace_size(ctypes.byref(_cfg(T=6400)))
    assert 0 < small < big and small % 256 == 0 and big % 256 == 0
    cfg = api.make_config(8192, 4096, 14336, 4096, 8, 2, "swiglu", "bf16")
    n = moe_lib.moe_workspace_size(ctypes.byref(cfg))
    # grouped copies of x, the hidden activation and the expert outputs dominate
    rows = 8192 * 2
    assert n >= rows * (4096 + 14336 + 4096) * 2


def test_null_pointers_and_workspace(moe_lib):
    cfg = _cfg()
    ws = moe_lib.moe_workspace_size(ctypes.byref(cfg))
    # x, W_router, bias, noise, W_in, W_up, W_out | output, indices, gates, aux | counts, drops
    args = [FAKE] * 7 + [FAKE, FAKE, FAKE, FAKE] + [None, None]
    # x is NULL
    st = moe_lib.moe_forward(ctypes.byref(cfg), None, *args[1:], FAKE, ws, None)
    assert st == api.MOE_ERR_INVALID_ARG
    assert "x" in moe_lib.moe_last_error_message().decode()
    # W_up may be NULL for linear experts, but the workspace may not
    st = moe_lib.moe_forward(ctypes.byref(cfg), *args, None, ws, None)
    assert st == api.MOE_ERR_WORKSPACE
    st = moe_lib.moe_forward(ctypes.byref(cfg), *args, FAKE + 16, ws, None)   # misaligned
    assert st == api.MOE_ERR_WORKSPACE
    st = moe_lib.moe_forward(ctypes.byref(cfg), *args, FAKE, ws - 1, None)    # too small
    assert st == api.MOE_ERR_WORKSPACE
    assert moe_lib.moe_workspace_init(None, 1024, None) == api.MOE_ERR_WORKSPACE
    code = ctypes.c_int32()
    assert moe_lib.moe_device_status(None, 1024, ctypes.byref(code), None) == api.MOE_ERR_WORKSPACE


def test_row_tensors_must_be_16_byte_aligned(moe_lib):
    cfg = api.make_config(64, 64, 128, 64, 8, 2, "swiglu", "bf16")
    ws = moe_lib.moe_workspace_size(ctypes.byref(cfg))
    st = moe_lib.moe_route(ctypes.byref(cfg), FAKE + 8, FAKE, None, None, FAKE, FAKE, FAKE, None,
                           FAKE, ws, None)
    assert st == api.MOE_ERR_INVALID_ARG
    assert "x must be 16-byte aligned" in moe_lib.moe_last_error_message().decode()
    st = moe_lib.moe_expert_ffn(ctypes.byref(cfg), FAKE, FAKE, FAKE, FAKE + 2, FAKE, FAKE, FAKE,
                                ws, None)
    assert st == api.MOE_ERR_INVALID_ARG
    assert "W_up must be 16-byte aligned" in moe_lib.moe_last_error_message().decode()
    st = moe_lib.moe_combine(ctypes.byref(cfg), FAKE, FAKE, FAKE, FAKE + 4, None)
    assert st == api.MOE_ERR_INVALID_ARG


def test_workspace_holds_the_split_router_weights(moe_lib):
    """bf16 with E <= 64 adds 6 * EP * d bf16 for the tensor-core router
    (W_router's three terms, and W_noise's for the fused noisy router)."""
    a = api.make_config(64, 4096, 128, 64, 8, 2, "swiglu", "bf16")
    b = api.make_config(64, 4096, 128, 64, 100, 2, "swiglu", "bf16")   # E > 64: SIMT router
    c = api.make_config(64, 4096, 128, 64, 16, 2, "swiglu", "bf16")
    na, nb, nc = (moe_lib.moe_workspace_size(ctypes.byref(x)) for x in (a, b, c))
    assert na >= 6 * 16 * 4096 * 2 and nc >= 6 * 16 * 4096 * 2
    assert nb > 0


def test_shard_and_gather_argument_checks(moe_lib):
    cfg = api.make_config(64, 64, 128, 64, 8, 2, "swiglu", "bf16")
    ws = moe_lib.moe_workspace_size(ctypes.byref(cfg))
    outs = [FAKE] * 7                      # counts, offsets, dest, perm, drop, f, aux
    st = moe_lib.moe_dispatch_shard(ctypes.byref(cfg), None, FAKE, FAKE, FAKE, *outs, FAKE,
                                    FAKE, ws, None)
    assert st == api.MOE_ERR_INVALID_ARG and "shard" in moe_lib.moe_last_error_message().decode()
    for rank, world, T_g, records in [(2, 2, 128, FAKE), (-1, 2, 128, FAKE), (0, 0, 128, FAKE),
                                      (0, 2, 32, FAKE), (0, 2, 128, None)]:
        sh = api.MoeShard(rank, world, T_g, records)
        st = moe_lib.moe_dispatch_shard(ctypes.byref(cfg), ctypes.byref(sh), FAKE, FAKE, FAKE,
                                        *outs, FAKE, FAKE, ws, None)
        assert st == api.MOE_ERR_INVALID_ARG, (rank, world, T_g)
    assert moe_lib.moe_dispatch_count(ctypes.byref(cfg), FAKE, None, FAKE, ws, None) == \
        api.MOE_ERR_INVALID_ARG
    assert moe_lib.moe_dispatch_count(ctypes.byref(cfg), FAKE, FAKE, FAKE, ws - 1, None) == \
        api.MOE_ERR_WORKSPACE
    assert moe_lib.moe_shard_record(ctypes.byref(cfg), FAKE, None, FAKE, FAKE, ws, None) == \
        api.MOE_ERR_INVALID_ARG
    assert moe_lib.moe_shard_record(ctypes.byref(cfg), FAKE, FAKE, None, FAKE, ws, None) == \
        api.MOE_ERR_INVALID_ARG
    # gather: perm_token required, x aligned
    st = moe_lib.moe_expert_ffn_gather(ctypes.byref(cfg), FAKE, None, FAKE, FAKE, FAKE, FAKE,
                                       FAKE, FAKE, ws, None)
    assert st == api.MOE_ERR_INVALID_ARG and "perm_token" in moe_lib.moe_last_error_message().decode()
    st = moe_lib.moe_expert_ffn_gather(ctypes.byref(cfg), FAKE + 8, FAKE, FAKE, FAKE, FAKE, FAKE,
                                       FAKE, FAKE, ws, None)
    assert st == api.MOE_ERR_INVALID_ARG and "16-byte" in moe_lib.moe_last_error_message().decode()


def test_gate_noise_argument_checks(moe_lib):
    cfg = api.make_config(64, 64, 128, 64, 8, 2, "swiglu", "bf16")
    ws = moe_lib.moe_workspace_size(ctypes.byref(cfg))
    assert moe_lib.moe_gate_noise(ctypes.byref(cfg), FAKE, None, 1, 0, 0, FAKE, FAKE, ws,
                                  None) == api.MOE_ERR_INVALID_ARG
    assert moe_lib.moe_gate_noise(ctypes.byref(cfg), FAKE, FAKE, 1, 0, -1, FAKE, FAKE, ws,
                                  None) == api.MOE_ERR_INVALID_ARG
    assert moe_lib.moe_gate_noise(ctypes.byref(cfg), FAKE + 8, FAKE, 1, 0, 0, FAKE, FAKE, ws,
                                  None) == api.MOE_ERR_INVALID_ARG
    wide = api.make_config(64, 64, 128, 64, 100, 2, "swiglu", "bf16")     # E > 64
    ws2 = moe_lib.moe_workspace_size(ctypes.byref(wide))
    assert moe_lib.moe_gate_noise(ctypes.byref(wide), FAKE, FAKE, 1, 0, 0, FAKE, FAKE, ws2,
                                  None) == api.MOE_ERR_UNSUPPORTED
    # the fused noisy router: same limits, W_noise required
    outs = [FAKE, FAKE, FAKE, None, None]   # indices, gates, P, logits_out, noise_out
    assert moe_lib.moe_route_noisy(ctypes.byref(wide), FAKE, FAKE, None, FAKE, 1, 0, 0, *outs,
                                   FAKE, ws2, None) == api.MOE_ERR_UNSUPPORTED
    assert moe_lib.moe_route_noisy(ctypes.byref(cfg), FAKE, FAKE, None, None, 1, 0, 0, *outs,
                                   FAKE, ws, None) == api.MOE_ERR_INVALID_ARG
    assert moe_lib.moe_route_noisy(ctypes.byref(cfg), FAKE, FAKE, None, FAKE, 1, 0, -2, *outs,
                                   FAKE, ws, None) == api.MOE_ERR_INVALID_ARG


def test_backward_argument_checks(moe_lib):
    cfg = api.make_config(64, 64, 128, 64, 8, 2, "swiglu", "bf16")
    ws = moe_lib.moe_workspace_size(ctypes.byref(cfg))
    assert moe_lib.moe_combine_backward(ctypes.byref(cfg), None, FAKE, FAKE, FAKE, FAKE, FAKE,
                                        None) == api.MOE_ERR_INVALID_ARG
    assert moe_lib.moe_combine_backward(ctypes.byref(cfg), FAKE + 4, FAKE, FAKE, FAKE, FAKE, FAKE,
                                        None) == api.MOE_ERR_INVALID_ARG
    args = [FAKE] * 8                        # x, W, logits, idx, gates, f, dgates, daux
    ok_tail = [FAKE, FAKE, None, None, FAKE, ws, None]
    # T_batch below this call's T
    assert moe_lib.moe_route_backward(ctypes.byref(cfg), *args, 32, *ok_tail) == \
        api.MOE_ERR_INVALID_ARG
    # dW missing
    assert moe_lib.moe_route_backward(ctypes.byref(cfg), *args, 0, FAKE, None, None, None, FAKE,
                                      ws, None) == api.MOE_ERR_INVALID_ARG
    # workspace too small
    assert moe_lib.moe_route_backward(ctypes.byref(cfg), *args, 0, FAKE, FAKE, None, None, FAKE,
                                      ws - 256, None) == api.MOE_ERR_WORKSPACE


def test_expert_backward_argument_checks(moe_lib):
    cfg = api.make_config(64, 64, 128, 64, 8, 2, "swiglu", "bf16")
    n = moe_lib.moe_expert_backward_workspace_size(ctypes.byref(cfg))
    # padded rows (T*k + E*63) of Xp, dYp, [dA|dB] and H in bf16, [A|B] in fp32
    rows = 64 * 2 + 8 * 63
    assert n >= rows * ((64 + 64 + 2 * 128 + 128) * 2 + 2 * 128 * 4) and n % 256 == 0
    lin = api.make_config(64, 32, 0, 32, 8, 2, "linear", "f32")
    assert 0 < moe_lib.moe_expert_backward_workspace_size(ctypes.byref(lin)) < n
    ins = [FAKE] * 6                          # x_perm, offsets, W_in, W_up, W_out, dy_perm
    outs = [FAKE] * 4                         # dx_perm, dW_in, dW_up, dW_out
    # SwiGLU needs dW_up
    st = moe_lib.moe_expert_ffn_backward(ctypes.byref(cfg), *ins, FAKE, FAKE, None, FAKE, FAKE,
                                         n, None)
    assert st == api.MOE_ERR_INVALID_ARG and "dW_up" in moe_lib.moe_last_error_message().decode()
    # misaligned gradient output
    st = moe_lib.moe_expert_ffn_backward(ctypes.byref(cfg), *ins, FAKE + 4, FAKE, FAKE, FAKE,
                                         FAKE, n, None)
    assert st == api.MOE_ERR_INVALID_ARG and "dx_perm" in moe_lib.moe_last_error_message().decode()
    # workspace too small, misaligned
    assert moe_lib.moe_expert_ffn_backward(ctypes.byref(cfg), *ins, *outs, FAKE, n - 256,
                                           None) == api.MOE_ERR_WORKSPACE
    assert moe_lib.moe_expert_ffn_backward(ctypes.byref(cfg), *ins, *outs, FAKE + 16, n,
                                           None) == api.MOE_ERR_WORKSPACE
    # linear experts: W_out, W_up and their gradients may be NULL; dW_in may not
    st = moe_lib.moe_expert_ffn_backward(ctypes.byref(lin), FAKE, FAKE, FAKE, None, None, FAKE,
                                         FAKE, None, None, None, FAKE, n, None)
    assert st == api.MOE_ERR_INVALID_ARG and "dW_in" in moe_lib.moe_last_error_message().decode()
    # the saved-pre-activation backward: same checks, and linear experts refused
    st = moe_lib.moe_expert_ffn_backward_saved(ctypes.byref(cfg), *ins, FAKE, FAKE, None, FAKE,
                                               FAKE, n, None)
    assert st == api.MOE_ERR_INVALID_ARG and "dW_up" in moe_lib.moe_last_error_message().decode()
    assert moe_lib.moe_expert_ffn_backward_saved(ctypes.byref(cfg), *ins, *outs, FAKE, n - 256,
                                                 None) == api.MOE_ERR_WORKSPACE
    assert moe_lib.moe_expert_ffn_backward_saved(ctypes.byref(lin), FAKE, FAKE, FAKE, None, None,
                                                 FAKE, FAKE, FAKE, None, None, FAKE, n, None) \
        == api.MOE_ERR_UNSUPPORTED
    # rows back to tokens
    assert moe_lib.moe_permute_backward(ctypes.byref(cfg), None, FAKE, None, FAKE, None) == \
        api.MOE_ERR_INVALID_ARG
    assert moe_lib.moe_permute_backward(ctypes.byref(cfg), FAKE, FAKE, FAKE + 8, FAKE, None) == \
        api.MOE_ERR_INVALID_ARG


def test_swiglu_needs_three_matrices(moe_lib):
    cfg = api.make_config(64, 64, 128, 64, 8, 2, "swiglu", "bf16")
    ws = moe_lib.moe_workspace_size(ctypes.byref(cfg))
    st = moe_lib.moe_expert_ffn(ctypes.byref(cfg), FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, ws,
                                None)
    assert st == api.MOE_ERR_INVALID_ARG and "W_up" in moe_lib.moe_last_error_message().decode()


def test_status_strings(moe_lib):
    for s in range(6):
        assert moe_lib.moe_status_string(s).startswith(b"MOE_")
    assert moe_lib.moe_status_string(99) == b"unknown status"


def test_binding_refuses_missing_library(tmp_path):
    """No fallback: without the library every call raises."""
    saved = api._lib
    api._lib = None
    try:
        with pytest.raises(RuntimeError, match="not found"):
            api.load_library(str(tmp_path / "none.so"))
    finally:
        api._lib = saved


def test_training_forward_argument_checks(moe_lib):
    cfg = api.make_config(64, 64, 128, 64, 8, 2, "swiglu", "bf16")
    ws = moe_lib.moe_workspace_size(ctypes.byref(cfg))
    bws = moe_lib.moe_expert_backward_workspace_size(ctypes.byref(cfg))
    args = [FAKE] * 7                          # x_perm, offsets, W_in, W_up, W_out, y_perm, ws
    ok = lambda *tail: moe_lib.moe_expert_ffn_train(ctypes.byref(cfg), *args, ws, *tail)
    # the backward workspace: NULL, too small, misaligned
    assert ok(None, bws, None) == api.MOE_ERR_WORKSPACE
    assert "backward workspace" in moe_lib.moe_last_error_message().decode()
    assert ok(FAKE, bws - 256, None) == api.MOE_ERR_WORKSPACE
    assert ok(FAKE + 16, bws, None) == api.MOE_ERR_WORKSPACE
    # SwiGLU needs W_up; linear experts keep no pre-activations
    st = moe_lib.moe_expert_ffn_train(ctypes.byref(cfg), FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE,
                                      ws, FAKE, bws, None)
    assert st == api.MOE_ERR_INVALID_ARG and "W_up" in moe_lib.moe_last_error_message().decode()
    lin = api.make_config(64, 32, 0, 32, 8, 2, "linear", "f32")
    st = moe_lib.moe_expert_ffn_train(ctypes.byref(lin), FAKE, FAKE, FAKE, None, None, FAKE, FAKE,
                                      ws, FAKE, bws, None)
    assert st == api.MOE_ERR_UNSUPPORTED
