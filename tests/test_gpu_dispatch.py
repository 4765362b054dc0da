"""GPU dispatch (moe_dispatch) against the CPU oracle, on the same indices.

Everything integer is bit-exact: counts, offsets, dest, perm_token, drop
mask and the gathered rows; f is exact (same fp64 division, rounded to
fp32); aux within 1e-5 relative.
"""
import json
import os

import numpy as np
import pytest
import torch

from gpu_util import REL_ROUTE, dev, host
from mixture_experts_top_b200 import api
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def run_dispatch(T, d, E, k, cf, idx, P, x, dtype="bf16"):
    kind = "linear" if dtype == "f32" else "relu"
    cfg = api.make_config(T, d, 64, d, E, k, kind, dtype, cf)
    ws = api.alloc_workspace(cfg)
    R = T * k
    t = dict(
        counts=torch.full((E,), -1, dtype=torch.int32, device="cuda"),
        offsets=torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
        dest=torch.full((max(R, 1),), -9, dtype=torch.int32, device="cuda"),
        perm=torch.full((max(R, 1),), -5, dtype=torch.int32, device="cuda"),
        drop=torch.full((max(R, 1),), 7, dtype=torch.uint8, device="cuda"),
        f=torch.full((E,), -1.0, device="cuda"),
        aux=torch.full((1,), -1.0, device="cuda"),
        x_perm=torch.zeros((max(R, 1), d), dtype=torch.bfloat16 if dtype == "bf16" else torch.float32,
                           device="cuda"),
    )
    api.moe_dispatch(cfg, dev(x), dev(idx.astype(np.int32)), dev(P.astype(np.float32)), t["counts"],
                     t["offsets"], t["dest"], t["perm"], t["drop"], t["f"], t["aux"], t["x_perm"], ws)
    torch.cuda.synchronize()
    status = api.moe_device_status(ws)
    out = {key: host(v) for key, v in t.items()}
    out["status"] = status
    return out


def _random_routing(T, E, k, rng, skew=0.0):
    L = rng.standard_normal((T, E)).astype(np.float32)
    if skew:
        L[:, : max(1, E // 8)] += skew
    return O.top_k(L, k), O.softmax_rows(L)


def _x(T, d, rng, dtype="bf16"):
    xf = rng.standard_normal((T, d)).astype(np.float32)
    if dtype == "f32":
        return xf
    u = xf.view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def check(T, d, E, k, cf, idx, probs, x, dtype="bf16"):
    P = O.prob_mean(probs) if T > 0 else np.zeros(E)
    g = run_dispatch(T, d, E, k, cf, idx, P, x, dtype)
    o = O.dispatch(idx.reshape(T, k), E, cf)
    assert g["status"] == 0
    assert np.array_equal(g["counts"], o["counts"])
    assert np.array_equal(g["offsets"], o["offsets"])
    R = int(o["offsets"][-1])
    if T > 0:
        assert np.array_equal(g["dest"][: T * k], o["dest"].ravel())
        assert np.array_equal(g["drop"][: T * k], o["drop_mask"].ravel())
        assert np.array_equal(g["perm"][:R], o["perm_token"])
        assert (g["perm"][R:T * k] == -5).all()          # untouched beyond R
        assert np.array_equal(g["x_perm"][:R], x[o["perm_token"]])
    assert np.array_equal(g["f"], o["f"].astype(np.float32))
    aux_ref = O.aux_loss(o["f"], P.astype(np.float32).astype(np.float64)) if T > 0 else 0.0
    assert abs(float(g["aux"][0]) - aux_ref) <= REL_ROUTE * max(abs(aux_ref), 1e-30)
    return g, o


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (64, 8, 2), (255, 8, 2), (257, 8, 2), (1000, 64, 6),
                                   (4096, 64, 1), (5000, 256, 8), (3000, 7, 3), (513, 4, 4)])
@pytest.mark.parametrize("cf", [0.0, 0.5, 1.0, 1.25, 2.0])
def test_dispatch_bit_exact(T, E, k, cf):
    rng = np.random.default_rng(T * 7 + E + k)
    idx, probs = _random_routing(T, E, k, rng, skew=1.5)
    check(T, 64, E, k, cf, idx, probs, _x(T, 64, rng))


def test_dispatch_fp32_rows():
    rng = np.random.default_rng(4)
    idx, probs = _random_routing(333, 8, 2, rng)
    check(333, 32, 8, 2, 1.0, idx, probs, _x(333, 32, rng, "f32"), "f32")


def test_dispatch_wide_rows():
    """d = 4096 rows (the Mixtral width) gathered with 16-byte vectors."""
    rng = np.random.default_rng(5)
    idx, probs = _random_routing(700, 8, 2, rng)
    check(700, 4096, 8, 2, 0.0, idx, probs, _x(700, 4096, rng))


@pytest.mark.parametrize("d,dtype", [(8, "bf16"), (1024, "f32"), (1032, "f32"), (2064, "bf16"),
                                     (2056, "f32"), (6144, "bf16")])
@pytest.mark.parametrize("T", [300, 1100])
def test_dispatch_row_sizes(d, dtype, T):
    """Row sizes around the scatter's load-ahead depths (from 1024 tokens: whole
    rows of up to 4 KiB with 8 vectors a lane, else the first 8 KiB with 16 and
    the rest after; below, none): 16 bytes, exactly 4 KiB, just over 4 KiB,
    just over 8 KiB, 12 KiB."""
    rng = np.random.default_rng(d + T)
    idx, probs = _random_routing(T, 8, 2, rng)
    check(T, d, 8, 2, 1.0, idx, probs, _x(T, d, rng, dtype), dtype)


def test_dispatch_all_on_one_expert_with_capacity():
    """Collapse: every token on expert 3, capacity keeps the first cap tokens."""
    T, E, k = 1000, 8, 1
    idx = np.full((T, 1), 3, np.int32)
    probs = np.full((T, E), 1.0 / E)
    rng = np.random.default_rng(6)
    g, o = check(T, 32, E, k, 1.0, idx, probs, _x(T, 32, rng))
    assert int(g["drop"][:T].sum()) == T - 125


def test_dispatch_pfd_capacity_table(golden_dir):
    """The page's drop table, reproduced by the GPU dispatch."""
    gd = json.load(open(os.path.join(golden_dir, "pfd_capacity_table.json")))
    rng = np.random.default_rng(0)
    for router in gd["routers"].values():
        experts = np.repeat(np.arange(8), router["counts"])
        rng.shuffle(experts)
        idx = experts.reshape(64, 1).astype(np.int32)
        for factor, dropped in router["dropped"].items():
            g, _ = check(64, 32, 8, 1, float(factor), idx, np.full((64, 8), 0.125),
                         _x(64, 32, rng))
            assert int(g["drop"][:64].sum()) == dropped


def test_dispatch_empty_batch():
    g = run_dispatch(0, 64, 8, 2, 1.0, np.zeros((0, 2), np.int32), np.zeros(8), np.zeros((0, 64), np.uint16))
    assert (g["counts"] == 0).all() and (g["offsets"] == 0).all()
    assert (g["f"] == 0).all() and g["aux"][0] == 0


def test_dispatch_reports_bad_expert_index():
    """An index outside [0, E) is flagged on the device error word (the slot
    is treated as dropped); nothing faults."""
    T, E, k = 100, 8, 2
    rng = np.random.default_rng(8)
    idx, probs = _random_routing(T, E, k, rng)
    idx = idx.copy()
    idx[17, 1] = 8
    idx[40, 0] = -3
    g = run_dispatch(T, 32, E, k, 0.0, idx, O.prob_mean(probs), _x(T, 32, rng))
    assert g["status"] == 1                          # kDevBadExpertIndex
    assert g["dest"][17 * k + 1] == -1 and g["drop"][17 * k + 1] == 1
