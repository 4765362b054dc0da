"""One batch split over ranks, each rank's calls run one after another on one
GPU (no kernel waits on another rank's): moe_route and moe_dispatch_count per
block of tokens, the exchange's arithmetic on the host (shard.combine_stats,
which shard.exchange runs over a process group), then moe_dispatch_shard,
moe_expert_ffn and moe_combine per block.

The result must be the single-batch layer's (moe_forward on all tokens): the
same keep decisions with the capacity binding, the same f, the same aux on
every rank (within the 1e-5 of P summed in another order), and bit-identical
output rows.  Router inputs with exact fp32 logits (integer tokens, weights
in 1/16 steps) make the routing independent of how the router splits its
work for a given block size.
"""
import numpy as np
import pytest
import torch

from gpu_util import REL_ROUTE, cfg_of, dev, host, rel_close
from mixture_experts_top_b200 import api, shard
from mixture_experts_top_b200.layer import MoeForward
from oracle import moe_oracle as O
from workloads import WORKLOADS, make_exact_router_inputs, make_inputs

pytestmark = pytest.mark.gpu


def _inputs(w, seed):
    inp = make_inputs(w, seed=seed)
    ex = make_exact_router_inputs(w.T, w.d, w.E, w.dtype, seed=seed)
    inp["x"], inp["W_router"] = ex["x"], ex["W_router"]
    if inp["logit_bias"] is not None:       # keep the hot experts; +3.0 is exact
        inp["logit_bias"] = np.round(inp["logit_bias"] * 16) / 16
    inp["noise"] = None
    return inp


def _run_shards(w, inp, blocks):
    W = [dev(inp[key]) for key in ("W_in", "W_up", "W_out")]
    Wr, bias = dev(inp["W_router"]), dev(inp["logit_bias"])
    starts = np.concatenate([[0], np.cumsum(blocks)])
    ranks = []
    for r, n in enumerate(blocks):
        cfg = cfg_of(w, T=n)
        ws = api.alloc_workspace(cfg)
        x = dev(inp["x"][starts[r]:starts[r + 1]])
        idx = torch.empty((n, w.top_k), dtype=torch.int32, device="cuda")
        gates = torch.empty((n, w.top_k), dtype=torch.float32, device="cuda")
        P = torch.empty(w.E, dtype=torch.float32, device="cuda")
        api.moe_route(cfg, x, Wr, bias, None, idx, gates, P, None, ws)
        counts = torch.empty(w.E, dtype=torch.int32, device="cuda")
        api.moe_dispatch_count(cfg, idx, counts, ws)
        ranks.append(dict(cfg=cfg, ws=ws, x=x, idx=idx, gates=gates, P=P, counts=counts))
    torch.cuda.synchronize()
    all_counts, P, T_g = shard.combine_stats([d["counts"].cpu() for d in ranks],
                                             [d["P"].cpu() for d in ranks], blocks)
    assert T_g == w.T
    all_counts, P = all_counts.cuda().contiguous(), P.cuda()
    outs = []
    for r, d in enumerate(ranks):
        cfg, n, k = d["cfg"], blocks[r], w.top_k
        t = dict(counts=torch.empty(w.E, dtype=torch.int32, device="cuda"),
                 offsets=torch.empty(w.E + 1, dtype=torch.int32, device="cuda"),
                 dest=torch.empty((n, k), dtype=torch.int32, device="cuda"),
                 perm=torch.empty(n * k, dtype=torch.int32, device="cuda"),
                 drop=torch.empty((n, k), dtype=torch.uint8, device="cuda"),
                 f=torch.empty(w.E, dtype=torch.float32, device="cuda"),
                 aux=torch.empty(1, dtype=torch.float32, device="cuda"))
        x_perm = torch.empty((n * k, w.d), dtype=d["x"].dtype, device="cuda")
        api.moe_dispatch_shard(cfg, r, len(blocks), T_g, all_counts, d["x"], d["idx"], P,
                               t["counts"], t["offsets"], t["dest"], t["perm"], t["drop"], t["f"],
                               t["aux"], x_perm, d["ws"])
        y_perm = torch.empty((n * k, w.d_out), dtype=torch.float32, device="cuda")
        api.moe_expert_ffn(cfg, x_perm, t["offsets"], *W, y_perm, d["ws"])
        out = torch.empty((n, w.d_out), dtype=d["x"].dtype, device="cuda")
        api.moe_combine(cfg, y_perm, t["dest"], d["gates"], out)
        torch.cuda.synchronize()
        assert api.moe_device_status(d["ws"]) == 0
        res = {key: host(v) for key, v in t.items()}
        res.update(output=host(out), idx=host(d["idx"]))
        outs.append(res)
    return outs


REDUCED = {
    "fine_grained": WORKLOADS["fine_grained"].replace(T=1100, d=256, d_hidden=352, d_out=256),
    "switch_relu": WORKLOADS["switch_relu"].replace(T=1024, d=256, d_hidden=512, d_out=256,
                                                    noise=False),
    "mixtral": WORKLOADS["mixtral"].replace(T=600, d=512, d_hidden=1024, d_out=512,
                                            capacity_factor=1.0),
}


@pytest.mark.parametrize("name,blocks", [("fine_grained", [300, 500, 300]),
                                         ("switch_relu", [1, 511, 512]),
                                         ("mixtral", [200, 400])])
def test_sharded_batch_equals_single_batch(name, blocks):
    w = REDUCED[name]
    assert sum(blocks) == w.T and w.capacity_factor > 0
    inp = _inputs(w, seed=11)
    layer = MoeForward(cfg_of(w))
    full = layer(dev(inp["x"]), dev(inp["W_router"]), dev(inp["logit_bias"]), None,
                 dev(inp["W_in"]), dev(inp["W_up"]), dev(inp["W_out"]))
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    full = {key: host(getattr(full, key)) for key in ("output", "expert_indices", "drop_mask",
                                                      "counts", "aux_loss")}
    assert full["drop_mask"].any(), "the capacity must bind for this test to mean anything"
    outs = _run_shards(w, inp, blocks)

    cat = lambda key: np.concatenate([o[key] for o in outs])
    assert np.array_equal(cat("idx"), full["expert_indices"])
    assert np.array_equal(cat("drop"), full["drop_mask"])
    assert np.array_equal(sum(o["counts"] for o in outs), full["counts"])
    assert np.array_equal(cat("output").view(np.uint16), full["output"].view(np.uint16))
    for o in outs:
        assert np.array_equal(o["aux"], outs[0]["aux"])         # the same on every rank
        assert np.array_equal(o["f"], outs[0]["f"])
    assert rel_close(outs[0]["aux"], full["aux_loss"], REL_ROUTE)
    # and the oracle's single-batch routing
    o = O.dispatch(full["expert_indices"], w.E, w.capacity_factor)
    assert np.array_equal(cat("drop"), o["drop_mask"])
    assert rel_close(outs[0]["f"], o["f"], 1e-6)


def test_shard_with_wrong_counts_is_reported():
    w = REDUCED["mixtral"]
    inp = _inputs(w, seed=3)
    cfg = cfg_of(w, T=300)
    ws = api.alloc_workspace(cfg)
    x = dev(inp["x"][:300])
    idx = torch.empty((300, 2), dtype=torch.int32, device="cuda")
    g = torch.empty((300, 2), dtype=torch.float32, device="cuda")
    P = torch.empty(w.E, dtype=torch.float32, device="cuda")
    api.moe_route(cfg, x, dev(inp["W_router"]), None, None, idx, g, P, None, ws)
    wrong = torch.zeros((2, w.E), dtype=torch.int32, device="cuda")   # rank 0's row is not its counts
    E = w.E
    t = [torch.empty(E, dtype=torch.int32, device="cuda"),
         torch.empty(E + 1, dtype=torch.int32, device="cuda"),
         torch.empty((300, 2), dtype=torch.int32, device="cuda"),
         torch.empty(600, dtype=torch.int32, device="cuda"),
         torch.empty((300, 2), dtype=torch.uint8, device="cuda"),
         torch.empty(E, dtype=torch.float32, device="cuda"),
         torch.empty(1, dtype=torch.float32, device="cuda")]
    api.moe_dispatch_shard(cfg, 0, 2, 600, wrong, x, idx, P, *t,
                           torch.empty((600, w.d), dtype=torch.bfloat16, device="cuda"), ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 4
