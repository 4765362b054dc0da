"""One batch split over ranks, each rank's calls run one after another on one
GPU (no kernel waits on another rank's): shard.ShardStep per block of tokens
-- moe_route and moe_shard_record, the all-gather of the records (here the
records stacked in rank order, a stand-in for the collective used only in
this test), then moe_dispatch_shard and moe_expert_ffn_combine.

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
    steps, xs = [], []
    for r, n in enumerate(blocks):
        st = shard.ShardStep(cfg_of(w, T=n), r, len(blocks), w.T)
        x = dev(inp["x"][starts[r]:starts[r + 1]])
        st.route(x, Wr, bias, None)
        steps.append(st)
        xs.append(x)
    records = torch.stack([st.record for st in steps])
    c, p, t = shard.unpack_records(host(records))
    assert t.tolist() == list(blocks)
    outs = []
    for st, x in zip(steps, xs):
        st.exchange(gather=lambda rec, out: out.copy_(records))
        st.finish(x, *W)
        torch.cuda.synchronize()
        assert st.device_status() == 0
        o = st.out
        outs.append(dict(counts=host(o.counts), offsets=host(st.offsets), dest=host(st.dest),
                         perm=host(st.perm), drop=host(o.drop_mask), f=host(st.f),
                         aux=host(o.aux_loss), output=host(o.output), idx=host(o.expert_indices)))
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


def test_shard_record_layout():
    """moe_shard_record: counts per expert, then moe_route's P as fp32 bits,
    then T."""
    w = REDUCED["fine_grained"]
    inp = _inputs(w, seed=5)
    cfg = cfg_of(w)
    st = shard.ShardStep(cfg, 0, 1, w.T)
    st.route(dev(inp["x"]), dev(inp["W_router"]), dev(inp["logit_bias"]), None)
    torch.cuda.synchronize()
    c, p, t = shard.unpack_records(host(st.record)[None, :])
    idx = host(st.out.expert_indices)
    assert np.array_equal(c[0], np.bincount(idx.ravel(), minlength=w.E))
    assert np.array_equal(p[0], host(st.P)) and t[0] == w.T


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
    E = w.E
    wrong = torch.zeros((2, 2 * E + 1), dtype=torch.int32, device="cuda")
    wrong[:, 2 * E] = 300                 # token counts add up; rank 0's counts are not its own
    t = [torch.empty(E, dtype=torch.int32, device="cuda"),
         torch.empty(E + 1, dtype=torch.int32, device="cuda"),
         torch.empty((300, 2), dtype=torch.int32, device="cuda"),
         torch.empty(600, dtype=torch.int32, device="cuda"),
         torch.empty((300, 2), dtype=torch.uint8, device="cuda"),
         torch.empty(E, dtype=torch.float32, device="cuda"),
         torch.empty(1, dtype=torch.float32, device="cuda")]
    api.moe_dispatch_shard(cfg, 0, 2, 600, wrong, x, idx, None, *t,
                           torch.empty((600, w.d), dtype=torch.bfloat16, device="cuda"), ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 4
    # records whose token counts do not add up to T_global
    right = torch.zeros((2, 2 * E + 1), dtype=torch.int32, device="cuda")
    api.moe_shard_record(cfg, idx, P, right[0], ws)
    right[1, 2 * E] = 299
    api.moe_dispatch_shard(cfg, 0, 2, 600, right, x, idx, None, *t,
                           torch.empty((600, w.d), dtype=torch.bfloat16, device="cuda"), ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == 4
