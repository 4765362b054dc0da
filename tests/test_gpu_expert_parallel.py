"""Expert parallelism on one GPU, every rank played in turn by this process
(no kernel waits on another rank's): each rank routes and dispatches its own
tokens (ep_dispatch), the rows bound for each rank's experts are handed over
as the all-to-all would (contiguous slices in source order, a stand-in for
NCCL used only here), each rank runs its experts on its own weight slice
(ep_experts), the rows go back and each rank combines (ep_combine).

Every rank's output must be bit-identical to moe_forward on its tokens with
all E experts on one GPU: the same kept rows meet the same weights."""
import numpy as np
import pytest
import torch

from gpu_util import (REL_F32, ambiguous_tokens, bf16_to_f64, cfg_of, dev, host,
                      layer_tolerance)
from mixture_experts_top_b200 import api
from mixture_experts_top_b200 import expert_parallel as ep
from mixture_experts_top_b200.layer import MoeForward
from oracle import moe_oracle as O
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "mixtral": WORKLOADS["mixtral"].replace(T=400, d=256, d_hidden=512, d_out=256),
    "fine_grained": WORKLOADS["fine_grained"].replace(T=500, d=256, d_hidden=352, d_out=256),
    "tiny_linear": WORKLOADS["tiny_linear"],
}


@pytest.mark.parametrize("name,world", [("mixtral", 2), ("mixtral", 3), ("fine_grained", 4),
                                        ("fine_grained", 3), ("tiny_linear", 2)])
def test_expert_parallel_equals_single_gpu(name, world):
    w = CASES[name]
    ranges = ep.plan(w.E, world)
    W = make_inputs(w, seed=0)                              # replicated router, split experts
    Wd = {key: dev(W[key]) for key in ("W_router", "logit_bias", "W_in", "W_up", "W_out")}
    ranks = []
    for s in range(world):
        inp = make_inputs(w, seed=100 + s, with_experts=False)     # each rank its own tokens
        cfg = cfg_of(w)
        ws = api.alloc_workspace(cfg)
        x = dev(inp["x"])
        st = ep.ep_dispatch(cfg, x, Wd["W_router"], Wd["logit_bias"], dev(inp["noise"]), ws, world)
        ranks.append(dict(cfg=cfg, ws=ws, x=x, noise=dev(inp["noise"]), st=st, inp=inp))
    # the first all-to-all
    for r, (lo, hi) in enumerate(ranges):
        slices = [d["st"].sends[r] for d in ranks]
        x_recv = torch.cat([d["st"].x_perm[a:b] for d, (a, b, _) in zip(ranks, slices)])
        y_recv = torch.empty((x_recv.shape[0], w.d_out), dtype=torch.float32, device="cuda")
        lws = ep.ep_experts(ranks[0]["cfg"], hi - lo, x_recv, [c for _, _, c in slices],
                            Wd["W_in"][lo:hi], None if Wd["W_up"] is None else Wd["W_up"][lo:hi],
                            None if Wd["W_out"] is None else Wd["W_out"][lo:hi], y_recv)
        # the second all-to-all
        pos = 0
        for d, (a, b, _) in zip(ranks, slices):
            d["st"].y_perm[a:b] = y_recv[pos:pos + (b - a)]
            pos += b - a
        torch.cuda.synchronize()
        assert api.moe_device_status(lws) == 0
    for d in ranks:
        out = torch.empty((w.T, w.d_out), dtype=d["x"].dtype, device="cuda")
        got = ep.ep_combine(d["cfg"], d["st"], out)
        layer = MoeForward(d["cfg"])
        ref = layer(d["x"], Wd["W_router"], Wd["logit_bias"], d["noise"], Wd["W_in"], Wd["W_up"],
                    Wd["W_out"])
        torch.cuda.synchronize()
        assert layer.device_status() == 0 and api.moe_device_status(d["ws"]) == 0
        for key in ("expert_indices", "drop_mask", "counts", "aux_loss"):
            assert np.array_equal(host(got[key]), host(getattr(ref, key))), key
        g, r = host(got["output"]), host(ref.output)
        assert np.array_equal(g.view(np.uint16) if g.dtype == np.uint16 else g,
                              r.view(np.uint16) if r.dtype == np.uint16 else r)
        # and the oracle's layer on this rank's tokens
        weights = {key: W[key] for key in ("W_in", "W_up", "W_out")}
        o = O.moe_forward(d["inp"]["x"], W["W_router"], weights, top_k=w.top_k, kind=w.kind,
                          dtype=w.dtype, d_out=w.d_out, capacity_factor=w.capacity_factor,
                          logit_bias=W["logit_bias"], noise=d["inp"]["noise"])
        ok = ~ambiguous_tokens(o["logits"], w.top_k)
        assert ok.mean() > 0.99
        # a flipped near-tie may move later drops: compare where they agree
        ok &= (host(got["drop_mask"]) == o["drop_mask"]).all(axis=1)
        assert ok.mean() > 0.95
        assert np.array_equal(host(got["expert_indices"])[ok], o["expert_indices"][ok])
        if w.dtype == "f32":
            assert np.abs(g[ok] - o["output"][ok]).max() <= REL_F32 * np.abs(o["output"]).max()
        else:
            rms = float(np.sqrt(np.mean(o["Y"] ** 2)))
            err = np.abs(bf16_to_f64(g[ok]) - o["output"][ok])
            assert np.all(err <= layer_tolerance(o["output"][ok], rms))
