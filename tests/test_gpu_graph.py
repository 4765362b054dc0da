"""The layer captured as a CUDA graph and replayed.

Every kernel is launched as a programmatic dependent of the one before it,
some as thread-block clusters, and the pair GEMM, the router and the
dispatch keep counters in the workspace that the last CTA of each launch
puts back to 0; a captured step must therefore replay any number of times
and give the eager call's bits.  Checked on reduced Mixtral (top-2, pair
GEMM), Switch (top-1, combine fused in the down projection, noise), fine-grained
(E = 64, capacity) and a top-2 shape whose combine runs in the down
projection's epilogue: one eager call, then the captured
call replayed on the same inputs and again on new tokens copied into the
graph's input buffer, each replay against an eager call on those tokens.
"""
import numpy as np
import pytest
import torch

from gpu_util import cfg_of, dev, host
from mixture_experts_top_b200.layer import MoeForward
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "mixtral": WORKLOADS["mixtral"].replace(T=4096, d=512, d_hidden=1024, d_out=512),
    "switch_relu": WORKLOADS["switch_relu"].replace(T=1024, d=256, d_hidden=512, d_out=256),
    "fine_grained": WORKLOADS["fine_grained"].replace(T=1100, d=256, d_hidden=352, d_out=256),
    # top-2 combine in the down projection's epilogue: its arrival counters,
    # zeroed by the up projection, must be back at 0 for every replay
    "mixtral_fused_combine": WORKLOADS["mixtral"].replace(T=2048, d=256, d_hidden=4096,
                                                          d_out=256, E=4),
}
KEYS = ("output", "expert_indices", "gates", "aux_loss", "counts", "drop_mask")


def snapshot(o):
    return {k: host(getattr(o, k)).copy() for k in KEYS}


@pytest.mark.parametrize("name", list(CASES))
def test_captured_forward_replays_bit_exact(name):
    w = CASES[name]
    inp = make_inputs(w, seed=3)
    inp2 = make_inputs(w, seed=4, with_experts=False)
    W = {k: dev(inp[k]) for k in ("W_router", "logit_bias", "W_in", "W_up", "W_out")}
    x = dev(inp["x"])
    noise = dev(inp["noise"])
    x2, noise2 = dev(inp2["x"]), dev(inp2["noise"])

    eager = MoeForward(cfg_of(w))
    args = lambda xx, nn: (xx, W["W_router"], W["logit_bias"], nn, W["W_in"], W["W_up"], W["W_out"])
    ref1 = snapshot(eager(*args(x, noise)))
    torch.cuda.synchronize()
    ref2 = snapshot(eager(*args(x2, noise2)))
    torch.cuda.synchronize()
    assert eager.device_status() == 0

    layer = MoeForward(cfg_of(w))
    x_in = x.clone()
    n_in = None if noise is None else noise.clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        layer(*args(x_in, n_in))          # warm up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer(*args(x_in, n_in))
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    got1 = snapshot(layer.out)
    x_in.copy_(x2)
    if n_in is not None:
        n_in.copy_(noise2)
    g.replay()
    torch.cuda.synchronize()
    got2 = snapshot(layer.out)
    assert layer.device_status() == 0
    # the workspace's counters are back at 0 after the replays
    ctrl = host(layer.ws[:256]).view(np.uint32)
    assert (ctrl[1:] == 0).all(), ctrl[ctrl != 0]
    for ref, got in ((ref1, got1), (ref2, got2)):
        for k in KEYS:
            assert np.array_equal(ref[k], got[k]), k
    assert not np.array_equal(got1["output"], got2["output"])


def test_captured_expert_backward_replays_bit_exact():
    """The experts' backward (CTA-pair GEMMs, TMA-stored weight gradients)
    captured and replayed gives the eager call's bits."""
    from mixture_experts_top_b200 import api
    w = CASES["mixtral"].replace(T=1024)
    inp = make_inputs(w, seed=5)
    cfg = cfg_of(w)
    E, R = w.E, w.T * w.top_k
    rng = np.random.default_rng(6)
    counts = rng.multinomial(R - 40, np.full(E, 1.0 / E))
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32,
                           device="cuda")
    x_perm = dev(inp["x"].repeat(w.top_k, axis=0))
    dy = torch.from_numpy(rng.standard_normal((R, w.d_out)).astype(np.float32)).cuda()
    W = {key: dev(inp[key]) for key in ("W_in", "W_up", "W_out")}
    f32 = dict(dtype=torch.float32, device="cuda")

    def grads():
        return [torch.zeros((R, w.d), **f32), torch.zeros((E, w.d, w.d_hidden), **f32),
                torch.zeros((E, w.d, w.d_hidden), **f32), torch.zeros((E, w.d_hidden, w.d_out), **f32)]

    def run(out, bws):
        api.moe_expert_ffn_backward(cfg, x_perm, offsets, W["W_in"], W["W_up"], W["W_out"], dy,
                                    *out, bws)

    ref, bws0 = grads(), api.alloc_backward_workspace(cfg)
    run(ref, bws0)
    torch.cuda.synchronize()
    got, bws = grads(), api.alloc_backward_workspace(cfg)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run(got, bws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for t in got:
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run(got, bws)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert api.moe_device_status(bws) == 0
    for a, b in zip(ref, got):
        assert np.array_equal(host(a), host(b))
