#!/usr/bin/env python3
"""Benchmark of the MoE layer forward pass on B200 GPUs.

One step = one pass of the whole hot path (route -> dispatch -> experts ->
combine, aux loss included) over one batch of the Mixtral-shaped workload
(T=8192 tokens, D=4096, DH=14336, E=8, top-2 SwiGLU experts, bf16, fp32
router), synthetic seeded inputs, random-init weights of that shape.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (launched by torch.distributed.run): one batch of N x T tokens is
split over the ranks in contiguous blocks (weak scaling: T tokens per GPU);
every step all-gathers each rank's exchange record (2E+1 ints: slot counts,
probability means, token count) over NCCL, from which each rank's sharded
dispatch takes the batch's capacity positions, f and P; the step time is the
max over ranks; value = tokens of all ranks / that time.

At N=1 the line's `extras.workloads` adds the other configurations (decode,
fine-grained, Switch top-1, the small linear case), each timed the same way
after the main timed region.

The reference arm (--impl reference) times the CPU oracle, as it stands, on
the host cores (rank 0 only), one token of the workload per step, run as a
batch of its own (so each step also widens that token's two experts' bf16
weights to fp64).
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_top_b200 import accounting as A  # noqa: E402  (pure-Python counts)

METRIC = "MoE layer tokens/s at 1 B200 (Mixtral-shape bf16); GEMM % tensor peak, route GB/s"
WORKLOAD = "mixtral"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid):
        self.proc = None
        self.uuid = gpu_uuid

    def start(self):
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except (OSError, ValueError):
            self.proc = None
        self.t0 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i]
                          and "Not" not in r[5 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- profiles --

def profiled_traffic(kernel_file: str, summary: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the kernel source as it is now (sha256 recorded in the summary)."""
    path = os.path.join(ROOT, "profiles", summary)
    src = os.path.join(ROOT, "mixture_experts_top_b200", "csrc", kernel_file)
    if not (os.path.exists(path) and os.path.exists(src)):
        return None
    text = open(path).read()
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not (m_sha and m_b):
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != m_sha.group(1):
        return None
    return float(m_b.group(1))


def fused_combine(w) -> bool:
    """The form moe_forward uses: the combine in the down projection's
    epilogue (moe_expert_ffn_combine, no combine kernel), or moe_expert_ffn
    then moe_combine."""
    from mixture_experts_top_b200 import api as _api
    return _api.moe_forward_combine_fused(_api.make_config(
        w.T, w.d, w.d_hidden, w.d_out, w.E, w.top_k, w.kind, w.dtype, w.capacity_factor))


def launches_per_step(w, cfg, world: int = 1) -> int:
    """Kernels of this library launched by one timed step (route, dispatch,
    experts, combine), as the library picks them for this configuration:
    route = weight split + tensor-core router (its last tile writes P; bf16,
    E <= 64) or SIMT router + P mean; dispatch = count (its last CTA runs
    the scan) + scatter; experts = up and
    down GEMM (bf16) or the fp32 linear kernel; combine = 1, or 0 where it is
    fused into the down projection.  A rank of a split batch adds
    its exchange record (count + total)."""
    from mixture_experts_top_b200 import api as _api
    if w.T == 0:
        return 2                       # P mean and the dispatch scan only
    route = 2
    experts = 1 if w.kind == "linear" else 2
    record = 2 if world > 1 else 0
    return route + record + 2 + experts + (0 if fused_combine(w) else 1)


# ------------------------------------------------------------- ranks (N>1) --

def rank_token_seed(rank: int) -> int:
    """Seed of a rank's token batch: rank 0 uses the workload's own batch,
    other ranks independent batches; the weights (seed 0) are replicated."""
    return 0 if rank == 0 else 1000 + rank


def max_over_ranks(values, world: int, device="cpu"):
    """Element-wise max over ranks of a list of floats (the step time of the
    slowest rank decides)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def job_value(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# ---------------------------------------------------------- reference arm --

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_token_steps(w, inp, tokens):
    """Times the CPU oracle's full forward on single-token batches."""
    from oracle import moe_oracle as O
    weights = {k: inp[k] for k in ("W_in", "W_up", "W_out")}
    times = []
    for t in tokens:
        t0 = time.perf_counter()
        O.moe_forward(inp["x"][t:t + 1], inp["W_router"], weights, top_k=w.top_k, kind=w.kind,
                      dtype=w.dtype, d_out=w.d_out, capacity_factor=w.capacity_factor,
                      logit_bias=inp["logit_bias"],
                      noise=None if inp["noise"] is None else inp["noise"][t:t + 1])
        times.append(time.perf_counter() - t0)
    return times


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    from workloads import WORKLOADS, make_inputs
    w = WORKLOADS[args.workload]
    inp = make_inputs(w, seed=0)
    oracle_token_steps(w, inp, list(range(args.warmup)))
    tokens = [(args.warmup + i) % w.T for i in range(args.steps)]
    times = oracle_token_steps(w, inp, tokens)
    total = sum(times)
    value = len(tokens) / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(tokens), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle",
                         "sample": "one token of the batch per step, run as a batch of its own "
                                   "through the full oracle forward in fp64 (each step widens "
                                   "its experts' bf16 weights to fp64, which dominates)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


WORKLOAD_TITLES = {
    "mixtral": "Mixtral-shaped SwiGLU MoE layer",
    "decode": "Mixtral-shaped SwiGLU MoE layer, decode-sized batch",
    "fine_grained": "fine-grained SwiGLU MoE layer with four hot experts",
    "switch_relu": "Switch-style top-1 ReLU-MLP MoE layer with a noisy gate",
    "tiny_linear": "small linear-expert MoE layer",
}


def describe(w) -> str:
    """One-line description of a workload, from its own fields."""
    expert = {"linear": f"linear experts (d_out={w.d_out})",
              "relu": f"ReLU-MLP experts (DH={w.d_hidden})",
              "swiglu": f"SwiGLU experts (DH={w.d_hidden})"}[w.kind]
    cap = (f"capacity factor {w.capacity_factor:g} (ceil(cf*T*k/E) = "
           f"{A.capacity_slots(w.capacity_factor, w.T, w.top_k, w.E)} slots per expert)"
           if w.capacity_factor > 0 else "no capacity limit")
    prec = ("bf16 tokens and weights, fp32 router and accumulation" if w.dtype == "bf16"
            else "fp32 throughout")
    extras = []
    if w.n_hot:
        extras.append(f"+{w.hot_bias:g} logit bias on {w.n_hot} seeded experts")
    if w.noise:
        extras.append("noise z*softplus(x@W_noise) made on the host")
    return (f"{w.name}: {WORKLOAD_TITLES.get(w.name, 'MoE layer')}, T={w.T} tokens per GPU, "
            f"d={w.d}, E={w.E}, top_k={w.top_k}, {expert}, {cap}, {prec}"
            + ("; " + "; ".join(extras) if extras else ""))


def l2_note(w) -> str:
    nb = A.expert_weight_bytes(w.E, w.d, w.d_hidden, w.d_out, w.kind,
                               2 if w.dtype == "bf16" else 4)
    if nb > 126e6:
        return (f"no flush: each step streams {nb / 1e9:.2f} GB of expert weights "
                "(> 126 MB L2)")
    return f"no flush: the whole layer ({nb / 1e3:.0f} KB of weights) stays in L2"


def workload_config(w, n):
    par = ("dp1" if n == 1 else
           f"dp{n}: one batch of {n} x {w.T} tokens split over the ranks in contiguous blocks, "
           "replicated weights; per step one NCCL all-gather of each rank's 2E+1-int exchange "
           "record (slot counts, probability means, tokens) couples the capacity and the aux loss")
    return {"workload": describe(w),
            "T": w.T, "d": w.d, "d_hidden": w.d_hidden, "d_out": w.d_out, "E": w.E,
            "top_k": w.top_k, "capacity_factor": w.capacity_factor,
            "global_batch": w.T * n,
            "parallelism": par,
            "l2": l2_note(w)}


# ---------------------------------------------------------------- our arm --

def to_device(inp):
    import numpy as np
    import torch

    def dev(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return {k: dev(v) for k, v in inp.items()}


class LayerBench:
    """Buffers and timed loops of one workload on this GPU: the staged step
    (moe_route, moe_dispatch, moe_expert_ffn, moe_combine with device
    inputs) and the end-to-end step (moe_forward with host copies)."""

    def __init__(self, w, D, shard=None):
        """shard = (rank, world, group): this rank's block of one batch of
        world * T tokens, with the exchange of the ranks' records per step."""
        import torch
        from mixture_experts_top_b200 import api
        from mixture_experts_top_b200 import shard as S
        from mixture_experts_top_b200.layer import MoeForward
        self.w, self.D, self.shard = w, D, shard
        self.cfg = api.make_config(w.T, w.d, w.d_hidden, w.d_out, w.E, w.top_k, w.kind, w.dtype,
                                   w.capacity_factor)
        self.layer = MoeForward(self.cfg)
        T, k, E = w.T, w.top_k, w.E
        R = T * k
        i32 = dict(dtype=torch.int32, device="cuda")
        act = D["x"].dtype
        self.P = torch.empty(E, dtype=torch.float32, device="cuda")
        self.offsets = torch.empty(E + 1, **i32)
        self.dest = torch.empty(R, **i32)
        self.perm = torch.empty(R, **i32)
        self.f = torch.empty(E, dtype=torch.float32, device="cuda")
        self.x_perm = torch.empty((R, w.d), dtype=act, device="cuda")
        self.y_perm = torch.empty((R, w.d_out), dtype=torch.float32, device="cuda")
        self.stream = torch.cuda.current_stream()
        self.fused_combine = fused_combine(w)
        if shard is not None:
            self.record = torch.empty(S.record_ints(E), **i32)
            self.records = torch.empty((shard[1], S.record_ints(E)), **i32)

    def step(self, ev=None, marks=(0, 1, 2, 3, 4), x=None, noise=None, out=None, aux=None):
        """One pass of the hot path (x, noise, out, aux: other buffers than
        the bench's own, for the end-to-end loop).  ev[j] is recorded before stage j
        (route, dispatch, experts, combine) and ev[4] after the last, for
        the stage indices in `marks`.  Every recorded event separates two
        launches that could otherwise overlap (each kernel is launched as a
        programmatic dependent of the one before), so timed loops mark only
        the expert stage."""
        from mixture_experts_top_b200 import api
        D, o, cfg, s = self.D, self.layer.out, self.cfg, self.stream

        def mark(j):
            if ev is not None and j in marks:
                ev[j].record(s)
        mark(0)
        x = D["x"] if x is None else x
        noise = D["noise"] if noise is None else noise
        out = o.output if out is None else out
        aux = o.aux_loss if aux is None else aux
        api.moe_route(cfg, x, D["W_router"], D["logit_bias"], noise, o.expert_indices,
                      o.gates, self.P, None, self.layer.ws)
        if self.shard is not None:
            # this rank's record, all-gathered (NCCL) in rank order
            from mixture_experts_top_b200 import shard as S
            rank, world, group = self.shard
            api.moe_shard_record(cfg, o.expert_indices, self.P, self.record, self.layer.ws)
            S.gather_records(self.record, self.records, group)
        mark(1)
        if self.shard is not None:
            rank, world, _ = self.shard
            api.moe_dispatch_shard(cfg, rank, world, world * self.w.T, self.records, x,
                                   o.expert_indices, None, o.counts, self.offsets, self.dest,
                                   self.perm, o.drop_mask, self.f, aux, self.x_perm,
                                   self.layer.ws)
        else:
            api.moe_dispatch(cfg, x, o.expert_indices, self.P, o.counts, self.offsets,
                             self.dest, self.perm, o.drop_mask, self.f, aux, self.x_perm,
                             self.layer.ws)
        mark(2)
        if self.fused_combine:
            # the combine is the down projection's epilogue
            api.moe_expert_ffn_combine(cfg, self.x_perm, self.offsets, self.perm, self.dest,
                                       o.gates, D["W_in"], D["W_up"], D["W_out"], out,
                                       self.layer.ws)
            mark(3)
        else:
            api.moe_expert_ffn(cfg, self.x_perm, self.offsets, D["W_in"], D["W_up"], D["W_out"],
                               self.y_perm, self.layer.ws)
            mark(3)
            api.moe_combine(cfg, self.y_perm, self.dest, o.gates, out)
        mark(4)

    def timed(self, steps, warmup, barrier, clocks=None):
        """Device-timed loop: returns (ms for all steps, mean experts ms)."""
        import torch
        for _ in range(warmup):
            self.step()
        barrier()
        if clocks is not None:
            clocks.start()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
        barrier()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(self.stream)
        for i in range(steps):
            self.step(evs[i], marks=(2, 3))
        end.record(self.stream)
        barrier()
        self._evs = evs
        return start.elapsed_time(end), sum(e[2].elapsed_time(e[3]) for e in evs) / steps

    def graph_timed(self, steps, warmup):
        """The same step captured once as a CUDA graph and replayed `steps`
        times (the host enqueues one graph instead of each launch, which is
        what bounds the small configurations): device ms for all steps, or
        (None, reason) where the capture is refused."""
        import torch
        try:
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                self.step()
            torch.cuda.current_stream().wait_stream(side)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.step()
            for _ in range(warmup):
                g.replay()
            torch.cuda.synchronize()
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            start.record()
            for _ in range(steps):
                g.replay()
            end.record()
            torch.cuda.synchronize()
            del g
            return start.elapsed_time(end), None
        except Exception as exc:   # reported in the line, not raised
            torch.cuda.synchronize()
            return None, f"{type(exc).__name__}: {exc}"[:200]

    def stage_breakdown(self, steps, barrier):
        """The same steps again with an event between every two stages
        (diagnostic, outside the timed region): mean ms per stage."""
        evs = self._evs
        for i in range(steps):
            self.step(evs[i])
        barrier()
        return [sum(e[j].elapsed_time(e[j + 1]) for e in evs) / steps for j in range(4)]

    def e2e(self, steps, warmup, barrier):
        """End to end through the public call (moe_forward): every step
        copies its tokens (and noise) from pinned host memory and its output
        and aux_loss back to pinned host memory, on copy streams, double
        buffered, so step i's upload and step i-1's download overlap step
        i's compute.  Returns (ms for all steps, h2d bytes, d2h bytes)."""
        import torch
        from mixture_experts_top_b200 import api
        D, o, cfg, stream = self.D, self.layer.out, self.cfg, self.stream
        x, noise = D["x"], D["noise"]
        x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True).copy_(x)
        n_host = None if noise is None else torch.empty(noise.shape, dtype=noise.dtype,
                                                        pin_memory=True).copy_(noise)
        h2d = x.numel() * x.element_size() + (0 if noise is None else noise.numel() * 4)
        d2h = o.output.numel() * o.output.element_size() + 4
        s_up, s_dn = torch.cuda.Stream(), torch.cuda.Stream()
        bufs = []
        for _ in range(2):
            bufs.append(dict(
                x=torch.empty_like(x), noise=None if noise is None else torch.empty_like(noise),
                out=torch.empty_like(o.output), aux=torch.empty_like(o.aux_loss),
                out_host=torch.empty(o.output.shape, dtype=o.output.dtype, pin_memory=True),
                aux_host=torch.empty(1, dtype=torch.float32, pin_memory=True),
                uploaded=torch.cuda.Event(), computed=torch.cuda.Event(),
                downloaded=torch.cuda.Event()))
        self.ws_e2e = api.alloc_workspace(cfg)

        def run(n):
            for i in range(n):
                b = bufs[i % 2]
                with torch.cuda.stream(s_up):
                    s_up.wait_event(b["computed"])   # step i-2 finished reading b["x"]
                    b["x"].copy_(x_host, non_blocking=True)
                    if noise is not None:
                        b["noise"].copy_(n_host, non_blocking=True)
                    b["uploaded"].record(s_up)
                stream.wait_event(b["uploaded"])
                stream.wait_event(b["downloaded"])   # step i-2's output was copied out
                if self.shard is not None:
                    # a rank of a split batch: its public calls in order
                    self.step(x=b["x"], noise=b["noise"], out=b["out"], aux=b["aux"])
                else:
                    api.moe_forward(cfg, b["x"], D["W_router"], D["logit_bias"], b["noise"],
                                    D["W_in"], D["W_up"], D["W_out"], b["out"],
                                    o.expert_indices, o.gates, b["aux"], None, None,
                                    self.ws_e2e)
                b["computed"].record(stream)
                with torch.cuda.stream(s_dn):
                    s_dn.wait_event(b["computed"])
                    b["out_host"].copy_(b["out"], non_blocking=True)
                    b["aux_host"].copy_(b["aux"], non_blocking=True)
                    b["downloaded"].record(s_dn)

        run(warmup)
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        s_up.wait_stream(stream)                     # the first upload starts after s2
        run(steps)
        stream.wait_stream(s_dn)
        e2.record(stream)
        barrier()
        return s2.elapsed_time(e2), h2d, d2h

    def device_status(self):
        from mixture_experts_top_b200 import api
        st = self.layer.device_status()
        if st == 0 and getattr(self, "ws_e2e", None) is not None:
            st = api.moe_device_status(self.ws_e2e)
        return st


def gemm_roofline(w, rows, used, expert_ms, peaks, peak_src, regime):
    """The expert GEMMs (both launches) against their binding roofline.
    Algorithmic work: 2 FLOP per multiply-add of the kept rows; where
    streaming the used experts' weights takes longer than the FLOPs take on
    the tensor cores, the bound is HBM and the algorithmic bytes are the
    used experts' weights + rows in + the hidden activation written and
    read + fp32 rows out.  `regime` picks the tensor peak: "burst" (cuBLAS
    timed alone; a timed region well under a second) or "sustained" (cuBLAS
    back to back for seconds under the power cap)."""
    flops = A.expert_gemm_flops(rows, w.d, w.d_hidden, w.d_out, w.kind)
    t = expert_ms / 1e3
    burst = peaks["bf16_tflops"]
    sustained = peaks.get("bf16_tflops_sustained") or burst
    tensor_peak = burst if regime == "burst" else sustained
    if w.kind == "linear":
        # fp32 SIMT kernel: its peak is the fp32 FMA rate, not the tensor cores
        tensor_peak = burst = sustained = None
    hbm = peaks["hbm_gbs"]
    elem = 4 if w.kind == "linear" else 2
    # rows out: fp32 expert rows (kept for the combine), then with the combine
    # in the epilogue every token's bf16 output row; at top-1 only the latter
    out_bytes = rows * w.d_out * 4 if w.top_k > 1 or not fused_combine(w) else 0
    if fused_combine(w):
        out_bytes += w.T * w.d_out * 2
    gemm_bytes = (A.expert_weight_bytes(used, w.d, w.d_hidden, w.d_out, w.kind, elem)
                  + rows * w.d * elem + out_bytes
                  + (0 if w.kind == "linear" else 2 * rows * w.d_hidden * 2))
    tensor_bound = tensor_peak is not None and \
        flops / (tensor_peak * 1e12) >= gemm_bytes / (hbm * 1e9)
    if tensor_bound:
        ach = flops / t / 1e12
        g = {"bound": "tensor", "achieved": ach, "peak": tensor_peak, "unit": "TFLOP/s",
             "frac": ach / tensor_peak, "frac_of_burst": ach / burst,
             "frac_of_sustained": ach / sustained, "regime": regime,
             "peak_source": f"{peak_src} {regime} bf16 (cuBLAS)"}
    else:
        ach = gemm_bytes / t / 1e9
        g = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
             "peak_source": f"{peak_src} HBM copy bandwidth"}
    g.update({"algorithmic_bytes": gemm_bytes, "algorithmic_flops": flops, "ms": expert_ms})
    return g


def stage_rooflines(w, rows, stage_ms, hbm):
    elem = 2 if w.dtype == "bf16" else 4
    rb = A.router_bytes(w.T, w.d, w.E, w.top_k, elem, w.noise)
    pb = A.permute_bytes(w.T, rows, w.d, elem)
    cb = A.combine_bytes(w.T, rows, w.d_out, w.top_k, elem)
    out = {}
    for name, ms, nb in (("route", stage_ms[0], rb), ("dispatch", stage_ms[1], pb),
                         ("combine", stage_ms[3], cb)):
        if name == "combine" and fused_combine(w):
            out[name] = {"fused": "in the down projection's epilogue (no kernel)"}
            continue
        out[name] = {"ms": ms, "GB/s": nb / ms / 1e6, "frac_hbm": nb / ms / 1e6 / hbm,
                     "algorithmic_bytes": nb}
    return out


def regime_of(timed_s: float) -> str:
    """A timed region under two seconds runs at burst clocks (cuBLAS timed
    alone is the matching peak); longer ones settle under the power cap."""
    return "burst" if timed_s < 2.0 else "sustained"


def extra_workload(name, steps, warmup, peaks, peak_src, base_inputs=None):
    """tokens/s (device and end to end) and each stage's roofline fraction
    of another configuration, on this GPU, outside the main timed region."""
    import torch
    from workloads import WORKLOADS, make_inputs
    w = WORKLOADS[name]
    t0 = time.time()
    if base_inputs is not None:
        # the decode batch: the Mixtral-shaped weights (same seed, same shapes)
        inp = make_inputs(w, seed=0, with_experts=False)
        D = to_device(inp)
        D.update({k: base_inputs[k] for k in ("W_in", "W_up", "W_out")})
    else:
        D = to_device(make_inputs(w, seed=0))
    gen_s = time.time() - t0
    lb = LayerBench(w, D)
    sync = torch.cuda.synchronize
    ms, expert_ms = lb.timed(steps, warmup, sync)
    stage_ms = lb.stage_breakdown(steps, sync)
    stage_ms[2] = expert_ms
    e2e_ms, h2d, d2h = lb.e2e(steps, warmup, sync)
    graph_ms, graph_err = lb.graph_timed(steps, warmup)
    if lb.device_status() != 0:
        raise RuntimeError(f"{name}: device error word set")
    counts = lb.layer.out.counts.cpu().numpy()
    rows = A.kept_rows(counts, w.capacity_factor, w.T, w.top_k)
    used = int((counts > 0).sum())
    regime = regime_of(ms / 1e3)
    noisy = route_noisy_timing(w, lb, peaks) if w.noise else None
    res = {
        "workload": describe(w), "tokens_per_s": w.T / (ms / steps / 1e3),
        "ms_per_step": ms / steps,
        "e2e_tokens_per_s": w.T / (e2e_ms / steps / 1e3),
        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
        "graph": ({"tokens_per_s": w.T / (graph_ms / steps / 1e3), "ms_per_step": graph_ms / steps,
                   "note": "the same step captured once as a CUDA graph and replayed"}
                  if graph_ms is not None else {"unavailable": graph_err}),
        "experts": gemm_roofline(w, rows, used, expert_ms, peaks, peak_src, regime),
        "stages": stage_rooflines(w, rows, stage_ms, peaks["hbm_gbs"]),
        "rows": rows, "used_experts": used,
        "aux_loss": float(lb.layer.out.aux_loss.item()),
        "steps": steps, "warmup": warmup, "inputs_s": gen_s,
        **({"route_noisy": noisy} if noisy else {}),
    }
    del lb, D
    torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world):
    import torch
    import torch.distributed as dist

    from mixture_experts_top_b200 import api
    from workloads import WORKLOADS, make_inputs

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    w = WORKLOADS[args.workload]
    if args.tokens:
        w = w.with_tokens(args.tokens)
    if args.hidden:
        w = w.replace(d_hidden=args.hidden)
    peaks, peak_src = load_peaks()

    # inputs: weights identical on every rank, tokens drawn per rank
    t0 = time.time()
    inp = make_inputs(w, seed=0)
    if rank > 0:
        inp.update({k: v for k, v in make_inputs(w, seed=rank_token_seed(rank),
                                                 with_experts=False).items()
                    if k in ("x", "noise")})
    log(f"[rank {rank}] inputs generated in {time.time() - t0:.1f}s")
    D = to_device(inp)
    del inp
    # N > 1: one batch of N * T tokens split over the ranks in contiguous
    # blocks (rank r holds tokens [r T, (r + 1) T)); the capacity and aux
    # couple them through one all-gather of 2E+1 ints per rank and step.
    lb = LayerBench(w, D, shard=(rank, world, None) if world > 1 else None)
    cfg, o = lb.cfg, lb.layer.out
    T, k, E = w.T, w.top_k, w.E
    stream = lb.stream

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(0).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    elapsed_ms, expert_ms = lb.timed(args.steps, args.warmup, barrier, clocks)
    stage_ms = lb.stage_breakdown(args.steps, barrier)
    stage_ms[2] = expert_ms
    e2e_ms, h2d, d2h = lb.e2e(args.steps, args.warmup, barrier)
    clk = clocks.stop()
    status = lb.device_status()
    if status != 0:
        raise RuntimeError(f"device error word {status} after the benchmark")

    # max over ranks
    red = max_over_ranks([elapsed_ms, e2e_ms] + stage_ms, world, device="cuda")
    elapsed_ms, e2e_ms, stage_ms = red[0], red[1], red[2:]
    if rank != 0:
        return 0

    extras = {}
    if world == 1:
        graph_ms, graph_err = lb.graph_timed(args.steps, args.warmup)
        extras["graph"] = ({"tokens_per_s": T / (graph_ms / args.steps / 1e3),
                            "ms_per_step": graph_ms / args.steps,
                            "note": "the same step captured once as a CUDA graph and replayed"}
                           if graph_ms is not None else {"unavailable": graph_err})
    # The noisy gate's noise made on the device (moe_gate_noise), timed on
    # its own: the workload recipe hands the router a host-made noise tensor,
    # so this is not part of the step above.
    if D.get("W_noise") is not None and api.router_tc_width_supported(cfg):
        noise_dev = torch.empty((T, E), dtype=torch.float32, device="cuda")
        for _ in range(3):
            api.moe_gate_noise(cfg, D["x"], D["W_noise"], 7, 0, 0, noise_dev, lb.layer.ws)
        n_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        reps = 20
        n_ev[0].record(stream)
        for i in range(reps):
            api.moe_gate_noise(cfg, D["x"], D["W_noise"], 7, i, 0, noise_dev, lb.layer.ws)
        n_ev[1].record(stream)
        torch.cuda.synchronize()
        us = n_ev[0].elapsed_time(n_ev[1]) / reps * 1e3
        nb = T * w.d * 2 + w.d * E * 4 + T * E * 4
        extras["gate_noise"] = {"us": us, "GB/s": nb / us / 1e3,
                                "frac_hbm": nb / us / 1e3 / peaks["hbm_gbs"],
                                "note": "moe_gate_noise at this shape (x read, W_noise read, "
                                        "(T,E) fp32 noise written), back to back, x in L2"}

    # The routing half of the backward (moe_combine_backward +
    # moe_route_backward) and the experts' backward on this step's
    # intermediates, each timed on its own.
    if w.dtype == "bf16":
        extras["routing_backward"] = routing_backward(w, lb, peaks)
        extras["experts_backward"] = experts_backward(w, lb, peaks)
        if w.kind != "linear":
            extras["training_step"] = training_step(w, lb, peaks)

    counts = o.counts.cpu().numpy()
    rows = A.kept_rows(counts, w.capacity_factor, T, k)
    used = int((counts > 0).sum())
    ms_step = elapsed_ms / args.steps
    value = job_value(world, T, ms_step)
    regime = regime_of(elapsed_ms / 1e3)
    gemm = gemm_roofline(w, rows, used, stage_ms[2], peaks, peak_src, regime)
    # DRAM counters exist only for the captured workload (Mixtral shape, T = 8192).
    captured = w.name == "mixtral" and T == 8192 and w.d == 4096 and w.d_hidden == 14336
    gemm.update({
        "traffic": profiled_traffic("grouped_gemm.cu", "grouped_gemm_mixtral.md") if captured
                   else None,
        "traffic_note": "DRAM bytes of both launches of one step (ncu, Mixtral shape T=8192 "
                        "only), bytes per step",
        "kernel": "grouped_gemm_kernel (2 launches per step: up-projection with fused "
                  "activation, down-projection); achieved = algorithmic work of both / their "
                  "summed time (CUDA events on the launching stream, inside the timed loop)"})
    stages = stage_rooflines(w, rows, stage_ms, peaks["hbm_gbs"])
    stages["experts"] = {"ms": stage_ms[2], "frac": gemm["frac"], "bound": gemm["bound"]}
    stages["note"] = ("experts: events inside the timed loop; route, dispatch, combine: a "
                      "second pass of the same steps with an event between every two stages")

    # The other configurations, each on this GPU after the main line's
    # timed region (tokens/s, end to end, and each stage against its bound).
    if (world == 1 and not args.no_extras and args.workload == WORKLOAD and not args.tokens
            and not args.hidden):
        wl = {}
        for name in ("decode", "fine_grained", "switch_relu", "tiny_linear"):
            try:
                wl[name] = extra_workload(name, args.steps, args.warmup, peaks, peak_src,
                                          base_inputs=D if name == "decode" else None)
            except Exception as exc:   # reported, never hidden
                wl[name] = {"error": repr(exc)}
            log(f"[extras] {name}: done")
        extras["workloads"] = wl

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) tokens, N(0,1/fan_in) random-init weights)",
        "config": workload_config(w, world),
        "roofline": gemm,
        "stages": stages,
        **({"extras": extras} if extras else {}),
        "e2e": {"value": job_value(world, T, e2e_ms / args.steps), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "moe_forward via the Python binding; every step copies x from pinned host "
                       "memory and output + aux_loss back to pinned host memory, on copy "
                       "streams overlapped with the previous/next step's compute"},
        "gpu_launches": launches_per_step(w, cfg, world) * args.steps,
        "clocks": clk,
        "routing": {"rows": rows, "used_experts": used, "aux_loss": float(o.aux_loss.item())},
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_tokens)
    print(json.dumps(line), flush=True)
    return 0


def training_step(w, lb, peaks, steps=5, warmup=3):
    """One training step of the layer through the public calls, timed as a
    whole: the forward with the experts keeping their pre-activations
    (moe_route, moe_dispatch, moe_expert_ffn_train, moe_combine), then the
    backward from a fixed output gradient (moe_combine_backward,
    moe_route_backward, moe_expert_ffn_backward_saved, moe_permute_backward)."""
    import torch
    from mixture_experts_top_b200 import api
    D, o, cfg, stream = lb.D, lb.layer.out, lb.cfg, lb.stream
    T, k, E = w.T, w.top_k, w.E
    f32 = dict(dtype=torch.float32, device="cuda")
    Lg = torch.empty((T, E), **f32)
    gen = torch.Generator(device="cuda").manual_seed(9)
    dy = torch.randn((T, w.d_out), device="cuda", generator=gen).to(o.output.dtype)
    dyp = torch.empty((T * k, w.d_out), **f32)
    dg = torch.empty((T, k), **f32)
    daux = torch.ones(1, **f32)
    dx_route = torch.empty((T, w.d), **f32)
    dx_perm = torch.empty((T * k, w.d), **f32)
    dx = torch.empty((T, w.d), **f32)
    dWr = torch.empty((w.d, E), **f32)
    dbias = torch.empty(E, **f32)
    dWi = torch.empty(tuple(D["W_in"].shape), **f32)
    dWu = None if D["W_up"] is None else torch.empty(tuple(D["W_up"].shape), **f32)
    dWo = torch.empty(tuple(D["W_out"].shape), **f32)
    bws = api.alloc_backward_workspace(cfg)
    ws = lb.layer.ws

    def once():
        api.moe_route(cfg, D["x"], D["W_router"], D["logit_bias"], D["noise"], o.expert_indices,
                      o.gates, lb.P, Lg, ws)
        api.moe_dispatch(cfg, D["x"], o.expert_indices, lb.P, o.counts, lb.offsets, lb.dest,
                         lb.perm, o.drop_mask, lb.f, o.aux_loss, lb.x_perm, ws)
        api.moe_expert_ffn_train(cfg, lb.x_perm, lb.offsets, D["W_in"], D["W_up"], D["W_out"],
                                 lb.y_perm, ws, bws)
        api.moe_combine(cfg, lb.y_perm, lb.dest, o.gates, o.output)
        api.moe_combine_backward(cfg, dy, lb.y_perm, lb.dest, o.gates, dyp, dg)
        api.moe_route_backward(cfg, D["x"], D["W_router"], Lg, o.expert_indices, o.gates, lb.f,
                               dg, daux, 0, dx_route, dWr, dbias, None, ws)
        api.moe_expert_ffn_backward_saved(cfg, lb.x_perm, lb.offsets, D["W_in"], D["W_up"],
                                          D["W_out"], dyp, dx_perm, dWi, dWu, dWo, bws)
        api.moe_permute_backward(cfg, dx_perm, lb.dest, dx_route, dx)

    for _ in range(warmup):
        once()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(stream)
    for _ in range(steps):
        once()
    ev[1].record(stream)
    torch.cuda.synchronize()
    if api.moe_device_status(bws) != 0 or lb.device_status() != 0:
        raise RuntimeError("training step: device error word set")
    ms = ev[0].elapsed_time(ev[1]) / steps
    rows = A.kept_rows(o.counts.cpu().numpy(), w.capacity_factor, T, k)
    fwd = A.expert_gemm_flops(rows, w.d, w.d_hidden, w.d_out, w.kind)
    flops = 3 * fwd          # forward products, then their dgrad and wgrad
    ach = flops / (ms / 1e3) / 1e12
    del dyp, dx_perm, dWi, dWu, dWo, bws
    torch.cuda.empty_cache()
    return {"ms": ms, "tokens_per_s": T / (ms / 1e3), "expert_TFLOP/s": ach,
            "expert_frac_of_burst": ach / peaks["bf16_tflops"], "expert_flops": flops,
            "steps": steps, "warmup": warmup,
            "note": "forward (moe_route, moe_dispatch, moe_expert_ffn_train, moe_combine) and "
                    "backward (moe_combine_backward, moe_route_backward, "
                    "moe_expert_ffn_backward_saved, moe_permute_backward) from a fixed output "
                    "gradient, 13+ launches a step; expert FLOPs = 3x the forward's products "
                    "over the whole step's time"}


def routing_backward(w, lb, peaks):
    import torch
    from mixture_experts_top_b200 import api
    D, o, cfg, stream = lb.D, lb.layer.out, lb.cfg, lb.stream
    T, k, E = w.T, w.top_k, w.E
    Lg = torch.empty((T, E), dtype=torch.float32, device="cuda")
    api.moe_route(cfg, D["x"], D["W_router"], D["logit_bias"], D["noise"], o.expert_indices,
                  o.gates, lb.P, Lg, lb.layer.ws)
    api.moe_dispatch(cfg, D["x"], o.expert_indices, lb.P, o.counts, lb.offsets, lb.dest, lb.perm,
                     o.drop_mask, lb.f, o.aux_loss, lb.x_perm, lb.layer.ws)
    api.moe_expert_ffn(cfg, lb.x_perm, lb.offsets, D["W_in"], D["W_up"], D["W_out"], lb.y_perm,
                       lb.layer.ws)
    dyb = torch.randn((T, w.d_out), device="cuda").to(o.output.dtype)
    dyp = torch.empty((T * k, w.d_out), dtype=torch.float32, device="cuda")
    dgb = torch.empty((T, k), dtype=torch.float32, device="cuda")
    dxb = torch.empty((T, w.d), dtype=torch.float32, device="cuda")
    dWb = torch.empty((w.d, E), dtype=torch.float32, device="cuda")
    dbb = torch.empty(E, dtype=torch.float32, device="cuda")
    dab = torch.ones(1, dtype=torch.float32, device="cuda")

    def once():
        api.moe_combine_backward(cfg, dyb, lb.y_perm, lb.dest, o.gates, dyp, dgb)
        api.moe_route_backward(cfg, D["x"], D["W_router"], Lg, o.expert_indices, o.gates, lb.f,
                               dgb, dab, 0, dxb, dWb, dbb, None, lb.layer.ws)

    for _ in range(3):
        once()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(stream)
    for _ in range(10):
        once()
    ev[1].record(stream)
    torch.cuda.synchronize()
    us = ev[0].elapsed_time(ev[1]) / 10 * 1e3
    elem = 2 if w.dtype == "bf16" else 4
    kept = int((lb.dest >= 0).sum().item())
    nb = (T * w.d_out * elem + 2 * kept * w.d_out * 4
          + T * E * 4 * 2 + T * w.d * (elem + 4) + T * k * 16)
    return {"us": us, "GB/s": nb / us / 1e3, "frac_hbm": nb / us / 1e3 / peaks["hbm_gbs"],
            "note": "moe_combine_backward + moe_route_backward (6 launches): dy read, expert rows "
                    "read and their gradients written, logits and dlogits, x read and dx written"}


def route_noisy_timing(w, lb, peaks):
    """The router with the noisy gate's noise made inside it (moe_route_noisy)
    against the router fed a host-made noise tensor (moe_route), each back to
    back on this workload's tokens."""
    import torch
    from mixture_experts_top_b200 import api
    from mixture_experts_top_b200.api import router_tc_width_supported
    D, o, cfg, stream = lb.D, lb.layer.out, lb.cfg, lb.stream
    if D.get("W_noise") is None or not router_tc_width_supported(cfg):
        return None
    reps = 20

    def timed(fn):
        for _ in range(3):
            fn()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(stream)
        for _ in range(reps):
            fn()
        ev[1].record(stream)
        torch.cuda.synchronize()
        return ev[0].elapsed_time(ev[1]) / reps * 1e3

    fused = timed(lambda: api.moe_route_noisy(
        cfg, D["x"], D["W_router"], D["logit_bias"], D["W_noise"], 7, 0, 0, o.expert_indices,
        o.gates, lb.P, None, None, lb.layer.ws))
    host_noise = timed(lambda: api.moe_route(
        cfg, D["x"], D["W_router"], D["logit_bias"], D["noise"], o.expert_indices, o.gates, lb.P,
        None, lb.layer.ws))
    nb = A.router_bytes(w.T, w.d, w.E, w.top_k, 2, False) + w.d * w.E * 4
    return {"fused_us": fused, "host_noise_us": host_noise,
            "fused_GB/s": nb / fused / 1e3, "frac_hbm": nb / fused / 1e3 / peaks["hbm_gbs"],
            "note": "moe_route_noisy (noise logits from the router's own contraction, z and "
                    "softplus in the logit pass; x, W_router and W_noise read, indices and gates "
                    "written) vs moe_route reading a (T, E) noise tensor; back to back, 20 calls"}


def experts_backward(w, lb, peaks):
    """moe_expert_ffn_backward on this step's grouped rows with a seeded
    dy_perm: pack, recompute of the pre-activations, dH (with the activation
    backward in its epilogue), dX and the weight gradients, back to back."""
    import torch
    from mixture_experts_top_b200 import api
    D, o, cfg, stream = lb.D, lb.layer.out, lb.cfg, lb.stream
    T, k, E = w.T, w.top_k, w.E
    R = T * k
    gen = torch.Generator(device="cuda").manual_seed(5)
    dyp = torch.randn((R, w.d_out), device="cuda", generator=gen)
    dxp = torch.empty((R, w.d), device="cuda")
    dWi = torch.empty(tuple(D["W_in"].shape), device="cuda")
    dWu = None if D["W_up"] is None else torch.empty(tuple(D["W_up"].shape), device="cuda")
    dWo = torch.empty(tuple(D["W_out"].shape), device="cuda")
    bws = api.alloc_backward_workspace(cfg)

    def once():
        api.moe_expert_ffn_backward(cfg, lb.x_perm, lb.offsets, D["W_in"], D["W_up"], D["W_out"],
                                    dyp, dxp, dWi, dWu, dWo, bws)

    for _ in range(2):
        once()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    reps = 5
    ev[0].record(stream)
    for _ in range(reps):
        once()
    ev[1].record(stream)
    torch.cuda.synchronize()
    if api.moe_device_status(bws) != 0:
        raise RuntimeError("experts' backward: device error word set")
    ms = ev[0].elapsed_time(ev[1]) / reps

    # Training forward (the experts' rows and, kept in bws, their
    # pre-activations) against the plain forward, then the backward that
    # takes the kept pre-activations instead of recomputing them.
    def timed(fn):
        for _ in range(2):
            fn()
        ev[0].record(stream)
        for _ in range(reps):
            fn()
        ev[1].record(stream)
        torch.cuda.synchronize()
        return ev[0].elapsed_time(ev[1]) / reps

    saved = None
    if w.kind != "linear":
        fwd_ms = timed(lambda: api.moe_expert_ffn(cfg, lb.x_perm, lb.offsets, D["W_in"],
                                                  D["W_up"], D["W_out"], lb.y_perm, lb.layer.ws))
        train_ms = timed(lambda: api.moe_expert_ffn_train(cfg, lb.x_perm, lb.offsets, D["W_in"],
                                                          D["W_up"], D["W_out"], lb.y_perm,
                                                          lb.layer.ws, bws))
        saved_ms = timed(lambda: api.moe_expert_ffn_backward_saved(
            cfg, lb.x_perm, lb.offsets, D["W_in"], D["W_up"], D["W_out"], dyp, dxp, dWi, dWu, dWo,
            bws))
        saved = (fwd_ms, train_ms, saved_ms)
    if api.moe_device_status(bws) != 0 or lb.device_status() != 0:
        raise RuntimeError("experts' backward: device error word set")
    counts = o.counts.cpu().numpy()
    rows = A.kept_rows(counts, w.capacity_factor, T, k)
    mats = A.MATRICES[w.kind]
    fwd = A.expert_gemm_flops(rows, w.d, w.d_hidden, w.d_out, w.kind)
    algo = 2 * fwd                     # dgrad + wgrad: two products per forward product
    executed = algo + (fwd * (mats - 1) // mats)   # + the recomputed up projection(s)
    ach = algo / (ms / 1e3) / 1e12
    del dyp, dxp, dWi, dWu, dWo, bws
    torch.cuda.empty_cache()
    res = {"ms": ms, "TFLOP/s": ach, "frac_of_burst": ach / peaks["bf16_tflops"],
           "algorithmic_flops": algo, "executed_flops": executed,
           "note": "moe_expert_ffn_backward (pack, recompute of the pre-activations, dH with "
                   "the activation backward fused, dX, weight gradients): algorithmic FLOPs = "
                   "the dgrad and wgrad products (2x the forward's), executed adds the "
                   "recomputed up projection; back to back, 5 calls"}
    if saved is not None:
        fwd_ms, train_ms, saved_ms = saved
        ach_s = algo / (saved_ms / 1e3) / 1e12
        res["saved"] = {
            "ms": saved_ms, "TFLOP/s": ach_s, "frac_of_burst": ach_s / peaks["bf16_tflops"],
            "forward_experts_ms": fwd_ms, "train_forward_experts_ms": train_ms,
            "note": "moe_expert_ffn_train (the forward's experts keeping their fp32 "
                    "pre-activations in the backward workspace) against moe_expert_ffn, and "
                    "moe_expert_ffn_backward_saved (no recompute); back to back, 5 calls each"}
    return res


def cpu_baseline(w, tokens):
    """The oracle, as it stands, on one batch of `tokens` tokens of the
    workload (its first tokens), timed on the host cores."""
    from oracle import moe_oracle as O
    from workloads import make_inputs
    inp = make_inputs(w, seed=0)
    n = min(tokens, w.T)
    weights = {k: inp[k] for k in ("W_in", "W_up", "W_out")}
    t0 = time.perf_counter()
    O.moe_forward(inp["x"][:n], inp["W_router"], weights, top_k=w.top_k, kind=w.kind,
                  dtype=w.dtype, d_out=w.d_out, capacity_factor=w.capacity_factor,
                  logit_bias=inp["logit_bias"],
                  noise=None if inp["noise"] is None else inp["noise"][:n])
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"one batch of the workload's first {n} tokens through the full oracle "
                      f"forward in fp64 ({dt:.1f} s of CPU work, which includes widening the "
                      "used experts' bf16 weights to fp64 once per expert)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T (smaller cases for profiling; not a bench line)")
    ap.add_argument("--hidden", type=int, default=0,
                    help="override d_hidden (smaller cases for profiling; not a bench line)")
    ap.add_argument("--cpu-tokens", type=int, default=64,
                    help="tokens in the oracle's timed batch (cpu_baseline)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other configurations' figures (extras.workloads)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        return run_ours(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
