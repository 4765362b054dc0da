#!/usr/bin/env python3
"""Benchmark of the MoE layer forward pass on B200 GPUs.

One step = one pass of the whole hot path (route -> dispatch -> experts ->
combine, aux loss included) over one batch of the Mixtral-shaped workload
(T=8192 tokens, D=4096, DH=14336, E=8, top-2 SwiGLU experts, bf16, fp32
router), synthetic seeded inputs, random-init weights of that shape.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (launched by torch.distributed.run): every rank runs its own batch
(data parallel, weak scaling, no collective on the data path); the step time
is the max over ranks; value = tokens of all ranks / that time.

The reference arm (--impl reference) times the CPU oracle, as it stands, on
the host cores (rank 0 only), one token of the workload per step.
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


def launches_per_step(w, cfg) -> int:
    """Kernels of this library launched by one timed step (route, dispatch,
    experts, combine), as the library picks them for this configuration:
    route = weight split + tensor-core router + P mean (bf16, E <= 64) or
    SIMT router + P mean; dispatch = count + scan + scatter; experts = up and
    down GEMM (bf16) or the fp32 linear kernel; combine = 1."""
    from mixture_experts_top_b200 import api as _api
    if w.T == 0:
        return 2                       # P mean and the dispatch scan only
    route = 3 if _api.router_tc_width_supported(cfg) else 2
    experts = 1 if w.kind == "linear" else 2
    return route + 3 + experts + 1


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
                                   "through the full oracle forward"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, n):
    return {"workload": f"{w.name}: Mixtral-shaped SwiGLU MoE layer, T={w.T} tokens per GPU, "
                        f"D={w.d}, DH={w.d_hidden}, E={w.E}, top_k={w.top_k}, bf16 with fp32 "
                        "router and fp32 accumulation, no capacity limit",
            "T": w.T, "d": w.d, "d_hidden": w.d_hidden, "E": w.E, "top_k": w.top_k,
            "global_batch": w.T * n,
            "parallelism": f"dp{n} (independent batch per GPU, replicated weights)",
            "l2": "no flush: each step streams 2.8 GB of expert weights, > 126 MB L2"}


# ---------------------------------------------------------------- our arm --

def run_ours(args, rank, world):
    import numpy as np
    import torch
    import torch.distributed as dist

    from mixture_experts_top_b200 import accounting as A
    from mixture_experts_top_b200 import api
    from mixture_experts_top_b200.layer import MoeForward
    from workloads import WORKLOADS, make_inputs

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    w = WORKLOADS[args.workload]
    if args.tokens:
        w = w.with_tokens(args.tokens)
    peaks, peak_src = load_peaks()

    # inputs: weights identical on every rank, tokens drawn per rank
    t0 = time.time()
    inp = make_inputs(w, seed=0)
    if rank > 0:
        inp.update({k: v for k, v in make_inputs(w, seed=rank_token_seed(rank),
                                                 with_experts=False).items()
                    if k in ("x", "noise")})
    log(f"[rank {rank}] inputs generated in {time.time() - t0:.1f}s")

    def dev(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()

    x, Wr, bias, noise = dev(inp["x"]), dev(inp["W_router"]), dev(inp["logit_bias"]), dev(inp["noise"])
    W_in, W_up, W_out = dev(inp["W_in"]), dev(inp["W_up"]), dev(inp["W_out"])
    W_noise = dev(inp["W_noise"])
    del inp
    cfg = api.make_config(w.T, w.d, w.d_hidden, w.d_out, w.E, w.top_k, w.kind, w.dtype,
                          w.capacity_factor)
    layer = MoeForward(cfg)
    o = layer.out
    T, k, E = w.T, w.top_k, w.E
    R = T * k
    i32 = dict(dtype=torch.int32, device="cuda")
    P = torch.empty(E, dtype=torch.float32, device="cuda")
    offsets = torch.empty(E + 1, **i32)
    dest = torch.empty(R, **i32)
    perm = torch.empty(R, **i32)
    f = torch.empty(E, dtype=torch.float32, device="cuda")
    x_perm = torch.empty((R, w.d), dtype=torch.bfloat16, device="cuda")
    y_perm = torch.empty((R, w.d_out), dtype=torch.float32, device="cuda")
    ws = layer.ws
    stream = torch.cuda.current_stream()

    def step(ev=None, marks=(0, 1, 2, 3, 4)):
        # ev[j] is recorded before stage j (route, dispatch, experts, combine)
        # and ev[4] after the last, for the stage indices listed in `marks`.
        # Every recorded event separates two launches that could otherwise
        # overlap (each kernel is launched as a programmatic dependent of the
        # one before), so the timed loop marks only the expert stage.
        def mark(j):
            if ev is not None and j in marks:
                ev[j].record(stream)
        mark(0)
        api.moe_route(cfg, x, Wr, bias, noise, o.expert_indices, o.gates, P, None, ws)
        mark(1)
        api.moe_dispatch(cfg, x, o.expert_indices, P, o.counts, offsets, dest, perm, o.drop_mask,
                         f, o.aux_loss, x_perm, ws)
        mark(2)
        api.moe_expert_ffn(cfg, x_perm, offsets, W_in, W_up, W_out, y_perm, ws)
        mark(3)
        api.moe_combine(cfg, y_perm, dest, o.gates, o.output)
        mark(4)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(0).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        step(evs[i], marks=(2, 3))
    end.record(stream)
    barrier()
    elapsed_ms = start.elapsed_time(end)
    expert_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / args.steps

    # Stage breakdown (diagnostic, outside the timed region): the same steps
    # again with an event between every two stages.
    for i in range(args.steps):
        step(evs[i])
    barrier()
    stage_ms = [sum(e[j].elapsed_time(e[j + 1]) for e in evs) / args.steps for j in range(4)]
    stage_ms[2] = expert_ms

    # End to end through the public call (moe_forward): every step copies its
    # tokens from pinned host memory and its output and aux_loss back to pinned
    # host memory.  Copies run on their own streams, double-buffered, so step
    # i's upload and step i-1's download overlap step i's compute.
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
    ws_e2e = api.alloc_workspace(cfg)

    def e2e_steps(n):
        for i in range(n):
            b = bufs[i % 2]
            with torch.cuda.stream(s_up):
                s_up.wait_event(b["computed"])       # step i-2 finished reading b["x"]
                b["x"].copy_(x_host, non_blocking=True)
                if noise is not None:
                    b["noise"].copy_(n_host, non_blocking=True)
                b["uploaded"].record(s_up)
            stream.wait_event(b["uploaded"])
            stream.wait_event(b["downloaded"])       # step i-2's output was copied out
            api.moe_forward(cfg, b["x"], Wr, bias, b["noise"], W_in, W_up, W_out, b["out"],
                            o.expert_indices, o.gates, b["aux"], None, None, ws_e2e)
            b["computed"].record(stream)
            with torch.cuda.stream(s_dn):
                s_dn.wait_event(b["computed"])
                b["out_host"].copy_(b["out"], non_blocking=True)
                b["aux_host"].copy_(b["aux"], non_blocking=True)
                b["downloaded"].record(s_dn)

    e2e_steps(args.warmup)
    barrier()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    s_up.wait_stream(stream)                         # the first upload starts after s2
    e2e_steps(args.steps)
    stream.wait_stream(s_dn)
    e2.record(stream)
    barrier()
    e2e_ms = s2.elapsed_time(e2)
    clk = clocks.stop()
    status = layer.device_status() or api.moe_device_status(ws_e2e)
    if status != 0:
        raise RuntimeError(f"device error word {status} after the benchmark")

    # max over ranks
    red = max_over_ranks([elapsed_ms, e2e_ms] + stage_ms, world, device="cuda")
    elapsed_ms, e2e_ms, stage_ms = red[0], red[1], red[2:]
    if rank != 0:
        return 0

    # The noisy gate's noise made on the device (moe_gate_noise), timed on
    # its own: the workload recipe hands the router a host-made noise tensor,
    # so this is not part of the step above.
    extras = {}
    if W_noise is not None and api.router_tc_width_supported(cfg):
        noise_dev = torch.empty((T, E), dtype=torch.float32, device="cuda")
        for _ in range(3):
            api.moe_gate_noise(cfg, x, W_noise, 7, 0, 0, noise_dev, ws)
        n_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        reps = 20
        n_ev[0].record(stream)
        for i in range(reps):
            api.moe_gate_noise(cfg, x, W_noise, 7, i, 0, noise_dev, ws)
        n_ev[1].record(stream)
        torch.cuda.synchronize()
        us = n_ev[0].elapsed_time(n_ev[1]) / reps * 1e3
        nb = T * w.d * 2 + w.d * E * 4 + T * E * 4
        extras["gate_noise"] = {"us": us, "GB/s": nb / us / 1e3,
                                "frac_hbm": nb / us / 1e3 / peaks["hbm_gbs"],
                                "note": "moe_gate_noise at this shape (x read, W_noise read, "
                                        "(T,E) fp32 noise written), back to back, x in L2"}

    # The routing half of the backward (moe_combine_backward +
    # moe_route_backward) on this step's intermediates, timed on its own.
    Lg = torch.empty((T, E), dtype=torch.float32, device="cuda")
    api.moe_route(cfg, x, Wr, bias, noise, o.expert_indices, o.gates, P, Lg, ws)
    api.moe_dispatch(cfg, x, o.expert_indices, P, o.counts, offsets, dest, perm, o.drop_mask,
                     f, o.aux_loss, x_perm, ws)
    api.moe_expert_ffn(cfg, x_perm, offsets, W_in, W_up, W_out, y_perm, ws)
    dyb = torch.randn((T, w.d_out), device="cuda").to(o.output.dtype)
    dyp = torch.empty((R, w.d_out), dtype=torch.float32, device="cuda")
    dgb = torch.empty((T, k), dtype=torch.float32, device="cuda")
    dxb = torch.empty((T, w.d), dtype=torch.float32, device="cuda")
    dWb = torch.empty((w.d, E), dtype=torch.float32, device="cuda")
    dbb = torch.empty(E, dtype=torch.float32, device="cuda")
    dab = torch.ones(1, dtype=torch.float32, device="cuda")

    def backward_once():
        api.moe_combine_backward(cfg, dyb, y_perm, dest, o.gates, dyp, dgb)
        api.moe_route_backward(cfg, x, Wr, Lg, o.expert_indices, o.gates, f, dgb, dab, 0, dxb,
                               dWb, dbb, None, ws)

    for _ in range(3):
        backward_once()
    b_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    b_ev[0].record(stream)
    for _ in range(10):
        backward_once()
    b_ev[1].record(stream)
    torch.cuda.synchronize()
    b_us = b_ev[0].elapsed_time(b_ev[1]) / 10 * 1e3
    elem = 2 if w.dtype == "bf16" else 4
    kept = int((dest >= 0).sum().item())
    b_bytes = (T * w.d_out * elem + 2 * kept * w.d_out * 4
               + T * E * 4 * 2 + T * w.d * (elem + 4) + T * k * 16)
    extras["routing_backward"] = {
        "us": b_us, "GB/s": b_bytes / b_us / 1e3, "frac_hbm": b_bytes / b_us / 1e3 / peaks["hbm_gbs"],
        "note": "moe_combine_backward + moe_route_backward (6 launches): dy read, expert rows "
                "read and their gradients written, logits and dlogits, x read and dx written"}

    counts = o.counts.cpu().numpy()
    rows = A.kept_rows(counts, w.capacity_factor, T, k)
    used = int((counts > 0).sum())
    ms_step = elapsed_ms / args.steps
    value = job_value(world, T, ms_step)
    flops = A.expert_gemm_flops(rows, w.d, w.d_hidden, w.d_out, w.kind)
    t_exp = stage_ms[2] / 1e3
    # The GEMMs run back to back for the whole timed loop (seconds at the power
    # cap), so the sustained cuBLAS figure is the denominator; the burst
    # fraction is given beside it.  Where the expert weights take longer to
    # stream than the FLOPs take on the tensor cores (few rows per expert),
    # the bound is HBM instead: algorithmic bytes = the used experts' weights
    # + rows in + the hidden activation written and read + fp32 rows out.
    tensor_peak = peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"]
    burst_peak = peaks["bf16_tflops"]
    hbm = peaks["hbm_gbs"]
    elem = 4 if w.kind == "linear" else 2
    gemm_bytes = (A.expert_weight_bytes(used, w.d, w.d_hidden, w.d_out, w.kind, elem)
                  + rows * w.d * elem + rows * w.d_out * 4
                  + (0 if w.kind == "linear" else 2 * rows * w.d_hidden * 2))
    tensor_bound = flops / (tensor_peak * 1e12) >= gemm_bytes / (hbm * 1e9)
    kernel_note = ("grouped_gemm_kernel (2 launches per step: up-projection with fused "
                   "activation, down-projection); achieved = algorithmic work of both / their "
                   "summed time")
    if tensor_bound:
        gemm = {"bound": "tensor", "achieved": flops / t_exp / 1e12, "peak": tensor_peak,
                "unit": "TFLOP/s", "frac": flops / t_exp / 1e12 / tensor_peak,
                "frac_of_burst": flops / t_exp / 1e12 / burst_peak,
                "peak_source": (f"{peak_src} sustained bf16 (cuBLAS back to back for 4 s)"
                                if peaks.get("bf16_tflops_sustained") else
                                f"{peak_src} burst bf16 (cuBLAS)")}
    else:
        gemm = {"bound": "hbm", "achieved": gemm_bytes / t_exp / 1e9, "peak": hbm,
                "unit": "GB/s", "frac": gemm_bytes / t_exp / 1e9 / hbm,
                "peak_source": f"{peak_src} HBM copy bandwidth"}
    # DRAM counters exist only for the captured workload (Mixtral shape, T = 8192).
    captured = w.name == "mixtral" and T == 8192 and w.d == 4096
    gemm.update({
        "traffic": profiled_traffic("grouped_gemm.cu", "grouped_gemm_mixtral.md") if captured
                   else None,
        "traffic_note": "DRAM bytes of both launches of one step (ncu, Mixtral shape T=8192 "
                        "only), bytes per step",
        "algorithmic_bytes": gemm_bytes, "algorithmic_flops": flops,
        "kernel": kernel_note})
    rb = A.router_bytes(T, w.d, E, k, 2, w.noise)
    pb = A.permute_bytes(T, rows, w.d, 2)
    cb = A.combine_bytes(T, rows, w.d_out, k, 2)
    stages = {
        "route": {"ms": stage_ms[0], "GB/s": rb / stage_ms[0] / 1e6, "frac_hbm": rb / stage_ms[0] / 1e6 / hbm},
        "dispatch": {"ms": stage_ms[1], "GB/s": pb / stage_ms[1] / 1e6, "frac_hbm": pb / stage_ms[1] / 1e6 / hbm},
        "experts": {"ms": stage_ms[2], "TFLOP/s": flops / t_exp / 1e12,
                    "frac_tensor": flops / t_exp / 1e12 / tensor_peak},
        "combine": {"ms": stage_ms[3], "GB/s": cb / stage_ms[3] / 1e6, "frac_hbm": cb / stage_ms[3] / 1e6 / hbm},
        "note": "experts: events inside the timed loop; route, dispatch, combine: a second "
                "pass of the same steps with an event between every two stages",
    }
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
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
        "gpu_launches": launches_per_step(w, cfg) * args.steps,
        "clocks": clk,
        "routing": {"rows": rows, "used_experts": used, "aux_loss": float(o.aux_loss.item())},
    }
    if world == 1 and not args.no_cpu_baseline:
        import numpy as np  # noqa: F811
        from workloads import make_inputs as mk
        inp = mk(w, seed=0)
        times = oracle_token_steps(w, inp, list(range(args.cpu_tokens)))
        line["cpu_baseline"] = {
            "value": len(times) / sum(times), "unit": "tokens/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{len(times)} tokens of the batch, each run as a batch of its own through "
                      f"the full oracle forward ({sum(times):.1f} s of CPU work)"}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T (smaller cases for profiling; not a bench line)")
    ap.add_argument("--cpu-tokens", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
