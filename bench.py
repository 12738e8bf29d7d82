#!/usr/bin/env python
"""Benchmark of the frame-wise Gated DeltaNet forward on B200.

Workload: the 720p 60 s latent shape, B=1, H=20 heads of width d_k=d_v=112,
F=240 latent frames x L=920 tokens (23x40 grid), bf16 q/k/v, fp32 gates,
state and output, seeded synthetic inputs (the pages' minute-scale 720p
rollout; no dataset exists in this environment).  One step = one
gdn_frame_fwd call over the whole workload (gates, key normalisation, frame
maps, frame chain, read-out, stores).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs its own independent copy of the workload (the
recurrence shards over batch and heads with no exchange: weak scaling); the
step time is the max over ranks.  Prints one JSON line on rank 0.

--impl reference times the fp64 CPU oracle (the correctness reference of this
library) on the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN frame-recurrence tokens/s (720p-60s shape, bf16) and % of roofline"
WORKLOAD = "gdn_720p_60s"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0  # B200 HBM3e figure quoted as "about 8 TB/s"
FALLBACK_BF16_TFLOPS = 1590.0  # dense bf16 GEMM (burst) measured earlier on this machine
# algorithmic bytes per token-head: q, k, v bf16 (3 * 112 * 2) + o fp32 (112 * 4) + beta fp32
BYTES_PER_TOKEN_HEAD = 3 * 112 * 2 + 112 * 4 + 4
FLOPS_PER_TOKEN_HEAD = 6 * 112 * 112
PRECISION = ("bf16 q/k/v; fp16 tensor-core operands with fp32 accumulation; the state passes from frame to "
             "frame as fp16 (each frame's map contracts; alpha = 1 over 240 frames is tested) and is taken "
             "from state_in as fp16 high + low parts; fp32 o and state_out")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-streaming", action="store_true", help="skip the streaming-call leg")
    ap.add_argument("--frames", type=int, default=0,
                    help="use only the first N latent frames (a smaller case of the same kernel, for profiling)")
    ap.add_argument("--quick", action="store_true",
                    help="kernel leg only: no end-to-end leg, no ReLU-mode line, no CPU baseline")
    ap.add_argument("--profile-case", choices=["gdn", "relu", "tconv", "stream", "swa", "bwd"], default=None,
                    help="run three launches of one kernel on a small case (inputs larger than L2, under 1 GB) "
                         "and exit: the command profiled with ncu --set full")
    return ap.parse_args()


def profile_case(name: str):
    """Three launches of one kernel at a reduced size of its workload: gdn_tc_kernel
    on the first 48 frames of the 720p 60 s shape, relu_tc_kernel on 16 of the 81
    frames, the temporal convolution on 60 of the 240 frames, and one streaming
    call (F = 1, all 20 heads, 920 tokens; 12 MB, L2-resident as in the protocol)."""
    import torch

    import linear_attention_video_gdn_b200 as lib
    import synth
    dev = torch.device("cuda", 0)
    if name in ("gdn", "stream"):
        w = synth.WORKLOADS["gdn_720p_60s"].with_(F=48) if name == "gdn" else synth.WORKLOADS["gdn_stream_720p"]
        x = synth.inputs(w)
        q, k, v = (torch.from_numpy(x[n]).to(torch.bfloat16).to(dev) for n in "qkv")
        a, b = (torch.from_numpy(x[n]).to(dev) for n in "ab")
        F = w.F if name == "gdn" else 1
        s_in = torch.zeros((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev) if name == "stream" else None
        call = lambda: lib.gdn_frame_fwd(q, k, v, a, b, F=F, state_in=s_in)
    elif name == "relu":
        w = synth.WORKLOADS["relu_720p_81f"].with_(F=16)
        x = synth.inputs(w)
        q, k, v = (torch.from_numpy(x[n]).to(torch.bfloat16).to(dev) for n in "qkv")
        call = lambda: lib.relu_la_block_fwd(q, k, v, F=w.F)
    elif name == "bwd":  # the backward, first 24 of the 240 frames of the 720p 60 s shape
        w = synth.WORKLOADS["gdn_720p_60s"].with_(F=24)
        x = synth.inputs(w)
        q, k, v = (torch.from_numpy(x[n]).to(torch.bfloat16).to(dev) for n in "qkv")
        a, b = (torch.from_numpy(x[n]).to(dev) for n in "ab")
        d_o = torch.from_numpy(synth.grad_inputs(w)["d_o"]).to(dev)
        call = lambda: lib.gdn_frame_bwd(q, k, v, a, b, d_o, F=w.F)
    elif name == "swa":  # windowed softmax layer, first 24 of the 240 frames, W = 4
        F, L, d = 24, 920, 112
        q, k, v = (torch.from_numpy(synth.normal(7, t, 0, 20 * F * L * d).reshape(1, 20, F * L, d))
                   .to(torch.bfloat16).to(dev) for t in range(3))
        call = lambda: lib.softmax_window_fwd(q, k, v, F=F, W=4)
    else:
        cw = synth.CONV_WORKLOADS["tconv_720p_60s"]
        inp = synth.conv_inputs(cw, frames=60)
        xc = torch.from_numpy(inp["x"]).to(torch.bfloat16).to(dev)
        wc, bc = torch.from_numpy(inp["w"]).to(dev), torch.from_numpy(inp["bias"]).to(dev)
        cache = torch.zeros((cw.B, cw.HW, cw.C), dtype=torch.bfloat16, device=dev)
        call = lambda: lib.temporal_conv_fwd(xc, wc, bias=bc, cache_in=cache, cache_out=cache)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    print(f"profile case {name}: 3 launches done", flush=True)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# source files each profiled kernel is built from: a committed traffic figure
# counts only while their hash matches the figure's
KERNEL_SOURCES = {
    "gdn_tc": ("gdn_tc.cu", "tc_ptx.cuh", "common.cuh"),
    "relu_tc": ("relu_tc.cu", "tc_ptx.cuh", "common.cuh"),
    "temporal_conv": ("temporal_conv.cu", "f32x2.cuh", "tc_ptx.cuh", "common.cuh"),
    "softmax_window": ("softmax_window.cu", "f32x2.cuh", "tc_ptx.cuh", "common.cuh"),
    "gdn_bwd": ("gdn_bwd.cu", "common.cuh"),
}


def kernel_source_hash(kernel: str = "gdn_tc") -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "linear_attention_video_gdn_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str = "gdn_tc"):
    """DRAM bytes per launch of a kernel from its committed ncu summary
    (profiles/<kernel>_traffic.json), if it was taken on the current kernel
    source (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if d.get("kernel_source_sha") == kernel_source_hash(kernel):
            return d
    except Exception:
        pass
    return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running (read-only)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int, period_s: float = 0.02):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                self.reasons |= int(self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._ok:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        s = sorted(self.samples)
        return {"sm_mhz": s[len(s) // 2], "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in self.REASONS.items() if self.reasons & b], "samples": len(s)}


def gdn_workload(frames: int = 0):
    import synth
    w = synth.WORKLOADS[WORKLOAD]
    return w.with_(F=frames) if 0 < frames < w.F else w


def oracle_sample(w, frames: int, nthreads: int):
    """Run the fp64 oracle on all heads of the first `frames` frames of the workload;
    returns (seconds, tokens)."""
    import oracle
    import synth
    x = synth.inputs(w, frames=frames)  # the workload's first `frames` frames, every head
    # q, k, v are rounded to bf16 exactly as the device sees them
    import torch
    hx = {n: torch.from_numpy(x[n]).to(torch.bfloat16).float().numpy() for n in "qkv"}
    t0 = time.perf_counter()
    oracle.gdn(hx["q"], hx["k"], hx["v"], x["a"], x["b"], F=frames, L=w.L, nthreads=nthreads)
    dt = time.perf_counter() - t0
    return dt, w.B * frames * w.L


def cpu_baseline(w, target_s: float = 12.0):
    nthreads = os.cpu_count() or 1
    units = w.B * w.H * ((w.dv + 15) // 16)
    t1, _ = oracle_sample(w, 2, nthreads)
    per_frame = max(t1 / 2, 1e-4)
    frames = int(max(2, min(w.F, target_s / per_frame)))
    dt, tokens = oracle_sample(w, frames, nthreads)
    return {"value": tokens / dt, "unit": "tokens/s", "cores": min(nthreads, units), "kind": "oracle",
            "sample": f"all {w.B * w.H} heads x first {frames} of {w.F} frames (L={w.L}, d=112), fp64 "
                      f"per-token recurrence in C on {min(nthreads, units)} threads, {dt:.1f} s"}


def run_reference(args, rank: int):
    """The oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return
    w = gdn_workload()
    nthreads = os.cpu_count() or 1
    units = w.B * w.H * ((w.dv + 15) // 16)
    budget = 150.0 / max(1, args.steps + args.warmup)
    t1, _ = oracle_sample(w, 1, nthreads)
    frames = int(max(1, min(w.F, budget / max(t1, 1e-4))))
    for _ in range(args.warmup):
        oracle_sample(w, frames, nthreads)
    times = []
    tokens = 0
    for _ in range(args.steps):
        dt, tokens = oracle_sample(w, frames, nthreads)
        times.append(dt)
    tot = sum(times)
    value = tokens * len(times) / tot
    sample = f"all {w.B * w.H} heads x first {frames} of {w.F} frames per step, fp64 C oracle, {min(nthreads, units)} threads"
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": w.B, "H": w.H, "F": w.F, "L": w.L, "dk": w.dk, "dv": w.dv,
                       "sample_frames": frames},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": min(nthreads, units), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def max_over_ranks(value: float, device, world: int) -> float:
    """The largest per-rank value (the step time of the slowest rank); every rank
    gets it.  With one rank, the value itself."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Weak scaling: every rank processes its own copy of the workload, so the job
    processes world x tokens in the slowest rank's step time."""
    return world * tokens_per_rank / (ms_max / 1e3)


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import linear_attention_video_gdn_b200 as lib
    import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = gdn_workload(args.frames)
    x = synth.inputs(w)
    tokens = w.B * w.N
    token_heads = tokens * w.H
    # host copies (pinned) for the end-to-end leg, device copies for the kernel leg
    hq, hk, hv = (torch.from_numpy(x[n]).to(torch.bfloat16).pin_memory() for n in "qkv")
    ha, hb = (torch.from_numpy(x[n]).pin_memory() for n in "ab")
    q, k, v, a, b = (t.to(dev) for t in (hq, hk, hv, ha, hb))
    o = torch.empty((w.B, w.H, w.N, w.dv), dtype=torch.float32, device=dev)
    opts = lib.make_opts(lib.DTYPE_BF16)
    ws = lib.alloc_workspace(lib.workspace_bytes(lib.OP_GDN, w.B, w.H, w.F, w.L, w.dk, w.dv, opts), dev)
    stream = torch.cuda.current_stream()

    def step():
        lib.gdn_frame_fwd(q, k, v, a, b, F=w.F, o=o, workspace=ws)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev, world)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    ms_e2e, h2d, d2h, cbound = None, 0, 0, None
    if not args.quick:
        ms_e2e, h2d, d2h, cbound = end_to_end_leg(args, lib, torch, dist, w, dev, stream, world,
                                                  (hq, hk, hv, ha, hb))
    if rank != 0:
        return
    cpu_on = world == 1 and not args.no_cpu_baseline
    del q, k, v, a, b, o, ws
    extra = {}
    if not args.quick:
        extra["relu_la"] = relu_leg(args, lib, synth, torch, dev, stream, cpu_on)
        if not args.no_streaming:
            extra["streaming"] = streaming_leg(args, lib, synth, torch, dev, stream, cpu_on)
        extra["configs_other"] = small_configs_leg(args, lib, synth, torch, dev, stream, cpu_on)
        extra["temporal_conv"] = temporal_conv_leg(args, lib, synth, torch, dev, stream, cpu_on)
        extra["softmax_window"] = softmax_window_leg(args, lib, synth, torch, dev, stream, cpu_on)
        extra["backward"] = backward_leg(args, lib, synth, torch, dev, stream, cpu_on)
        extra["rope"] = rope_leg(args, lib, synth, torch, dev, stream, cpu_on)
    peak, peak_src = measured_peaks()
    alg_bytes = token_heads * BYTES_PER_TOKEN_HEAD + w.B * w.H * (w.F * 4 + w.dk * w.dv * 4)
    achieved = alg_bytes / (ms / 1e3) / 1e9
    tr = ncu_traffic("gdn_tc") if w.F == 240 else None
    line = {
        "metric": METRIC,
        "value": whole_job_tokens_per_s(tokens, world, ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "precision": PRECISION,
        "data": "synthetic",
        "config": {"workload": WORKLOAD if w.F == 240 else f"{WORKLOAD} first {w.F} frames",
                   "B": w.B, "H": w.H, "F": w.F, "L": w.L, "dk": w.dk, "dv": w.dv,
                   "tokens_per_step_per_gpu": tokens, "token_heads_per_step_per_gpu": token_heads,
                   "parallelism": f"dp{world} (independent batch per GPU, no exchange)",
                   "l2": "inputs larger than the 126 MB L2 (2.97 GB per GPU at F=240); no flush needed"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_src} hbm_gbs (headline fraction); frac_vs_8tbs_spec is against the "
                                    f"8 TB/s HBM3e figure", "frac_vs_8tbs_spec": achieved / SPEC_HBM_GBS,
                     "alg_bytes_per_launch": alg_bytes,
                     "traffic": None if tr is None else tr["dram_bytes_per_launch"],
                     "traffic_source": None if tr is None else tr["source"]},
        "gpu_launches": args.steps,
        "kernel": "gdn_tc_kernel (tcgen05/TMEM/TMA, persistent, one CTA per SM)",
        "clocks": clk.summary(),
    }
    if ms_e2e is not None:
        line["e2e"] = {"value": whole_job_tokens_per_s(tokens, world, ms_e2e), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
                       "call": "gdn_frame_fwd_host (C ABI, pinned host buffers, copies + kernel + sync)",
                       "pcie_floor": cbound}
    line.update(extra)
    if cpu_on and not args.quick:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)


def _events_ms(fn, n, stream):
    """Mean device time of fn() over n calls, CUDA events on `stream`."""
    import torch
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n


def _roofline(alg_bytes, ms, peak, peak_src):
    ach = alg_bytes / (ms / 1e3) / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
            "peak_source": f"{peak_src} hbm_gbs", "frac_vs_8tbs_spec": ach / SPEC_HBM_GBS,
            "alg_bytes_per_launch": alg_bytes}


def _gdn_alg_bytes(w, esz=2):
    """Algorithmic bytes of one gdn_frame_fwd call: q, k, v read once, o (fp32)
    written once, gates and the output state."""
    th = w.B * w.H * w.N
    return th * (esz * (2 * w.dk + w.dv) + 4 * w.dv + 4) + w.B * w.H * (w.F * 4 + w.dk * w.dv * 4)


def _oracle_tokens_per_s(fn, tokens, target_s=2.0):
    """Run fn() (one oracle call over `tokens` sequence tokens) until about
    target_s seconds have passed; tokens per second."""
    t0 = time.perf_counter()
    n = 0
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= target_s:
            return tokens * n / dt, n, dt


def end_to_end_leg(args, lib, torch, dist, w, dev, stream, world, host):
    hq, hk, hv, ha, hb = host
    # end to end through the host-buffer C-ABI call (copies inside the timed region)
    ho = torch.empty((w.B, w.H, w.N, w.dv), dtype=torch.float32).pin_memory()
    hopts = lib.make_opts(lib.DTYPE_BF16)
    hws = lib.alloc_workspace(lib.host_workspace_bytes(w.B, w.H, w.F, w.L, w.dk, w.dv, hopts), dev)
    lib.gdn_frame_fwd_host(hq, hk, hv, ha, hb, F=w.F, o=ho, workspace=hws)
    if world > 1:
        dist.barrier()
    n_e2e = max(1, args.e2e_steps)
    ms_e2e = _events_ms(lambda: lib.gdn_frame_fwd_host(hq, hk, hv, ha, hb, F=w.F, o=ho, workspace=hws), n_e2e,
                        stream)
    ms_e2e = max_over_ranks(ms_e2e, dev, world)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, ha, hb))
    d2h = ho.numel() * ho.element_size()
    del hws
    return ms_e2e, h2d, d2h, copy_bound(torch, dev, (hq, hk, hv, ha, hb), ho)


def copy_bound(torch, dev, host_in, host_out):
    """The PCIe floor of the end-to-end leg: the same bytes as plain pinned copies
    (cudaMemcpyAsync through torch), host -> device alone, device -> host alone,
    and both at once on two streams (the link is full duplex)."""
    dins = [torch.empty_like(t, device=dev) for t in host_in]
    dout = torch.empty_like(host_out, device=dev)
    s1, s2 = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def h2d():
        with torch.cuda.stream(s1):
            for d, h in zip(dins, host_in):
                d.copy_(h, non_blocking=True)

    def d2h():
        with torch.cuda.stream(s2):
            host_out.copy_(dout, non_blocking=True)

    def timed(fns):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for fn in fns:
            fn()
        torch.cuda.synchronize()
        return (time.perf_counter() - t0) * 1e3

    h2d(), d2h()
    res = {"h2d_only_ms": min(timed([h2d]) for _ in range(2)), "d2h_only_ms": min(timed([d2h]) for _ in range(2)),
           "both_ms": min(timed([h2d, d2h]) for _ in range(2)),
           "method": "the same bytes as plain pinned cudaMemcpyAsync copies on two streams, host wall clock "
                     "around device syncs, best of 2"}
    del dins, dout
    return res


def relu_leg(args, lib, synth, torch, dev, stream, cpu_baseline_on):
    """The ReLU block-causal mode at its own workload (B=2, H=20, F=81, L=920)."""
    wr = synth.WORKLOADS["relu_720p_81f"]
    xr = synth.inputs(wr)
    rq, rk, rv = (torch.from_numpy(xr[n]).to(torch.bfloat16).to(dev) for n in "qkv")
    ro = torch.empty((wr.B, wr.H, wr.N, wr.dv), dtype=torch.float32, device=dev)
    opts = lib.make_opts(lib.DTYPE_BF16)
    rws = lib.alloc_workspace(lib.workspace_bytes(lib.OP_RELU_LA, wr.B, wr.H, wr.F, wr.L, wr.dk, wr.dv, opts), dev)
    call = lambda: lib.relu_la_block_fwd(rq, rk, rv, F=wr.F, o=ro, workspace=rws)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    rms = _events_ms(call, max(5, args.steps // 2), stream)
    rbytes = wr.B * wr.H * wr.N * (3 * wr.dk * 2 + wr.dv * 4) + wr.B * wr.H * wr.dk * (wr.dv + 1) * 4
    peak, src = measured_peaks()
    roof = _roofline(rbytes, rms, peak, src)
    tr = ncu_traffic("relu_tc")
    roof["traffic"] = None if tr is None else tr["dram_bytes_per_launch"]
    roof["traffic_source"] = None if tr is None else tr["source"]
    out = {"workload": "relu_720p_81f", "B": wr.B, "H": wr.H, "F": wr.F, "L": wr.L, "d": wr.dk, "ms": rms,
           "tokens_per_s": wr.B * wr.N / (rms / 1e3), "roofline": roof,
           "achieved_gbs": rbytes / (rms / 1e3) / 1e9, "frac_hbm": rbytes / (rms / 1e3) / 1e9 / peak,
           "l2": "inputs 2.0 GB, larger than L2; no flush needed"}
    del rq, rk, rv, ro, rws
    if cpu_baseline_on:
        import oracle
        frames = 2
        xs = synth.inputs(wr, frames=frames)
        hx = {n: torch.from_numpy(xs[n]).to(torch.bfloat16).float().numpy() for n in "qkv"}
        nthreads = os.cpu_count() or 1
        tps, n, dt = _oracle_tokens_per_s(
            lambda: oracle.relu_la(hx["q"], hx["k"], hx["v"], F=frames, L=wr.L, nthreads=nthreads),
            wr.B * frames * wr.L)
        out["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": min(nthreads, wr.B * wr.H),
                               "kind": "oracle", "sample": f"all {wr.B * wr.H} heads x first {frames} of {wr.F} "
                                                           f"frames, {n} runs in {dt:.1f} s"}
    return out


def small_configs_leg(args, lib, synth, torch, dev, stream, cpu_baseline_on):
    """The tiny fp32 case (launch latency) and the 480p 5 s shape, each timed
    on its own with CUDA events, with its roofline and the oracle beside it."""
    import oracle
    out = {}
    peak, src = measured_peaks()
    for name in ("tiny_fp32", "gdn_480p_5s"):
        w = synth.WORKLOADS[name]
        x = synth.inputs(w)
        dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
        q, k, v = (torch.from_numpy(x[n]).to(dt).to(dev) for n in "qkv")
        a, b = (torch.from_numpy(x[n]).to(dev) for n in "ab")
        o = torch.empty((w.B, w.H, w.N, w.dv), dtype=torch.float32, device=dev)
        s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
        opts = lib.make_opts(lib.DTYPE_F32 if w.dtype == "f32" else lib.DTYPE_BF16)
        ws = lib.alloc_workspace(lib.workspace_bytes(lib.OP_GDN, w.B, w.H, w.F, w.L, w.dk, w.dv, opts), dev)
        call = lambda: lib.gdn_frame_fwd(q, k, v, a, b, F=w.F, o=o, state_out=s_out, workspace=ws)
        for _ in range(5):
            call()
        torch.cuda.synchronize()
        n = 200 if name == "tiny_fp32" else 50
        # L2 flush between timed calls for the 480p shape (its 184 MB of bytes are close to L2's 126 MB)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if name != "tiny_fp32" else None
        if flush is None:
            ms = _events_ms(call, n, stream)
            l2 = "not flushed (launch-latency case)"
        else:
            tot = 0.0
            for _ in range(n):
                flush.zero_()
                tot += _events_ms(call, 1, stream)
            ms = tot / n
            l2 = "256 MB buffer written between timed calls (L2 flushed)"
        nb = _gdn_alg_bytes(w, 4 if w.dtype == "f32" else 2)
        d = {"workload": name, "B": w.B, "H": w.H, "F": w.F, "L": w.L, "dk": w.dk, "dv": w.dv, "dtype": w.dtype,
             "ms": ms, "us_per_call": ms * 1e3, "tokens_per_s": w.B * w.N / (ms / 1e3),
             "roofline": _roofline(nb, ms, peak, src), "l2": l2}
        if name == "tiny_fp32":
            d["roofline"]["bound"] = "latency"
        if cpu_baseline_on:
            hx = {n_: t.float().cpu().numpy() for n_, t in (("q", q), ("k", k), ("v", v))}
            nthreads = os.cpu_count() or 1
            frames = w.F if name == "tiny_fp32" else 3
            sl = slice(0, frames * w.L)
            tps, runs, secs = _oracle_tokens_per_s(
                lambda: oracle.gdn(hx["q"][:, :, sl], hx["k"][:, :, sl], hx["v"][:, :, sl], x["a"][:, :, :frames],
                                   x["b"][:, :, sl], F=frames, L=w.L, nthreads=nthreads), w.B * frames * w.L)
            d["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                                 "sample": f"all {w.B * w.H} heads x first {frames} of {w.F} frames, {runs} runs "
                                           f"in {secs:.1f} s"}
        out[name] = d
        del q, k, v, a, b, o, s_out, ws, flush
    return out


def streaming_leg(args, lib, synth, torch, dev, stream, cpu_baseline_on):
    """The streaming block-cache decode at the 720p shape, run as the protocol:
    240 frames x 4 denoising steps = 960 calls of one frame (F = 1, 20 heads,
    920 tokens); every step reads the committed state of the previous frame,
    state_out is NULL on steps 1-3 and the 4th step commits the state that the
    next frame reads.  Fresh inputs per call come from a pool of 16 distinct
    calls (200 MB, more than L2), cycled.  Timed with the automatic chunk
    segments and with one CTA per frame (segments = 1)."""
    w = synth.WORKLOADS["gdn_stream_720p"]
    steps, frames, pool_n = w.steps, w.F, 16
    pool = []
    for c in range(pool_n):
        x = synth.inputs(w, call=c)
        pool.append([torch.from_numpy(x[n]).to(torch.bfloat16).to(dev) for n in "qkv"] +
                    [torch.from_numpy(x[n]).to(dev) for n in "ab"])
    o = torch.empty((w.B, w.H, w.L, w.dv), dtype=torch.float32, device=dev)
    sbuf = [torch.zeros((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev) for _ in range(2)]
    calls = frames * steps
    out = {"workload": "gdn_stream_720p", "B": w.B, "H": w.H, "L": w.L, "d": w.dk, "frames": frames,
           "steps_per_frame": steps, "calls_timed": calls,
           "protocol": "state_in = committed state of the previous frame; state_out NULL on steps 1-3, committed "
                       "on step 4",
           "l2": f"inputs cycled from a pool of {pool_n} distinct calls (about 200 MB, more than L2)"}
    peak, src = measured_peaks()
    for tag, segs in (("auto", 0), ("one_cta_per_frame", 1)):
        o_ = lib.make_opts(lib.DTYPE_BF16, segments=segs)
        wsb = lib.alloc_workspace(lib.workspace_bytes(lib.OP_GDN, w.B, w.H, 1, w.L, w.dk, w.dv, o_), dev)

        def protocol(nf):
            cur = 0
            for f in range(nf):
                for st in range(steps):
                    q_, k_, v_, a_, b_ = pool[(f * steps + st) % pool_n]
                    lib.gdn_frame_fwd(q_, k_, v_, a_, b_, F=1, state_in=None if f == 0 else sbuf[cur],
                                      state_out=(sbuf[cur ^ 1] if st == steps - 1 else None), o=o, workspace=wsb,
                                      segments=segs)
                cur ^= 1

        protocol(4)
        torch.cuda.synchronize()
        ms = _events_ms(lambda: protocol(frames), 1, stream)
        out[f"us_per_call_{tag}"] = ms * 1e3 / calls
        out[f"ms_protocol_{tag}"] = ms
        del wsb
    us = out["us_per_call_auto"]
    # bytes per call: q, k, v (bf16), gates, o (fp32), state in (fp32); + state out on one call in 4
    nb = w.B * w.H * (w.L * (3 * w.dk * 2 + 4 + w.dv * 4) + 4 + w.dk * w.dv * 4 * (1 + 1 / steps))
    out.update({"step_tokens_per_s": w.B * w.L / (us / 1e6), "frames_committed_per_s": 1e6 / (us * steps),
                "roofline": _roofline(nb, us / 1e3, peak, src)})
    out["roofline"]["alg_bytes_per_call"] = nb
    if cpu_baseline_on:
        import oracle
        x = synth.inputs(w, call=0)
        hx = {n: torch.from_numpy(x[n]).to(torch.bfloat16).float().numpy() for n in "qkv"}
        S = np.zeros((w.B, w.H, w.dk, w.dv))
        nthreads = os.cpu_count() or 1
        tps, runs, secs = _oracle_tokens_per_s(
            lambda: oracle.gdn(hx["q"], hx["k"], hx["v"], x["a"], x["b"], F=1, L=w.L, state_in=S,
                               nthreads=nthreads), w.B * w.L)
        out["cpu_baseline"] = {"value": tps, "unit": "step tokens/s", "cores": nthreads, "kind": "oracle",
                               "sample": f"one streaming call (20 heads, 920 tokens) repeated {runs} times in "
                                         f"{secs:.1f} s"}
    return out


def temporal_conv_leg(args, lib, synth, torch, dev, stream, cpu_baseline_on):
    """The causal temporal convolution with the block-boundary cache at the 720p
    latent grid and model width (HW = 920, C = 2240, bf16): the whole 60 s clip
    as one block of 240 frames, and the clip generated as 24 blocks of 10
    frames with the cache carried in place from block to block."""
    peak, src = measured_peaks()
    out = {}
    cw = synth.CONV_WORKLOADS["tconv_720p_60s"]
    inp = synth.conv_inputs(cw)
    x = torch.from_numpy(inp["x"]).to(torch.bfloat16).to(dev)
    del inp["x"]
    w_, b_ = torch.from_numpy(inp["w"]).to(dev), torch.from_numpy(inp["bias"]).to(dev)
    cache = torch.zeros((cw.B, cw.HW, cw.C), dtype=torch.bfloat16, device=dev)
    y = torch.empty_like(x)
    call = lambda: lib.temporal_conv_fwd(x, w_, bias=b_, cache_in=cache, cache_out=cache, y=y)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ms = _events_ms(call, max(10, args.steps), stream)
    es = 2
    nb = 2 * es * x.numel() + 2 * es * cache.numel()
    roof = _roofline(nb, ms, peak, src)
    tr = ncu_traffic("temporal_conv")
    roof["traffic"] = None if tr is None else tr["dram_bytes_per_launch"]
    roof["traffic_source"] = None if tr is None else tr["source"]
    out["whole_clip"] = {"workload": cw.name, "B": cw.B, "F": cw.F, "HW": cw.HW, "C": cw.C, "dtype": cw.dtype,
                         "ms": ms, "frames_per_s": cw.B * cw.F / (ms / 1e3),
                         "tokens_per_s": cw.B * cw.F * cw.HW / (ms / 1e3),
                         "roofline": roof,
                         "l2": "x and y 0.99 GB each, larger than L2; no flush needed"}
    del x, y
    sw = synth.CONV_WORKLOADS["tconv_stream_720p"]
    pool_n = 8
    pool = [torch.from_numpy(synth.conv_inputs(sw, block=i)["x"]).to(torch.bfloat16).to(dev) for i in range(pool_n)]
    ys = torch.empty_like(pool[0])
    sc = torch.zeros((sw.B, sw.HW, sw.C), dtype=torch.bfloat16, device=dev)

    def blocks():
        for i in range(sw.blocks):
            lib.temporal_conv_fwd(pool[i % pool_n], w_, bias=b_, cache_in=sc if i else None, cache_out=sc, y=ys)

    blocks()
    torch.cuda.synchronize()
    ms_eager = _events_ms(blocks, 3, stream)
    # the same 24 calls replayed as one CUDA graph: the device time without the
    # Python call overhead between blocks (each call launches one kernel)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        blocks()
    graph.replay()
    torch.cuda.synchronize()
    ms_s = _events_ms(graph.replay, 5, torch.cuda.current_stream())
    del graph
    nbs = sw.blocks * (2 * es * pool[0].numel() + es * sc.numel()) + (sw.blocks - 1) * es * sc.numel()
    out["streaming_blocks"] = {"workload": sw.name, "B": sw.B, "F_per_block": sw.F, "blocks": sw.blocks,
                               "HW": sw.HW, "C": sw.C, "ms_all_blocks": ms_s, "us_per_block": ms_s * 1e3 / sw.blocks,
                               "us_per_block_eager": ms_eager * 1e3 / sw.blocks,
                               "timing": "the 24 calls captured in one CUDA graph and replayed; us_per_block_eager "
                                         "times them as Python calls",
                               "frames_per_s": sw.B * sw.F * sw.blocks / (ms_s / 1e3),
                               "roofline": _roofline(nbs, ms_s, peak, src),
                               "l2": f"blocks cycled from a pool of {pool_n} distinct blocks (330 MB, more than "
                                     f"L2)"}
    del pool, ys, sc
    if cpu_baseline_on:
        import oracle
        n_pos = 92
        xs = synth.conv_inputs(sw, frames=sw.F)["x"][:, :, :n_pos]
        xs = torch.from_numpy(np.ascontiguousarray(xs)).to(torch.bfloat16).float().numpy()
        tps, runs, secs = _oracle_tokens_per_s(lambda: oracle.temporal_conv(xs, inp["w"], bias=inp["bias"]),
                                               sw.B * sw.F * n_pos)
        out["cpu_baseline"] = {"value": tps, "unit": "tokens/s (latent positions x frames, all 2240 channels)",
                               "cores": 1, "kind": "oracle",
                               "sample": f"one block of {sw.F} frames x {n_pos} of {sw.HW} latent positions, "
                                         f"{runs} runs in {secs:.1f} s"}
    return out


def softmax_window_leg(args, lib, synth, torch, dev, stream, cpu_baseline_on):
    """The windowed softmax layer at the 720p 60 s shape (B=1, H=20, F=240, L=920,
    d=112, bf16), window W = 4 latent frames (the current one and three before:
    about one second of the clip).  Bound: tensor cores."""
    B, H, F, L, d, W = 1, 20, 240, 920, 112, 4
    N = F * L
    q, k, v = (torch.from_numpy(synth.normal(7, t, 0, B * H * N * d).reshape(B, H, N, d)).to(torch.bfloat16).to(dev)
               for t in range(3))
    o = torch.empty((B, H, N, d), dtype=torch.float32, device=dev)
    call = lambda: lib.softmax_window_fwd(q, k, v, F=F, W=W, o=o)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ms = _events_ms(call, 5, stream)
    keys = sum(min(f + 1, W) * L for f in range(F))  # keys seen by one query row, summed over a head's frames
    flops = 4.0 * d * B * H * L * keys               # q.k and p.v, 2 flops per multiply-add
    tf = flops / (ms / 1e3) / 1e12
    peak = FALLBACK_BF16_TFLOPS
    mp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    src = "fallback bf16_tflops (burst)"
    if os.path.exists(mp):
        try:
            with open(mp) as f:
                peak = float(json.load(f)["bf16_tflops"])
            src = "measured bf16_tflops (burst)"
        except Exception:
            pass
    out = {"workload": "swa_720p_60s_w4", "B": B, "H": H, "F": F, "L": L, "d": d, "W": W, "ms": ms,
           "tokens_per_s": B * N / (ms / 1e3),
           "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                        "peak_source": src, "alg_flops_per_launch": flops,
                        "traffic": None if ncu_traffic("softmax_window") is None
                        else ncu_traffic("softmax_window")["dram_bytes_per_launch"]},
           "l2": "q, k, v 1.48 GB and o 1.98 GB, larger than L2; no flush needed"}
    del q, k, v, o
    if cpu_baseline_on:
        import oracle
        Fs = 5  # the first five frames of every head (frames 0-3 fill the window)
        def head_prefix(t):  # frames 0..Fs-1 of every head: one contiguous run of the draw per head
            x = np.stack([synth.normal(7, t, h * N * d, Fs * L * d) for h in range(H)]).reshape(B, H, Fs * L, d)
            return torch.from_numpy(x).to(torch.bfloat16).float().numpy()
        qs, ks, vs = (head_prefix(t) for t in range(3))
        nthreads = os.cpu_count() or 1
        tps, runs, secs = _oracle_tokens_per_s(
            lambda: oracle.softmax_window(qs, ks, vs, F=Fs, L=L, W=W, nthreads=nthreads), B * Fs * L, target_s=4.0)
        out["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                               "sample": f"all {H} heads x first {Fs} of {F} frames (windows of 1-4 frames, "
                                         f"below the 4-frame average), {runs} runs in {secs:.1f} s"}
    return out


def backward_leg(args, lib, synth, torch, dev, stream, cpu_baseline_on):
    """gdn_frame_bwd on the headline workload (720p 60 s: B=1, H=20, F=240, L=920,
    d=112, bf16 q, k, v; fp32 dL/do ~ N(0, 1), no start state).  One call =
    the forward recompute, Q^T dO per frame, the adjoint frame chain and the
    frame kernel."""
    w = synth.WORKLOADS["gdn_720p_60s"]
    x = synth.inputs(w)
    q, k, v = (torch.from_numpy(x[n]).to(torch.bfloat16).to(dev) for n in "qkv")
    a, b = (torch.from_numpy(x[n]).to(dev) for n in "ab")
    d_o = torch.from_numpy(synth.grad_inputs(w)["d_o"]).to(dev)
    del x
    opts = lib.make_opts(lib.DTYPE_BF16)
    ws = lib.alloc_workspace(lib.workspace_bytes(lib.OP_GDN_BWD, w.B, w.H, w.F, w.L, w.dk, w.dv, opts), dev)
    out = lib.gdn_frame_bwd(q, k, v, a, b, d_o, F=w.F, workspace=ws)
    call = lambda: lib.gdn_frame_bwd(q, k, v, a, b, d_o, F=w.F, workspace=ws, out=out)
    for _ in range(2):
        call()
    torch.cuda.synchronize()
    ms = _events_ms(call, 3, stream)
    th, fh = w.B * w.H * w.N, w.B * w.H * w.F
    # read q, k, v (bf16), beta and dL/do; write dq, dk, dv and dbeta (fp32); alpha and dalpha per frame
    alg_bytes = th * (2 * (2 * w.dk + w.dv) + 4 + 4 * w.dv + 4 * (2 * w.dk + w.dv) + 4) + fh * 8
    peak, peak_src = measured_peaks()
    res = {"workload": WORKLOAD, "B": w.B, "H": w.H, "F": w.F, "L": w.L, "d": w.dk, "ms": ms,
           "tokens_per_s": w.B * w.N / (ms / 1e3),
           "roofline": dict(_roofline(alg_bytes, ms, peak, peak_src), scope="the whole call (four launches)",
                            frame_kernel_traffic=None if ncu_traffic("gdn_bwd") is None
                            else ncu_traffic("gdn_bwd")["dram_bytes_per_launch"]),
           "launches_per_call": 4,
           "l2": "inputs 2.97 GB and dL/do 1.98 GB, larger than L2; no flush needed"}
    del q, k, v, a, b, d_o, out, ws
    if cpu_baseline_on:
        import oracle
        Fs = 4
        xs = synth.inputs(w, frames=Fs)
        ds = synth.normal(w.seed, synth.TID_DO, 0, w.B * w.H * w.N * w.dv).reshape(w.B, w.H, w.N, w.dv)[:, :, :Fs * w.L]
        qs, ks, vs = (torch.from_numpy(xs[n]).to(torch.bfloat16).float().numpy() for n in "qkv")
        nthreads = os.cpu_count() or 1
        tps, runs, secs = _oracle_tokens_per_s(
            lambda: oracle.gdn_bwd(qs, ks, vs, xs["a"], xs["b"], ds, F=Fs, L=w.L, nthreads=nthreads),
            w.B * Fs * w.L, target_s=4.0)
        res["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                               "sample": f"the backward of the first {Fs} of {w.F} frames of all {w.H} heads, "
                                         f"{runs} runs in {secs:.1f} s"}
    return res


def rope_leg(args, lib, synth, torch, dev, stream, cpu_baseline_on):
    """The headline workload (720p 60 s) with the 3D RoPE on q and k: 920 tokens
    per frame as a 23 x 40 latent grid (grid_w = 40).  The forward is the
    tensor-core kernel's RoPE instantiation (the rotation fused where q and k
    are loaded) after the angle-table kernel; the backward with the embedding
    is timed beside it (one call: table, tensor-core recompute, Q^T dO,
    adjoint chain, frame kernel, the transpose rotation of dq and dk)."""
    w = synth.WORKLOADS["gdn_720p_60s"]
    x = synth.inputs(w)
    q, k, v = (torch.from_numpy(x[n]).to(torch.bfloat16).to(dev) for n in "qkv")
    a, b = (torch.from_numpy(x[n]).to(dev) for n in "ab")
    rope = dict(grid_w=40)
    opts = lib.make_opts(lib.DTYPE_BF16, rope=rope)
    o = torch.empty((w.B, w.H, w.N, w.dv), dtype=torch.float32, device=dev)
    s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    ws = lib.alloc_workspace(lib.workspace_bytes(lib.OP_GDN, w.B, w.H, w.F, w.L, w.dk, w.dv, opts), dev)
    call = lambda: lib.gdn_frame_fwd(q, k, v, a, b, F=w.F, o=o, state_out=s_out, workspace=ws, rope=rope)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ms = _events_ms(call, max(5, args.steps // 2), stream)
    peak, src = measured_peaks()
    # the same algorithmic bytes as without the embedding: the angle table (a few KB) stays in L2
    roof = dict(_roofline(_gdn_alg_bytes(w), ms, peak, src), traffic=None,
                traffic_source="not captured for the RoPE instantiation")
    res = {"workload": f"{WORKLOAD} with the 3D RoPE (grid 23 x 40)", "B": w.B, "H": w.H, "F": w.F, "L": w.L,
           "d": w.dk, "ms": ms, "tokens_per_s": w.B * w.N / (ms / 1e3), "roofline": roof,
           "kernel": "gdn_tc_kernel<0,1,0> after the angle-table kernel", "launches_per_call": 2,
           "l2": "inputs 2.97 GB, larger than L2; no flush needed"}
    del o, s_out, ws
    d_o = torch.from_numpy(synth.grad_inputs(w)["d_o"]).to(dev)
    bopts = lib.make_opts(lib.DTYPE_BF16, rope=rope)
    bws = lib.alloc_workspace(lib.workspace_bytes(lib.OP_GDN_BWD, w.B, w.H, w.F, w.L, w.dk, w.dv, bopts), dev)
    g = lib.gdn_frame_bwd(q, k, v, a, b, d_o, F=w.F, workspace=bws, rope=rope)
    bcall = lambda: lib.gdn_frame_bwd(q, k, v, a, b, d_o, F=w.F, workspace=bws, out=g, rope=rope)
    bcall()
    torch.cuda.synchronize()
    res["backward_ms"] = _events_ms(bcall, 2, stream)
    res["backward_launches_per_call"] = 6
    del q, k, v, a, b, d_o, g, bws
    if cpu_baseline_on:
        import oracle
        frames = 3
        xs = synth.inputs(w, frames=frames)
        hx = {n: torch.from_numpy(xs[n]).to(torch.bfloat16).float().numpy() for n in "qkv"}
        nthreads = os.cpu_count() or 1
        tps, runs, secs = _oracle_tokens_per_s(
            lambda: oracle.gdn(hx["q"], hx["k"], hx["v"], xs["a"], xs["b"], F=frames, L=w.L, nthreads=nthreads,
                               rope=rope), w.B * frames * w.L)
        res["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                               "sample": f"all {w.H} heads x first {frames} of {w.F} frames with the embedding, "
                                         f"{runs} runs in {secs:.1f} s"}
    return res


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.profile_case:
        profile_case(args.profile_case)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
