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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN frame-recurrence tokens/s (720p-60s shape, bf16) and % of roofline"
WORKLOAD = "gdn_720p_60s"
FALLBACK_HBM_GBS = 6650.0
# algorithmic bytes per token-head: q, k, v bf16 (3 * 112 * 2) + o fp32 (112 * 4) + beta fp32
BYTES_PER_TOKEN_HEAD = 3 * 112 * 2 + 112 * 4 + 4
FLOPS_PER_TOKEN_HEAD = 6 * 112 * 112


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
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in ("gdn_tc.cu", "tc_ptx.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "linear_attention_video_gdn_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic():
    """DRAM bytes per launch of the GDN kernel from the committed ncu summary, if it
    was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "gdn_tc_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if d.get("kernel_source_sha") == kernel_source_hash():
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

    ms_e2e, h2d, d2h, relu = None, 0, 0, None
    if not args.quick:
        ms_e2e, h2d, d2h, relu = end_to_end_and_relu(args, lib, synth, torch, dist, w, dev, stream, world, rank,
                                                     (hq, hk, hv, ha, hb), opts)
    if rank != 0:
        return
    peak, peak_src = measured_peaks()
    alg_bytes = token_heads * BYTES_PER_TOKEN_HEAD + w.B * w.H * (w.F * 4 + w.dk * w.dv * 4)
    achieved = alg_bytes / (ms / 1e3) / 1e9
    tr = ncu_traffic() if w.F == 240 else None
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
        "precision": "bf16 q/k/v, fp16 tensor-core operands, fp32 accumulation, fp32 state and output",
        "data": "synthetic",
        "config": {"workload": WORKLOAD if w.F == 240 else f"{WORKLOAD} first {w.F} frames",
                   "B": w.B, "H": w.H, "F": w.F, "L": w.L, "dk": w.dk, "dv": w.dv,
                   "tokens_per_step_per_gpu": tokens, "token_heads_per_step_per_gpu": token_heads,
                   "parallelism": f"dp{world} (independent batch per GPU, no exchange)",
                   "l2": "inputs larger than the 126 MB L2 (2.97 GB per GPU at F=240); no flush needed"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_src} hbm_gbs", "alg_bytes_per_launch": alg_bytes,
                     "traffic": None if tr is None else tr["dram_bytes_per_launch"],
                     "traffic_source": None if tr is None else tr["source"]},
        "gpu_launches": args.steps,
        "kernel": "gdn_tc_kernel (tcgen05/TMEM/TMA, persistent, one CTA per SM)",
        "clocks": clk.summary(),
    }
    if ms_e2e is not None:
        line["e2e"] = {"value": whole_job_tokens_per_s(tokens, world, ms_e2e), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
                       "call": "gdn_frame_fwd_host (C ABI, pinned host buffers, copies + kernel + sync)"}
    if relu is not None:
        streaming = relu.pop("streaming", None)
        line["relu_la"] = relu
        if streaming is not None:
            line["streaming"] = streaming
    if world == 1 and not args.no_cpu_baseline and not args.quick:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)


def end_to_end_and_relu(args, lib, synth, torch, dist, w, dev, stream, world, rank, host, opts):
    hq, hk, hv, ha, hb = host
    # end to end through the host-buffer C-ABI call (copies inside the timed region)
    ho = torch.empty((w.B, w.H, w.N, w.dv), dtype=torch.float32).pin_memory()
    hopts = lib.make_opts(lib.DTYPE_BF16)
    hws = lib.alloc_workspace(lib.host_workspace_bytes(w.B, w.H, w.F, w.L, w.dk, w.dv, hopts), dev)
    lib.gdn_frame_fwd_host(hq, hk, hv, ha, hb, F=w.F, o=ho, workspace=hws)
    if world > 1:
        dist.barrier()
    n_e2e = max(1, args.e2e_steps)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(n_e2e):
        lib.gdn_frame_fwd_host(hq, hk, hv, ha, hb, F=w.F, o=ho, workspace=hws)
    t1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(t0.elapsed_time(t1) / n_e2e, dev, world)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, ha, hb))
    d2h = ho.numel() * ho.element_size()
    del hws

    # the ReLU block-causal mode at its own workload (reported beside the headline)
    relu = None
    if rank == 0:
        wr = synth.WORKLOADS["relu_720p_81f"]
        xr = synth.inputs(wr)
        rq, rk, rv = (torch.from_numpy(xr[n]).to(torch.bfloat16).to(dev) for n in "qkv")
        ro = torch.empty((wr.B, wr.H, wr.N, wr.dv), dtype=torch.float32, device=dev)
        rws = lib.alloc_workspace(lib.workspace_bytes(lib.OP_RELU_LA, wr.B, wr.H, wr.F, wr.L, wr.dk, wr.dv, opts), dev)
        for _ in range(3):
            lib.relu_la_block_fwd(rq, rk, rv, F=wr.F, o=ro, workspace=rws)
        torch.cuda.synchronize()
        r0 = torch.cuda.Event(enable_timing=True)
        r1 = torch.cuda.Event(enable_timing=True)
        nr = max(5, args.steps // 2)
        r0.record(stream)
        for _ in range(nr):
            lib.relu_la_block_fwd(rq, rk, rv, F=wr.F, o=ro, workspace=rws)
        r1.record(stream)
        torch.cuda.synchronize()
        rms = r0.elapsed_time(r1) / nr
        rbytes = wr.B * wr.H * wr.N * (3 * wr.dk * 2 + wr.dv * 4)
        peak, _ = measured_peaks()
        relu = {"workload": "relu_720p_81f", "ms": rms, "tokens_per_s": wr.B * wr.N / (rms / 1e3),
                "achieved_gbs": rbytes / (rms / 1e3) / 1e9, "frac_hbm": rbytes / (rms / 1e3) / 1e9 / peak}
        del rq, rk, rv, ro, rws
        relu["streaming"] = None
        if not args.no_streaming:
            relu["streaming"] = streaming_leg(lib, synth, torch, dev, stream)
    return ms_e2e, h2d, d2h, relu


def streaming_leg(lib, synth, torch, dev, stream):
    """Streaming decode at the 720p shape: one frame per call (F = 1, 20 heads,
    920 tokens), 4 calls per frame with fresh q, k, v and gates, the state
    committed by the 4th.  Timed over 20 frames with the automatic chunk
    segments and with one CTA per frame (segments = 1)."""
    ws_ = synth.WORKLOADS["gdn_stream_720p"].with_(F=1)
    calls = []
    for c in range(8):  # 8 calls' inputs, cycled (about 100 MB)
        x = synth.inputs(ws_, call=c)
        calls.append([torch.from_numpy(x[n]).to(torch.bfloat16).to(dev) for n in "qkv"] +
                     [torch.from_numpy(x[n]).to(dev) for n in "ab"])
    o = torch.empty((ws_.B, ws_.H, ws_.L, ws_.dv), dtype=torch.float32, device=dev)
    s_in = torch.zeros((ws_.B, ws_.H, ws_.dk, ws_.dv), dtype=torch.float32, device=dev)
    s_out = torch.empty_like(s_in)
    out = {"workload": "gdn_stream_720p (F=1 per call, 4 calls per frame)", "frames_timed": 20}
    for tag, segs in (("auto", 0), ("one_cta_per_frame", 1)):
        o_ = lib.make_opts(lib.DTYPE_BF16, segments=segs)
        wsb = lib.alloc_workspace(lib.workspace_bytes(lib.OP_GDN, ws_.B, ws_.H, 1, ws_.L, ws_.dk, ws_.dv, o_), dev)

        def frame(i):
            for st in range(4):
                q_, k_, v_, a_, b_ = calls[(4 * i + st) % 8]
                lib.gdn_frame_fwd(q_, k_, v_, a_, b_, F=1, state_in=s_in, state_out=(s_out if st == 3 else None),
                                  o=o, workspace=wsb, segments=segs)

        for i in range(3):
            frame(i)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(20):
            frame(i)
        t1.record(stream)
        torch.cuda.synchronize()
        out[f"us_per_call_{tag}"] = t0.elapsed_time(t1) / 80 * 1e3
    us = out["us_per_call_auto"]
    # bytes per call: q, k, v (bf16), gates, o (fp32), state in (fp32); +state out on one call in 4
    nb = ws_.B * ws_.H * (ws_.L * (3 * ws_.dk * 2 + 4 + ws_.dv * 4) + 4 + ws_.dk * ws_.dv * 4 * 1.25)
    peak, _ = measured_peaks()
    out.update({"frame_tokens_per_s": ws_.B * ws_.L / (us / 1e6), "alg_bytes_per_call": nb,
                "achieved_gbs": nb / (us / 1e6) / 1e9, "frac_hbm": nb / (us / 1e6) / 1e9 / peak,
                "l2": "not flushed; the call is latency-bound (its bytes take about 3 us of HBM time)"})
    return out


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank)
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
