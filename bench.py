#!/usr/bin/env python
"""Benchmark of the SSM long convolution hot path on B200.

One JSON line on stdout (rank 0).  A step is one pass of the hot path over one
batch: the headline workload is the H3-125M-layer-shaped convolution
(B=8, H=768, L=1024, N=64, fp16 I/O, filter regenerated on the device every
step): one ssm_conv_fwd call, i.e. the filter-generation kernel followed by
the fused tensor-core FFT convolution kernel.  The roofline object describes
the dominant kernel, the fused convolution, timed on its own in the same run.
Rank 0 also times the rest of the metric's range by default ("configs"): the
L = 8192 fused conv, L = 65536 state passing and the H3 mixer, each with its
own roofline and clocks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--others] [--impl ours|reference]

Timing: W untimed warm-up steps; then K steps, each preceded by an L2 flush
(a 256 MiB write then a 256 MiB read, outside the per-step events) and bracketed by events
on the launching stream; a barrier and a synchronize bracket the loop; the
value is the max over ranks.  Multi-GPU runs shard nothing: every rank runs
its own full batch (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fft_long_convolution_flashconv_b200 import workloads as W  # noqa: E402

HEADLINE = "cfg2_conv_f16_B8_H768_L1024"
METRIC = "conv elements/s (B·H·L per sec) and achieved HBM GB/s fraction, L=1K–64K"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
DT_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            return float(json.load(fh)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxs.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sms) if sms else None,
                "sm_max_mhz": max(maxs) if maxs else None,
                "reasons": sorted(reasons), "samples": len(sms)}


# ------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from fft_long_convolution_flashconv_b200 import _lib, api

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    lib = _lib.load()
    wl = W.make(args.workload)
    stream = torch.cuda.current_stream()

    def T(x, dt="f32"):
        td = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[dt]
        return torch.tensor(np.asarray(x), dtype=torch.float64).to(td).to(dev).contiguous()

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rflush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    res = {}
    step_fn, conv_fn, units, alg_bytes, kern_per_step, e2e_fn, e2e_bytes, dom_fn = build_step(wl, T, dev, api, lib)
    # warm-up
    for _ in range(args.warmup):
        step_fn()
    torch.cuda.synchronize()
    # clocks: sample over a sustained-load phase plus the timed loop
    sampler = ClockSampler(local_rank)
    sampler.start()
    t_end = time.time() + args.load_seconds
    while time.time() < t_end:
        for _ in range(20):
            step_fn()
        torch.cuda.synchronize()
    # One step = the library calls of build_step, captured once into a CUDA
    # graph and replayed, so host-side call overhead does not leave the GPU idle
    # inside the timed interval (the same kernels, arguments and stream order).
    graph = None
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step_fn()
        graph.replay()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    wall0 = time.time()
    for i in range(args.steps):
        flush_l2(flush, rflush)
        ev[i][0].record(stream)
        if graph is not None:
            ev[i][1].record(stream)
            graph.replay()
        else:
            conv_fn(ev[i][1])     # records ev[i][1] right before the dominant launch
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.time() - wall0
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(c) for a, b, c in ev]
    tot_ms = sum(step_ms)
    # the dominant kernel on its own: graph-replayed, L2 flushed before each launch
    for _ in range(3):
        dom_fn()
    torch.cuda.synchronize()
    dgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(dgraph):
        dom_fn()
    dgraph.replay()
    torch.cuda.synchronize()
    dom_ms = []
    for i in range(args.steps):
        flush_l2(flush, rflush)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dgraph.replay()
        b.record(stream)
        torch.cuda.synchronize()
        dom_ms.append(a.elapsed_time(b))
    conv_avg = sum(dom_ms) / len(dom_ms)
    tot_ms, conv_avg = max_over_ranks([tot_ms, conv_avg], world, dev)
    ms_per_step = tot_ms / args.steps
    value = job_value(units, world, ms_per_step)

    # end to end through the C ABI with pinned host buffers
    e2e_ms, = max_over_ranks([e2e_fn(args.e2e_steps)], world, dev)
    e2e_val = job_value(units, world, e2e_ms)

    peak, peak_kind = hbm_peak()
    achieved = alg_bytes / (conv_avg / 1e3) / 1e9
    traffic = profiled_traffic(args.workload)
    res.update(dict(
        metric=METRIC, value=value, unit="conv elements/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
        ms_per_step=ms_per_step, higher_is_better=True, scaling="weak", vs_baseline=None,
        dtype="f16" if wl.dtype == "f16" else ("bf16" if wl.dtype == "bf16" else "f32"),
        data="synthetic",
        config=dict(workload=args.workload, B=wl.B, H=wl.H, L=wl.L, N=wl.N, io_dtype=wl.dtype,
                    timing="CUDA-graph replay of the step's library calls" if args.graph else "direct calls",
                    filter="generated on device every step" if "conv" in args.workload else None,
                    arithmetic="tensor-core operands in the I/O type or fp16, fp32 accumulation; "
                               "fp32 register arithmetic and fp32 filter",
                    l2="flushed before every step (256 MiB write + 256 MiB read, outside the per-step events)",
                    parallelism=f"replicas x{world} (rows independent, no collective)"),
        roofline=dict(bound="hbm", achieved=achieved, peak=peak, unit="GB/s", frac=achieved / peak,
                      traffic=traffic, kernel=dominant_kernel_name(wl), peak_source=peak_kind,
                      algorithmic_bytes_per_launch=alg_bytes, avg_launch_ms=conv_avg,
                      step_achieved_gbs=units * 2 * DT_BYTES[wl.dtype] / (ms_per_step / 1e3) / 1e9),
        e2e=dict(value=e2e_val, unit="conv elements/s", h2d_bytes_per_step=e2e_bytes[0],
                 d2h_bytes_per_step=e2e_bytes[1]),
        gpu_launches=kern_per_step * args.steps,
        clocks=clocks, wall_s=wall,
    ))
    if not args.headline_only and rank == 0:
        res["configs"] = secondary_configs(T, dev, api, args, local_rank)
    if args.others and rank == 0:
        res["headline_split"] = split_headline(T, dev, api, args)
    return res


def max_over_ranks(vals, world, device):
    """Element-wise max over ranks of per-rank device timings (ms).  Every rank
    takes this collective step at the same point, so the slowest replica sets
    the job's time."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def job_value(units_per_rank, world, ms_per_step):
    """Whole-job throughput: the units every rank processed per step over the
    (max-over-ranks) step time."""
    return units_per_rank * world / (ms_per_step / 1e3)


def flush_l2(wbuf, rbuf):
    """Outside the timed interval: write 256 MiB (evicts every cached line),
    then read another 256 MiB so that the dirty lines are written back here and
    L2 is left holding clean, unrelated data."""
    wbuf.zero_()
    rbuf.sum()


def build_step(wl, T, dev, api, lib):
    """Return the step closures for a convolution workload.  A step is one
    ssm_conv_fwd call: the filter is regenerated on the device and the fused
    FFT convolution runs (for L >= 1024 both happen in one kernel launch)."""
    import torch
    if not isinstance(wl, W.ConvWorkload) or wl.chunk:
        raise SystemExit("headline workload must be a fused-convolution config")
    u = T(wl.u, wl.dtype)
    dt, lam, Bp, Cp, D = T(wl.dt), T(wl.lam), T(wl.Bp), T(wl.Cp), T(wl.D)
    y = torch.empty_like(u)
    ws = torch.empty(max(int(lib.ssm_conv_workspace(wl.H, wl.L)), 1), dtype=torch.uint8, device=dev)
    s = DT_BYTES[wl.dtype]
    units = wl.B * wl.H * wl.L
    # kernels per ssm_conv_fwd call: the filter kernel then the convolution,
    # except for L >= 1024 with N > 64 (and no tensor-core conv), where the
    # convolution kernel generates the filter itself
    tc_conv = wl.L == 1024 and wl.dtype != "f32"
    launches = 1 if (wl.L >= 1024 and wl.N > 64 and not tc_conv) else 2
    # algorithmic bytes of the dominant kernel (the convolution on a given
    # filter): u read + y write + the fp32 filter read
    alg = units * 2 * s + wl.H * wl.L * 4
    f_given = torch.empty((wl.H, wl.L), dtype=torch.float32, device=dev)

    def step():
        api.ssm_conv_fwd(u, dt, lam, Bp, Cp, D, workspace=ws, out=y)

    def conv(ev_mid):
        ev_mid.record(torch.cuda.current_stream())
        api.ssm_conv_fwd(u, dt, lam, Bp, Cp, D, workspace=ws, out=y)

    def dominant():
        api.fftconv_fwd(u, f_given, D, out=y)

    api.ssm_kernel_gen(dt, lam, Bp, Cp, wl.L, out=f_given)

    # e2e: pinned host input u -> device, one ssm_conv_fwd C-ABI call, result y -> pinned
    # host, every step.  The SSM parameters (dt, lambda, B, C, D) are the layer's weights:
    # they go to the device once, from pinned host memory, before the timed steps.  Steps are
    # pipelined the way a serving loop runs them: step i's input goes up on a copy stream
    # while step i-1 computes, and its result comes back on another copy stream while step
    # i+1 computes (device inputs, outputs and host outputs double-buffered; events order
    # every reuse of a buffer).
    hu = torch.empty(u.shape, dtype=u.dtype, pin_memory=True)
    hu.copy_(u.cpu())
    hp = [x.cpu().pin_memory() for x in (dt, lam, Bp, Cp, D)]
    dp = [torch.empty_like(x, device=dev) for x in hp]
    for a, h in zip(dp, hp):
        a.copy_(h)
    hys = [torch.empty(u.shape, dtype=u.dtype, pin_memory=True) for _ in range(2)]
    dus = [torch.empty_like(u) for _ in range(2)]
    dys = [torch.empty_like(u) for _ in range(2)]
    h2d = hu.numel() * hu.element_size()
    d2h = hys[0].numel() * hys[0].element_size()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def e2e(n):
        cur = torch.cuda.current_stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def run(steps, t0=None):
            if t0 is not None:
                t0.record(cur)
            s_in.wait_stream(cur)
            s_out.wait_stream(cur)
            for i in range(steps):
                b = i % 2
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_comp[b])  # step i-2 has finished reading dus[b]
                    dus[b].copy_(hu, non_blocking=True)
                    ev_in[b].record(s_in)
                cur.wait_event(ev_in[b])
                if i >= 2:
                    cur.wait_event(ev_out[b])  # step i-2's result has left dys[b]
                api.ssm_conv_fwd(dus[b], dp[0], dp[1], dp[2], dp[3], dp[4], workspace=ws, out=dys[b])
                ev_comp[b].record(cur)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[b])
                    hys[b].copy_(dys[b], non_blocking=True)
                    ev_out[b].record(s_out)
            cur.wait_stream(s_in)
            cur.wait_stream(s_out)

        run(4)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        run(n, e0)
        e1.record(cur)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    return step, conv, units, alg, launches, e2e, (h2d, d2h), dominant


def tensor_peak():
    """Dense 16-bit tensor-core peak in TFLOP/s: the measured burst figure (the
    mixer is timed in isolation), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            return float(json.load(fh)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def graph_time(fn, n, flush, rflush, stream):
    """Average CUDA-event time of one call of fn, captured once in a CUDA graph
    and replayed n times, the L2 flushed before every replay (outside the
    events).  Returns (avg_ms, list_of_ms)."""
    import torch
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    g.replay()
    torch.cuda.synchronize()
    ms = []
    for _ in range(n):
        flush_l2(flush, rflush)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b))
    del g
    return sum(ms) / len(ms), ms


def secondary_configs(T, dev, api, args, local_rank):
    """The other workloads of the metric's range (L = 8K fused, L = 64K state
    passing, the H3 mixer), each timed on the device with CUDA events (graph
    replay, L2 flushed before every call), each with its own roofline and the
    clocks sampled while it ran.  The headline line's value stays the L = 1K
    workload."""
    import torch
    out = {}
    peak, peak_kind = hbm_peak()
    tpeak, tpeak_kind = tensor_peak()
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rflush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    n = max(3, args.other_steps)

    def hbm_roof(kernel, nbytes, ms, note):
        a = nbytes / (ms / 1e3) / 1e9
        return dict(bound="hbm", achieved=a, peak=peak, unit="GB/s", frac=a / peak, traffic=None,
                    kernel=kernel, peak_source=peak_kind, algorithmic_bytes_per_launch=nbytes,
                    avg_launch_ms=ms, bytes_note=note)

    # ---- L = 8192 fused block-FFT regime (bf16, B=4, H=1024)
    wl = W.make("cfg3_conv_bf16_B4_H1024_L8192")
    u = T(wl.u, "bf16")
    dt, lam, Bp, Cp, D = T(wl.dt), T(wl.lam), T(wl.Bp), T(wl.Cp), T(wl.D)
    f = torch.empty((wl.H, wl.L), dtype=torch.float32, device=dev)
    y = torch.empty_like(u)
    ws = torch.empty(api.ssm_conv_workspace_bytes(wl.H, wl.L), dtype=torch.uint8, device=dev)
    api.ssm_kernel_gen(dt, lam, Bp, Cp, wl.L, out=f)
    units = wl.B * wl.H * wl.L
    sampler = ClockSampler(local_rank)
    sampler.start()
    ms_conv, _ = graph_time(lambda: api.fftconv_fwd(u, f, D, out=y), n, flush, rflush, stream)
    ms_step, _ = graph_time(lambda: api.ssm_conv_fwd(u, dt, lam, Bp, Cp, D, workspace=ws, out=y), n, flush,
                            rflush, stream)
    clocks = sampler.stop()
    out[wl.name] = dict(
        step="ssm_conv_fwd (filter generated on the device, then the fused conv)",
        step_ms=ms_step, value=units / (ms_step / 1e3), unit="conv elements/s",
        roofline=hbm_roof(dominant_kernel_name(wl), units * 4 + wl.H * wl.L * 4, ms_conv,
                          "u read + y written (bf16) + fp32 filter read, conv on a given filter"),
        clocks=clocks)
    cfg3_ns_per_elem = ms_conv * 1e6 / units
    del u, y, f, ws

    # ---- L = 65536 state passing (fp16, B=1, H=2560, chunk 8192)
    wl = W.make("cfg4_statepass_f16_B1_H2560_L65536_T8192")
    u = T(wl.u, "f16")
    dt, lam, Bp, Cp, D = T(wl.dt), T(wl.lam), T(wl.Bp), T(wl.Cp), T(wl.D)
    y = torch.empty_like(u)
    ws = torch.empty(api.statepass_workspace_bytes(wl.B, wl.H, wl.L, wl.N, wl.chunk), dtype=torch.uint8,
                     device=dev)
    units = wl.B * wl.H * wl.L
    sampler = ClockSampler(local_rank)
    sampler.start()
    ms, _ = graph_time(lambda: api.fftconv_statepass(u, dt, lam, Bp, Cp, D, wl.chunk, workspace=ws, out=y),
                       max(3, n // 2), flush, rflush, stream)
    clocks = sampler.stop()
    out[wl.name] = dict(
        step="fftconv_statepass (chunk filter, chunk convs, end states, carry, initial-state term)",
        step_ms=ms, value=units / (ms / 1e3), unit="conv elements/s",
        roofline=hbm_roof("the whole state-passing step", units * 4, ms, "u read + y written (fp16)"),
        per_elem_vs_L8192_conv=(ms * 1e6 / units) / cfg3_ns_per_elem,
        clocks=clocks)
    del u, y, ws

    # ---- H3 mixer (fp16, B=8, L=2048, 12 heads x 64)
    mw = W.make("cfg5_h3mixer_f16_B8_L2048_d768")
    q, k, v = T(mw.q, "f16"), T(mw.k, "f16"), T(mw.v, "f16")
    Cs, dt, lam, Bp, Cp, D = T(mw.Cshift), T(mw.dt), T(mw.lam), T(mw.Bp), T(mw.Cp), T(mw.D)
    o = torch.empty_like(q)
    ws = torch.empty(api.h3_mixer_workspace_bytes(mw.B, mw.L, mw.heads, mw.head_dim, mw.N), dtype=torch.uint8,
                     device=dev)
    sampler = ClockSampler(local_rank)
    sampler.start()
    ms, _ = graph_time(lambda: api.h3_mixer_fwd(q, k, v, Cs, dt, lam, Bp, Cp, D, mw.heads, workspace=ws, out=o),
                       n, flush, rflush, stream)
    clocks = sampler.stop()
    flops = 2.0 * 2.0 * mw.B * mw.heads * (mw.L * (mw.L + 1) / 2) * mw.head_dim
    units = mw.B * mw.L * mw.heads * mw.head_dim
    tf = flops / (ms / 1e3) / 1e12
    out[mw.name] = dict(
        step="h3_mixer_fwd (filters, shift SSM, Toeplitz-form mixer)", step_ms=ms,
        value=units / (ms / 1e3), unit="output elements/s",
        roofline=dict(bound="tensor", achieved=tf, peak=tpeak, unit="TFLOP/s", frac=tf / tpeak, traffic=None,
                      kernel="the whole mixer call", peak_source=tpeak_kind, algorithmic_flops=flops,
                      avg_launch_ms=ms, flops_note="causal half of S = Q K~^T and O = P V per (b, head)"),
        hbm_frac=(4 * units * 2) / 1e9 / (ms / 1e3) / peak,
        clocks=clocks)
    del q, k, v, o, ws

    # ---- long arbitrary filter at an EEG-clip length (fp32, B=8, H=256, L=12000): fftconv_long_fwd
    B, H, L = 8, 256, 12000
    rng = np.random.default_rng(12000)
    u = T(rng.normal(size=(B, H, L)).astype(np.float32))
    f = T((rng.normal(size=(H, L)) * np.exp(-np.arange(L) / 4000.0)).astype(np.float32))
    D = T(rng.normal(size=H).astype(np.float32))
    y = torch.empty_like(u)
    ws = torch.empty(max(1, api.long_conv_workspace_bytes(B, H, L)), dtype=torch.uint8, device=dev)
    units = B * H * L
    sampler = ClockSampler(local_rank)
    sampler.start()
    ms, _ = graph_time(lambda: api.fftconv_long_fwd(u, f, D, out=y, workspace=ws), n, flush, rflush, stream)
    clocks = sampler.stop()
    out["longconv_f32_B8_H256_L12000"] = dict(
        step="fftconv_long_fwd (arbitrary filter as long as the clip, four-step FFT, fp32)", step_ms=ms,
        value=units / (ms / 1e3), unit="conv elements/s",
        roofline=hbm_roof("the whole long-convolution call", units * 8 + H * L * 4, ms,
                          "u read + y written (fp32) + fp32 filter read"),
        clocks=clocks)
    return out


def split_headline(T, dev, api, args):
    """The headline step's two kernels timed separately (filter, then conv)."""
    import torch
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rflush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    wl = W.make(HEADLINE)
    u = T(wl.u, "f16")
    dt, lam, Bp, Cp, D = T(wl.dt), T(wl.lam), T(wl.Bp), T(wl.Cp), T(wl.D)
    f = torch.empty((wl.H, wl.L), dtype=torch.float32, device=dev)
    y = torch.empty_like(u)
    ms_gen, _ = graph_time(lambda: api.ssm_kernel_gen(dt, lam, Bp, Cp, wl.L, out=f), args.other_steps, flush,
                           rflush, stream)
    ms_conv, _ = graph_time(lambda: api.fftconv_fwd(u, f, D, out=y), args.other_steps, flush, rflush, stream)
    return {wl.name + " (separate kernels)": dict(gen_ms=ms_gen, conv_ms=ms_conv)}


def profiled_traffic(workload):
    """DRAM bytes per conv launch from a committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "fftconv_traffic.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
    except Exception:
        return None
    if d.get("workload") != workload or d.get("source_sha1") != kernel_source_sha1():
        return None
    return d.get("dram_bytes_per_launch")


def dominant_kernel_name(wl):
    if wl.dtype != "f32" and wl.L == 1024:
        return "fftconv_tc_kernel (tensor-core fused block-FFT conv, L = 1024, given filter)"
    if wl.dtype != "f32" and wl.L in (2048, 4096, 8192):
        return "fftconv_tcl_kernel (tensor-core fused block-FFT conv, L = 2K..8K, given filter)"
    return "fftconv_kernel (CUDA-core fused FFT conv, given filter)"


def kernel_source_sha1():
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "fft_long_convolution_flashconv_b200", "csrc")
    for name in ("fftconv_tc.cu", "fftconv_tc_long.cu", "fftconv_impl.cuh", "fft_stockham.cuh", "common.cuh",
                 "tc100.cuh"):
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


# ------------------------------------------------------------------------- oracle arm
def oracle_sample(wl, rows_per_step):
    """One bounded sample of the headline workload on the CPU oracle: filter
    generation for the channels touched + the direct causal convolution of
    ``rows_per_step`` rows (fp64)."""
    from oracle import cref
    from oracle import ssm_oracle as O
    rows = np.arange(rows_per_step) % (wl.B * wl.H)
    bs, hs = rows // wl.H, rows % wl.H
    uh = np.unique(hs)
    t0 = time.perf_counter()
    f = O.ssm_filter(wl.dt[uh], wl.lam[uh], wl.Bp[uh], wl.Cp[uh], wl.L)
    fmap = {h: i for i, h in enumerate(uh)}
    u = wl.u[bs, hs][None]                                     # 1 x rows x L
    fr = f[[fmap[h] for h in hs]]
    cref.causal_conv(u, fr, wl.D[hs].astype(np.float64))
    return time.perf_counter() - t0, len(rows) * wl.L


def cpu_baseline(wl, target_s):
    from oracle import cref
    dt, n = oracle_sample(wl, 64)
    rows = int(min(wl.B * wl.H, max(64, 64 * target_s / max(dt, 1e-6))))
    dt, n = oracle_sample(wl, rows)
    return dict(value=n / dt, unit="conv elements/s", cores=cref.num_threads(), kind="oracle",
                sample=f"{rows} rows of {wl.name} (filter generation for their channels + fp64 direct "
                       f"causal convolution, plain C with OpenMP), {dt:.1f} s")


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from oracle import cref
    wl = W.make(args.workload)
    rows = max(8, int(args.ref_rows))
    for _ in range(args.warmup):
        oracle_sample(wl, 8)
    tot, units = 0.0, 0
    for _ in range(args.steps):
        dt, n = oracle_sample(wl, rows)
        tot += dt
        units += n
    value = units / tot
    return dict(metric=METRIC, value=value, unit="conv elements/s", n_gpus=world, steps=args.steps,
                warmup=args.warmup, ms_per_step=tot / args.steps * 1e3, higher_is_better=True, scaling="weak",
                vs_baseline=None, dtype="f64", data="synthetic", impl="reference",
                config=dict(workload=args.workload, B=wl.B, H=wl.H, L=wl.L, N=wl.N, io_dtype=wl.dtype,
                            timing="host wall clock around each oracle sample (the oracle runs on the CPU)",
                            note=f"each step is a bounded sample of {rows} rows on the CPU oracle"),
                cpu_baseline=dict(value=value, unit="conv elements/s", cores=cref.num_threads(), kind="oracle",
                                  sample=f"{rows} rows per step of {wl.name}"),
                e2e=dict(value=value, unit="conv elements/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the L=8K, L=64K and mixer workloads (rank 0 times them by default)")
    ap.add_argument("--others", action="store_true", help="also time the headline's two kernels separately")
    ap.add_argument("--other-steps", type=int, default=10)
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--load-seconds", type=float, default=1.5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-rows", type=int, default=512)
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time direct library calls instead of a CUDA-graph replay of them")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("for --gpus N > 1 launch with torch.distributed.run --nproc-per-node N")
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(W.make(args.workload), args.cpu_seconds)
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
