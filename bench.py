"""Throughput of the sink-window attention hot path on B200.

Workload (one "step"): one 40-frame prompt segment of the 240 s stream —
30 attention layers, H=12, D=128, 1560 tokens per latent frame (30x52 grid),
3 sink + 9 local frames, LoL jitter sigma=0.8 — in steady state: the segment
opens with a prompt switch (KV recache of all 30 layers: K = RoPE(RMSNorm(X
Wk)), V = X Wv for the 12 cached frames, X [18720, 1536]), then for each of
the 40 latent frames and each of the 30 layers, RoPE + append of the frame's
K/V into the layer's sink+ring cache and sink-window attention of the
frame's 1560 queries over the 12 cached frames (18720 keys). Inputs are
seeded synthetic tensors, N(0,1)*0.5, from per-layer pools of 16 frames
resident in HBM; the 30 caches (3.45 GB in bf16) exceed L2, so no L2 flush is
needed between steps.

Metric: latent frames/s through the 30-layer attention stack; the attention
kernel's achieved TFLOP/s against the measured dense-bf16 peak goes in
"roofline".

The line also carries the same stream over an E4M3 KV cache (fp8_stream:
bf16 staging copy, then the bf16 kernel; fp8_mma_stream: the FP8 tensor-core
attention), the recache kernel's TFLOP/s and the separate RoPE and append
entry points' HBM figures.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       [--cache bf16|fp8] [--layers L] [--separate] [--no-fp8-stream] [--no-cpu-baseline]
       python bench.py --mode attention|recache|append|rope [--workload wan|chunk] [--cache ...]
Under torchrun each rank runs an independent replica (no collective on the
data path; "replicas only"); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import swa_workloads as W  # noqa: E402

METRIC = "latent frames/s (30-layer attn stack) + sink-window attn TFLOP/s vs B200 peak"
UNIT = "latent frames/s"
SEGMENT = 40          # frames per prompt segment (a KV recache every 40 frames)
POOL = 16             # distinct input frames per layer


def attention_flops(w: W.Workload) -> float:
    """Algorithmic FLOPs of one layer-step of attention at steady state:
    Q K^T and P V, 2 * Nq * Nk * D each, per head."""
    nq = w.N * w.query_frames
    nk = w.slots * w.N
    return 4.0 * nq * nk * w.D * w.H


def recache_flops(w: W.Workload) -> float:
    """Algorithmic FLOPs of one layer's recache: X [S*N, d_model] times
    [Wk | Wv] [d_model, 2*H*D] (the RMSNorm and RoPE epilogue not counted)."""
    return 2.0 * (w.slots * w.N) * w.dm * (2 * w.H * w.D)


def append_bytes(w: W.Workload, cache_elem: int) -> float:
    """Algorithmic HBM bytes of one append: read K, V (bf16) and write them to the cache."""
    n = w.N * w.H * w.D
    scales = 2 * w.N * w.H * 4 if cache_elem == 1 else 0
    return 2 * n * 2 + 2 * n * cache_elem + scales


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_index, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        # the median over every sample taken while the timed region ran
        med = statistics.median(sm) if sm else None
        return {"sm_mhz": med, "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


def gpu_index_for(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return ids[local_rank]
    return str(local_rank)


def replica_seed_offset(rank: int) -> int:
    """Replicas stream different synthetic inputs: rank r offsets every layer
    seed by 1000 r (30 layers per rank, so no two ranks share a seed)."""
    return 1000 * rank


def layer_seed_base(w: W.Workload, layer: int, seed_offset: int) -> int:
    """Seed of one layer's Q/K/V input pools (the pools use base + 1, 2, 3)."""
    return (w.seed * 1_000_003 + (layer + seed_offset) * 10_007) & ((1 << 62) - 1)


def max_over_ranks(value: float, dist: bool, device: str = "cuda") -> float:
    """The slowest rank's device time. Every rank calls it at the same point
    (one collective, same order on all ranks); without a process group it is
    the identity."""
    if not dist:
        return value
    import torch.distributed as tdist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
class Stream:
    """30 layers of caches and input pools on one GPU."""

    def __init__(self, w: W.Workload, cache_dtype: str, device: str, seed_offset: int = 0, fused: bool = True,
                 fp8_mma: bool = False):
        import sink_window_attention_b200 as swa
        self.swa = swa
        self.fused = fused and not fp8_mma  # ll_append_and_attend instead of append, then attention
        # E4M3 cache read by the FP8 tensor-core attention (ll_sink_window_attention_fp8_mma) after the append
        self.fp8_mma = fp8_mma and cache_dtype == "fp8"
        self.w = w
        self.device = device
        self.layers = w.layers
        eps = w.eps
        self.rope = swa.Rope(pairs=w.pairs, grid_h=w.grid_h, grid_w=w.grid_w, theta0=w.theta0, sigma_t=w.sigma_t,
                             eps=None if eps is None else [float(e) for e in eps], t_offset=w.t_offset)
        self.caches = [swa.KVCache(1, w.H, w.D, w.N, cache_dtype, device=device) for _ in range(self.layers)]
        shape = (POOL, 1, w.N, w.H, w.D)
        self.q, self.k, self.v = [], [], []
        for l in range(self.layers):
            base = layer_seed_base(w, l, seed_offset)
            self.q.append(W.normal(shape, base + 1, w.qkv_scale, torch.bfloat16, device))
            self.k.append(W.normal(shape, base + 2, w.qkv_scale, torch.bfloat16, device))
            self.v.append(W.normal(shape, base + 3, w.qkv_scale, torch.bfloat16, device))
        self.out = torch.empty((1, w.N, w.H, w.D), dtype=torch.bfloat16, device=device)
        # prompt-switch inputs per layer: hidden states of the 12 cached frames and the projections
        dm = w.dm
        self.rx, self.rwk, self.rwv, self.rg = [], [], [], []
        for l in range(self.layers):
            base = (w.seed * 7_919 + (l + seed_offset) * 104_729) & ((1 << 62) - 1)
            self.rx.append(W.normal((1, w.slots * w.N, dm), base + 1, 1.0, torch.bfloat16, device))
            self.rwk.append(W.normal((dm, w.H * w.D), base + 2, 1.0 / math.sqrt(dm), torch.bfloat16, device))
            self.rwv.append(W.normal((dm, w.H * w.D), base + 3, 1.0 / math.sqrt(dm), torch.bfloat16, device))
            self.rg.append(W.uniform((w.H * w.D,), base + 4, 0.5, 1.5, torch.float32, device))
        # fill every slot once so the segments below run in steady state
        for l in range(self.layers):
            for f in range(w.slots):
                swa.kvcache_append(self.caches[l], self.k[l][f % POOL], self.v[l][f % POOL], f, self.rope)
        torch.cuda.synchronize()

    def held_frames(self, last: int):
        """Frame held by each occupied cache slot once frames 0..last are
        written (the library's slot map over the sinks and the last ring's
        worth of frames)."""
        w = self.w
        held = [-1] * w.slots
        for f in list(range(min(w.n_sink, last + 1))) + list(range(max(w.n_sink, last - w.n_local + 1), last + 1)):
            held[self.swa.slot_of_frame(f, w.n_sink, w.n_local)] = f
        return [f for f in held if f >= 0]

    def switch(self, first: int, recache_events=None) -> int:
        """Prompt switch before frame `first`: the KV recache of every layer
        (the cached frames re-projected from their hidden states with the new
        prompt's projections). Returns the number of launches."""
        swa = self.swa
        held = self.held_frames(first - 1)
        if recache_events is not None:
            recache_events[0].record()
        for l in range(self.layers):
            swa.kv_recache(self.caches[l], self.rx[l], self.rwk[l], self.rwv[l], self.rg[l], 1e-6, held, self.rope)
        if recache_events is not None:
            recache_events[1].record()
            recache_events[2].append((recache_events[0], recache_events[1]))
            recache_events[0] = torch.cuda.Event(enable_timing=True)
            recache_events[1] = torch.cuda.Event(enable_timing=True)
        return self.layers

    def frames(self, first: int, last: int, attn_events=None, qkv=None, on_output=None) -> int:
        """Frames first .. last-1 through every layer: per frame and layer,
        RoPE + append of the frame's K/V and attention of its queries (one
        fused launch for a bf16 cache; append, then attention for an FP8
        cache). on_output(f, layer, out) sees each attention output before
        the next launch overwrites it. Returns the number of launches."""
        swa = self.swa
        launches = 0
        for f in range(first, last):
            for l in range(self.layers):
                if qkv is None:
                    q, k, v = self.q[l][f % POOL], self.k[l][f % POOL], self.v[l][f % POOL]
                else:
                    q, k, v = qkv(f, l)
                fused = self.fuses(l)
                if not fused:
                    swa.kvcache_append(self.caches[l], k, v, f, self.rope)
                    launches += 1
                if attn_events is not None:
                    attn_events[0].record()
                if fused:  # append + attention in one kernel
                    swa.append_and_attend(self.caches[l], k, v, q, f, self.rope, out=self.out)
                elif self.fp8_mma:
                    swa.sink_window_attention_fp8_mma(q, self.caches[l], f, self.rope, out=self.out)
                else:
                    swa.sink_window_attention(q, self.caches[l], f, self.rope, out=self.out)
                launches += self.attention_launches(l)
                if attn_events is not None:
                    attn_events[1].record()
                    attn_events[2].append((attn_events[0], attn_events[1]))
                    attn_events[0] = torch.cuda.Event(enable_timing=True)
                    attn_events[1] = torch.cuda.Event(enable_timing=True)
                if on_output is not None:
                    on_output(f, l, self.out)
        return launches

    def fuses(self, layer: int) -> bool:
        """Whether this layer's frames run through ll_append_and_attend (one
        launch for a bf16 or f32 cache; for an E4M3 cache the append with the
        staging dequantisation, then the attention kernel)."""
        return self.fused

    def attention_launches(self, layer: int) -> int:
        """Kernel launches of one attention call on this layer's cache (an
        E4M3 cache: the staging dequantisation (fused: with the append), or
        the V-scale pass of the FP8 tensor-core attention, then the attention
        kernel)."""
        return 2 if self.caches[layer].dtype == "fp8" else 1

    def step(self, seg: int, attn_events=None, recache_events=None) -> int:
        """One 40-frame segment: frames 40*(seg+1) .. 40*(seg+1)+39, opened by
        a prompt switch (recache of every layer)."""
        first = SEGMENT * (seg + 1)
        launches = self.switch(first, recache_events)
        return launches + self.frames(first, first + SEGMENT, attn_events)


def run_ours(args, rank, world, local_rank):
    torch.cuda.set_device(local_rank)
    from sink_window_attention_b200 import build
    build.build()
    import sink_window_attention_b200 as swa
    w = W.STREAM if args.cache == "bf16" else W.STREAM_FP8
    w = W.replace(w, layers=args.layers)
    st = Stream(w, "bf16" if args.cache == "bf16" else "fp8", "cuda", seed_offset=replica_seed_offset(rank),
                fused=not args.separate)
    fused = st.fuses(0)
    dist = world > 1
    if dist:
        import torch.distributed as tdist

    def barrier():
        torch.cuda.synchronize()
        if dist:
            tdist.barrier()

    for s in range(args.warmup):
        st.step(s)
    barrier()
    clocks = ClockSampler(gpu_index_for(local_rank))
    if rank == 0:
        clocks.start()
    ev = [torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True), []]
    rev = [torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True), []]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    barrier()
    t0.record()
    launches = 0
    for s in range(args.steps):
        launches += st.step(args.warmup + s, attn_events=ev, recache_events=rev)
    t1.record()
    barrier()
    clk = clocks.stop() if rank == 0 else None
    ms = t0.elapsed_time(t1)
    attn_ms = [a.elapsed_time(b) for a, b in ev[2]]
    dev_err = swa.device_error()
    if dev_err:
        raise RuntimeError(f"device error word {dev_err}")
    ms = max_over_ranks(ms, dist)

    # ---- end to end through the public API with host buffers (pinned), per step:
    # every frame's Q/K/V of every layer is copied host -> device on a copy
    # stream (double-buffered against compute), and each frame's last-layer
    # output is read back.
    e2e = run_e2e(st, args, barrier, dist)

    frames = SEGMENT * args.steps * world
    value = frames / (ms / 1e3)
    peaks, kind = measured_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    avg_attn_s = (sum(attn_ms) / len(attn_ms)) / 1e3
    fl = attention_flops(w)
    achieved = fl / avg_attn_s / 1e12
    # the timed launch is the fused append + attention in the default stream
    traffic_capture = ("attention_fused_stream" if fused else "attention_wan_single_layer") + (
        "_fp8" if args.cache == "fp8" else "")
    traffic = load_traffic(traffic_capture)
    recache_ms = [a.elapsed_time(b) for a, b in rev[2]]
    rc_layer_s = (sum(recache_ms) / len(recache_ms)) / 1e3 / w.layers
    rc_flops = recache_flops(w)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if args.cache == "bf16" else "bf16+fp8kv",
        "data": "synthetic",
        "config": {"workload": f"240s stream segment: {SEGMENT} latent frames x {w.layers} layers, H=12 D=128, "
                               f"1560 tok/frame, 3 sink + 9 local, LoL jitter 0.8, {args.cache} KV cache",
                   "frames_per_step": SEGMENT, "layers": w.layers, "tokens_per_frame": w.N, "keys": w.slots * w.N,
                   "heads": w.H, "head_dim": w.D, "kv_cache": args.cache,
                   "recache": f"all {w.layers} layers at the segment start (X [{w.slots * w.N}, {w.dm}])",
                   "l2": "inputs larger than L2 (30 caches x 115 MB)", "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "kernel": "sink_window_attention_kernel" + (
                         " (the frame's RoPE + append fused in: ll_append_and_attend)" if fused and args.cache != "fp8"
                         else " (+ the E4M3 append and bf16 staging kernel inside the timed call)"
                         if args.cache == "fp8" else ""),
                     "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "traffic_source": (f"ncu capture '{traffic_capture}' of this kernel version "
                                        "(profiles/traffic.json), not measured in this run"
                                        if traffic is not None else "no capture of this kernel version"),
                     "peak_kind": f"{kind} bf16 dense, sustained",
                     "algorithmic_flops_per_launch": fl, "avg_launch_us": round(avg_attn_s * 1e6, 2),
                     # the launch time in SM clock cycles at the run's median clock: separates a
                     # slower clock (power cap) from more work per launch when runs are compared
                     "avg_launch_kcycles_at_median_clock": (round(avg_attn_s * clk["sm_mhz"] * 1e3, 1)
                                                            if clk and clk.get("sm_mhz") else None)},
        "recache_kernel": {"achieved_tflops": round(rc_flops / rc_layer_s / 1e12, 1),
                           "us_per_layer": round(rc_layer_s * 1e6, 2), "flops_per_layer": rc_flops},
        "e2e": e2e,
        "hbm_kernels": hbm_kernels(args.cache),
        "fp8_stream": (fp8_stream(args, rank, seed_offset=replica_seed_offset(rank), barrier=barrier, dist=dist)
                       if args.cache == "bf16" and not args.no_fp8_stream else None),
        "fp8_mma_stream": (fp8_stream(args, rank, seed_offset=replica_seed_offset(rank), barrier=barrier, dist=dist,
                                      mma=True)
                           if args.cache == "bf16" and not args.no_fp8_stream else None),
        "gpu_launches": launches,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    return line


def fp8_stream(args, rank, seed_offset, barrier, dist, mma: bool = False):
    """The same segment workload over an E4M3 KV cache (per (token, head)
    fp32 scales): `steps` segments after `warmup`, device-timed like the
    main line (max over ranks). Its attention launches time the E4M3 -> bf16
    staging kernel and the attention kernel together; with `mma`, the
    V-scale pass and the FP8 tensor-core attention kernel (the append is a
    launch of its own there)."""
    w = W.replace(W.STREAM_FP8, layers=args.layers)
    st = Stream(w, "fp8", "cuda", seed_offset=seed_offset, fp8_mma=mma)
    for s in range(args.warmup):
        st.step(s)
    barrier()
    ev = [torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True), []]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    steps = max(2, args.steps // 2)
    t0.record()
    for s in range(steps):
        st.step(args.warmup + s, attn_events=ev)
    t1.record()
    barrier()
    if st.swa.device_error():
        raise RuntimeError("device error word set in the E4M3 stream")
    ms = max_over_ranks(t0.elapsed_time(t1), dist)
    attn_s = statistics.mean(a.elapsed_time(b) for a, b in ev[2]) / 1e3
    peaks, _ = measured_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    achieved = attention_flops(w) / attn_s / 1e12
    world = int(os.environ.get("WORLD_SIZE", "1"))
    out = {"value": round(SEGMENT * steps * world / (ms / 1e3), 3), "unit": UNIT, "steps": steps,
           "ms_per_step": round(ms / steps, 3), "kv_cache": "E4M3 codes + fp32 scale per (token, head)",
           "roofline": {"bound": "tensor",
                        "kernel": ("scale_max_kernel + sink_window_attention_kernel<E4M3Kv> (kind::f8f6f4) per "
                                   "ll_sink_window_attention_fp8_mma call; the append is a launch of its own" if mma
                                   else "append_stage_e4m3_kernel (append + bf16 staging copy) + "
                                        "sink_window_attention_kernel per ll_append_and_attend call"),
                        "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                        "frac": round(achieved / peak, 4), "avg_launch_us": round(attn_s * 1e6, 2)}}
    del st
    torch.cuda.empty_cache()
    return out


def run_e2e(st: Stream, args, barrier, dist):
    w = st.w
    L = st.layers
    n_host = 2  # host frames per layer (pinned); distinct frames cycle through them
    host = [[tuple(t[f].cpu().pin_memory() for t in (st.q[l], st.k[l], st.v[l])) for f in range(n_host)]
            for l in range(L)]
    dev = [[tuple(torch.empty_like(st.q[0][0]) for _ in range(3)) for _ in range(L)] for _ in range(2)]
    out_host = torch.empty((SEGMENT, 1, w.N, w.H, w.D), dtype=torch.bfloat16).pin_memory()
    copy = torch.cuda.Stream()
    comp = torch.cuda.current_stream()
    ready = [torch.cuda.Event() for _ in range(2)]
    free = [torch.cuda.Event() for _ in range(2)]
    for e in free:
        e.record(comp)
    host_x = st.rx[0].cpu().pin_memory()      # the prompt-switch hidden states of one layer
    x_ready = torch.cuda.Event()
    h2d = 3 * w.N * w.H * w.D * 2 * L * SEGMENT + host_x.numel() * 2 * L
    d2h = w.N * w.H * w.D * 2 * SEGMENT

    def seg(s, start=None):
        def load(i):
            b = i % 2
            with torch.cuda.stream(copy):
                if start is not None and i == 0:
                    copy.wait_event(start)      # no copy of the timed region starts before it
                copy.wait_event(free[b])
                for l in range(L):
                    for t_dev, t_host in zip(dev[b][l], host[l][(i + s) % n_host]):
                        t_dev.copy_(t_host, non_blocking=True)
                ready[b].record(copy)

        held = st.held_frames(SEGMENT * (s + 1) - 1)
        with torch.cuda.stream(copy):             # every layer's X crosses PCIe at the switch
            if start is not None:
                copy.wait_event(start)
            copy.wait_stream(comp)
            for l in range(L):
                st.rx[l].copy_(host_x, non_blocking=True)
            x_ready.record(copy)
        comp.wait_event(x_ready)
        for l in range(L):
            st.swa.kv_recache(st.caches[l], st.rx[l], st.rwk[l], st.rwv[l], st.rg[l], 1e-6, held, st.rope)
        load(0)
        for i in range(SEGMENT):
            if i + 1 < SEGMENT:
                load(i + 1)
            b = i % 2
            comp.wait_event(ready[b])
            f = SEGMENT * (s + 1) + i
            for l in range(L):
                q, k, v = dev[b][l]
                if st.fuses(l):
                    st.swa.append_and_attend(st.caches[l], k, v, q, f, st.rope, out=st.out)
                else:
                    st.swa.kvcache_append(st.caches[l], k, v, f, st.rope)
                    st.swa.sink_window_attention(q, st.caches[l], f, st.rope, out=st.out)
            free[b].record(comp)
            out_host[i].copy_(st.out, non_blocking=True)

    steps = max(2, args.steps // 2)
    seg(args.warmup + args.steps)
    barrier()
    a = torch.cuda.Event(enable_timing=True)
    bb = torch.cuda.Event(enable_timing=True)
    a.record()
    for s in range(steps):
        seg(args.warmup + args.steps + 1 + s, start=a if s == 0 else None)
    bb.record()
    barrier()
    ms = max_over_ranks(a.elapsed_time(bb), dist)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    return {"value": round(SEGMENT * steps * world / (ms / 1e3), 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps}


ATTN_SOURCES = ("ll_attention.cuh", "ll_common.cuh", "ll_rope_append.cuh")


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ATTN_SOURCES:
        with open(os.path.join(ROOT, "sink_window_attention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_traffic(capture: str):
    """DRAM bytes (read + write) per launch of one ncu capture, from the
    committed data file profiles/traffic.json — a figure taken by ncu on an
    earlier run, not a measurement of this run — and only while the kernel
    sources still hash to the version that capture names; otherwise None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(capture)
    if not rec or rec.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    return int(rec["dram_bytes_per_launch"])


# ---------------------------------------------------------------------------
# oracle on the host cores (cpu_baseline and the --impl reference arm)
# ---------------------------------------------------------------------------
class OracleStep:
    """The oracle holding a steady-state 12-frame history of one layer; each
    call times one layer-step restricted to `rows` query rows (all heads, all
    18720 keys) plus the K rotation of the appended frame."""

    def __init__(self, w: W.Workload, seed: int = 0):
        from oracle import rope as orope
        from oracle.stream import StreamOracle
        self.w = w
        eps = w.eps
        om = orope.head_frequencies(w.H, w.pairs, w.theta0, w.sigma_t,
                                    None if eps is None else eps.astype(np.float64))
        self.so = StreamOracle(w.H, w.D, w.grid_h, w.grid_w, om, w.pairs, w.t_offset)
        self.rng = np.random.default_rng(seed)
        self.f = 0
        for _ in range(w.slots):
            self._append()

    def _append(self):
        w = self.w
        self.so.append(self.f, self.rng.standard_normal((w.N, w.H, w.D)) * w.qkv_scale,
                       self.rng.standard_normal((w.N, w.H, w.D)) * w.qkv_scale)
        self.f += 1

    def time(self, rows: int) -> float:
        """Seconds for one sample: the append of one frame and the attention
        of its first `rows` query rows."""
        w = self.w
        q = self.rng.standard_normal((w.N, w.H, w.D)) * w.qkv_scale
        t0 = time.perf_counter()
        self._append()
        self.so.attend(q, self.f - 1, rows=np.arange(rows))
        return time.perf_counter() - t0


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# The oracle's sample, shared by the cpu_baseline of our arm and every step of
# the reference arm: one steady-state layer-step (append of one latent frame
# and attention of its query rows over the 12-frame window), restricted to the
# first `rows` query rows so that one sample takes about STEP_TARGET_S on the
# host (all rows when the host is fast enough). One whole layer-step is one of
# the 30 layers of one latent frame; the per-segment recache (1/40 of a
# layer's recache per layer-step, under 1 % of the work) is not included.
STEP_TARGET_S = 3.0


def oracle_rows(ora: "OracleStep") -> int:
    """Query rows per sample: a probe of 64 rows (all of them in a frame of
    fewer; the faster of two runs, the first pays for page faults) scaled to
    STEP_TARGET_S, never fewer rows than the probe nor more than a frame."""
    probe = min(64, ora.w.N)
    t = min(ora.time(probe), ora.time(probe))
    return int(max(probe, min(ora.w.N, probe * STEP_TARGET_S / max(t, 1e-3))))


def oracle_sample_desc(w: W.Workload, rows: int) -> str:
    return (f"one steady-state layer-step in float64 NumPy restricted to {rows} of its {w.N} query rows: append "
            f"of 1 latent frame and attention of those rows, all {w.H} heads, over {w.slots * w.N} keys; "
            f"= {rows}/{w.N} x 1/{w.layers} of one latent frame through the {w.layers}-layer stack (the recache, "
            f"under 1 % of the work, not included)")


def oracle_frames(w: W.Workload, rows: int) -> float:
    """Latent frames of stack work that one sample of `rows` rows amounts to."""
    return rows / w.N / w.layers


# The cpu_baseline of our arm repeats that sample until about this much host
# time has been spent (at least one sample, at most BASELINE_MAX_SAMPLES).
BASELINE_TARGET_S = 12.0
BASELINE_MAX_SAMPLES = 8


def cpu_baseline(w: W.Workload):
    ora = OracleStep(w)
    rows = oracle_rows(ora)
    times = []
    while not times or (sum(times) < BASELINE_TARGET_S and len(times) < BASELINE_MAX_SAMPLES):
        times.append(ora.time(rows))
    t = sum(times)
    return {"value": round(len(times) * oracle_frames(w, rows) / t, 6), "unit": UNIT, "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{len(times)} consecutive samples, each {oracle_sample_desc(w, rows)}; took {t:.2f} s"}


def run_reference(args, rank, world):
    """The oracle on the host cores, timed as it runs: every step is one
    oracle sample and ms_per_step is its measured wall time; value is the
    latent frames that work amounts to per second."""
    if rank != 0:
        return None
    w = W.STREAM
    ora = OracleStep(w)
    rows = oracle_rows(ora)
    samples = []
    for s in range(args.warmup + args.steps):
        t = ora.time(rows)
        if s >= args.warmup:
            samples.append(t)
    step_s = statistics.mean(samples)
    value = oracle_frames(w, rows) / step_s
    return {"impl": "reference", "metric": METRIC, "value": round(value, 7), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"240s stream segment: latent frames x {w.layers} layers, H=12 D=128, "
                                   "1560 tok/frame, 3 sink + 9 local, LoL jitter 0.8",
                       "step": f"{rows}/{w.N} of one layer-step = {oracle_frames(w, rows):.3g} latent frame",
                       "parallelism": "host cores"},
            "extrapolated": {"ms_per_latent_frame": round(step_s / oracle_frames(w, rows) * 1e3, 1),
                             "note": "the measured step time scaled to a whole latent frame through the stack "
                                     "(rows and layers); not a measurement"},
            "cpu_baseline": {"value": round(value, 7), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": oracle_sample_desc(w, rows)},
            "e2e": {"value": round(value, 7), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_attention_only(args):
    """Wan-shaped single layer (H=12, D=128, 1560 queries over 18720 keys):
    `warmup` + `steps` attention launches at steady state, each timed with CUDA
    events on the launching stream. A small, self-contained case for kernel
    timing and profiler captures."""
    from sink_window_attention_b200 import build
    build.build()
    import sink_window_attention_b200 as swa
    w = W.WAN if args.workload == "wan" else W.CHUNK
    st = Stream(W.replace(w, layers=1, sigma_t=0.8, jitter_seed=4), "fp8" if args.cache == "fp8mma" else args.cache,
                "cuda")
    c = w.query_frames
    q = W.normal((1, c * w.N, w.H, w.D), 99, w.qkv_scale, torch.bfloat16, "cuda")
    out = torch.empty_like(q)
    f0 = 3 * 40  # a steady-state frame (chunk start) with all 12 slots valid
    # before each launch a 256 MB write evicts the cache from L2 (as in the
    # 30-layer stream) and a 0.1 ms device sleep lets the host enqueue the
    # launch ahead of the GPU, so the events see the device time of the call
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")
    ev = []
    for i in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.zero_()
        torch.cuda._sleep(200_000)
        a.record()
        if args.cache == "fp8mma":
            swa.sink_window_attention_fp8_mma(q, st.caches[0], f0, st.rope, out=out)
        else:
            swa.sink_window_attention(q, st.caches[0], f0, st.rope, out=out)
        b.record()
        ev.append((a, b))
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) / 1e3 for a, b in ev[args.warmup:]]
    assert swa.device_error() == 0
    fl = attention_flops(w)
    peaks, kind = measured_peaks()
    t = statistics.median(times)
    return {"mode": "attention", "workload": w.name, "cache": args.cache, "launches": len(times),
            "median_us": round(t * 1e6, 2),
            "min_us": round(min(times) * 1e6, 2), "tflops": round(fl / t / 1e12, 1),
            "frac_of_burst_peak": round(fl / t / 1e12 / peaks["bf16_tflops"], 4), "peak_kind": kind}


def run_append_only(args):
    """RoPE + append of one Wan frame (or a 3-frame chunk with --workload
    chunk) into a layer cache (bf16 or E4M3 cache): `warmup` + `steps`
    launches, each after a 256 MB write that evicts L2, timed with CUDA
    events; achieved HBM bandwidth from the algorithmic bytes."""
    from sink_window_attention_b200 import build
    build.build()
    import sink_window_attention_b200 as swa
    w = W.WAN if args.workload == "wan" else W.CHUNK
    c = w.query_frames
    st = Stream(W.replace(w, layers=1, sigma_t=0.8, jitter_seed=4), args.cache, "cuda")
    ks = [W.normal((1, c * w.N, w.H, w.D), 50 + i, w.qkv_scale, torch.bfloat16, "cuda") for i in range(2)]
    vs = [W.normal((1, c * w.N, w.H, w.D), 60 + i, w.qkv_scale, torch.bfloat16, "cuda") for i in range(2)]
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")
    f0 = 3 * 40
    ev = []
    for i in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.zero_()
        torch.cuda._sleep(200_000)
        a.record()
        swa.kvcache_append(st.caches[0], ks[i % 2], vs[i % 2], f0 + c * i, st.rope)
        b.record()
        ev.append((a, b))
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) / 1e3 for a, b in ev[args.warmup:]]
    assert swa.device_error() == 0
    nbytes = c * append_bytes(w, 1 if args.cache == "fp8" else 2)
    peaks, kind = measured_peaks()
    t = statistics.median(times)
    return {"mode": "append", "workload": w.name, "frames": c, "cache": args.cache, "launches": len(times),
            "median_us": round(t * 1e6, 2), "algorithmic_bytes": nbytes, "gbs": round(nbytes / t / 1e9, 1),
            "frac_of_hbm_peak": round(nbytes / t / 1e9 / peaks["hbm_gbs"], 4), "peak_kind": kind}


def hbm_kernels(cache: str):
    """The HBM-bound kernels timed alone (each launch after an L2 flush): the
    RoPE + append of one Wan frame and of a 3-frame chunk into this run's
    cache type, and the in-place RoPE of the same Q sizes. In the stream the
    append is fused into the attention launch and the Q rotation into its Q
    load, so these are the separate entry points' figures."""
    out = {}
    for wl in ("wan", "chunk"):
        a = argparse.Namespace(workload=wl, cache=cache, steps=10, warmup=3)
        for name, fn in (("append", run_append_only), ("rope", run_rope_only)):
            r = fn(a)
            out[f"{name}_{wl}"] = {k: r[k] for k in ("median_us", "algorithmic_bytes", "gbs", "frac_of_hbm_peak")}
    return out


def rope_bytes(w: W.Workload, frames: int) -> float:
    """Algorithmic HBM bytes of an in-place RoPE of `frames` frames of one
    bf16 [N, H, D] tensor: every element read once and written once."""
    return 2.0 * 2 * frames * w.N * w.H * w.D


def run_rope_only(args):
    """In-place RoPE (ll_rope_apply) of one Wan frame's Q (or a 3-frame chunk
    with --workload chunk): `warmup` + `steps` launches, each after a 256 MB
    write that evicts L2, timed with CUDA events; achieved HBM bandwidth from
    the algorithmic bytes."""
    from sink_window_attention_b200 import build
    build.build()
    import sink_window_attention_b200 as swa
    w = W.replace(W.WAN if args.workload == "wan" else W.CHUNK, sigma_t=0.8, jitter_seed=4)
    c = w.query_frames
    rope = swa.Rope(pairs=w.pairs, grid_h=w.grid_h, grid_w=w.grid_w, theta0=w.theta0, sigma_t=w.sigma_t,
                    eps=[float(e) for e in w.eps], t_offset=w.t_offset)
    xs = [W.normal((1, c * w.N, w.H, w.D), 70 + i, w.qkv_scale, torch.bfloat16, "cuda") for i in range(2)]
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")
    ev = []
    for i in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.zero_()
        torch.cuda._sleep(200_000)
        a.record()
        swa.rope_apply(xs[i % 2], 120 + c * i, rope)
        b.record()
        ev.append((a, b))
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) / 1e3 for a, b in ev[args.warmup:]]
    assert swa.device_error() == 0
    nbytes = rope_bytes(w, c)
    peaks, kind = measured_peaks()
    t = statistics.median(times)
    return {"mode": "rope", "workload": w.name, "frames": c, "launches": len(times), "median_us": round(t * 1e6, 2),
            "algorithmic_bytes": nbytes, "gbs": round(nbytes / t / 1e9, 1),
            "frac_of_hbm_peak": round(nbytes / t / 1e9 / peaks["hbm_gbs"], 4), "peak_kind": kind}


def run_recache_only(args):
    """One layer's KV recache at the Wan shape (X [18720, 1536], Wk, Wv
    [1536, 1536]): `warmup` + `steps` launches timed with CUDA events."""
    from sink_window_attention_b200 import build
    build.build()
    import sink_window_attention_b200 as swa
    st = Stream(W.replace(W.STREAM, layers=1), "bf16", "cuda")
    held = st.held_frames(SEGMENT - 1)
    times = []
    for i in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        swa.kv_recache(st.caches[0], st.rx[0], st.rwk[0], st.rwv[0], st.rg[0], 1e-6, held, st.rope)
        b.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(a.elapsed_time(b) / 1e3)
    assert swa.device_error() == 0
    w = st.w
    fl = recache_flops(w)
    peaks, kind = measured_peaks()
    t = statistics.median(times)
    return {"mode": "recache", "launches": len(times), "median_us": round(t * 1e6, 2),
            "tflops": round(fl / t / 1e12, 1), "frac_of_burst_peak": round(fl / t / 1e12 / peaks["bf16_tflops"], 4),
            "peak_kind": kind}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=8)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cache", default="bf16", choices=["bf16", "fp8", "fp8mma"],
                    help="fp8mma (--mode attention): the E4M3 cache read by the FP8 tensor-core attention")
    ap.add_argument("--layers", type=int, default=30)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--separate", action="store_true", help="append and attention as two calls (bf16 cache)")
    ap.add_argument("--no-fp8-stream", action="store_true", help="skip the E4M3-cache stream figure")
    ap.add_argument("--mode", default="stream", choices=["stream", "attention", "recache", "append", "rope"])
    ap.add_argument("--workload", default="wan", choices=["wan", "chunk"])
    args = ap.parse_args()
    if args.cache == "fp8mma" and args.mode != "attention":
        ap.error("--cache fp8mma times the FP8 tensor-core attention alone (--mode attention); the stream line "
                 "carries it as fp8_mma_stream")
    if args.mode == "attention":
        print(json.dumps(run_attention_only(args)), flush=True)
        return
    if args.mode == "recache":
        print(json.dumps(run_recache_only(args)), flush=True)
        return
    if args.mode == "append":
        print(json.dumps(run_append_only(args)), flush=True)
        return
    if args.mode == "rope":
        print(json.dumps(run_rope_only(args)), flush=True)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as tdist
            tdist.barrier()
            tdist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
