"""Seeded synthetic inputs and workload shapes for the sink-window attention path.

This module is the one piece of code that both the CPU oracle and the CUDA path
consume. It holds shapes and random-number recipes only: no RoPE, no softmax, no
cache policy, no projection. Every random number the method itself draws (the
LoL per-head jitter epsilon_h ~ U[-1, 1]) is produced here from a published
counter-based generator (SplitMix64, Steele, Lea & Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014) and passed to both sides as an
input.

Workloads (shapes follow the LongLive review, section "Implementation details":
Wan 2.1 1.3B backbone at 832x480, 12-frame window = 9 local + 3 sink frames):

* ``tiny``   fp32, B=1 H=2 D=64, 4x6 token grid, 20 frames, 1-frame queries.
* ``wan``    bf16, B=1 H=12 D=128, 30x52 token grid (1560 tokens/frame), 120 frames.
* ``chunk``  as ``wan`` but 3-frame query chunks, temporal offset 2000, LoL jitter
             sigma=0.8 on the temporal band.
* ``recache`` as ``wan`` plus a prompt switch: X [12*1560, 1536] ~ N(0,1),
             Wk, Wv ~ N(0, 1/1536), gamma ~ U[0.5, 1.5].
* ``stream`` 30 layers x 960 frames, recache every 40 frames, bf16 or FP8 cache.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple

import numpy as np
import torch

MASK64 = (1 << 64) - 1


def splitmix64(state: int) -> Tuple[int, int]:
    """One SplitMix64 step: returns (new_state, output), both 64-bit unsigned."""
    state = (state + 0x9E3779B97F4A7C15) & MASK64
    z = state
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return state, z ^ (z >> 31)


def uniform_pm1(seed: int, count: int) -> np.ndarray:
    """``count`` draws from U[-1, 1): SplitMix64 seeded with ``seed``, top 53 bits
    mapped to u in [0, 1), returned as 2u - 1 (exact in float64)."""
    state = seed & MASK64
    out = np.empty(count, dtype=np.float64)
    for i in range(count):
        state, z = splitmix64(state)
        u = (z >> 11) * (1.0 / (1 << 53))
        out[i] = 2.0 * u - 1.0
    return out


def jitter_eps(seed: int, H: int) -> np.ndarray:
    """Per-head LoL jitter draws epsilon_h, h = 0..H-1, rounded to float32 (the
    precision in which the C interface receives them)."""
    return uniform_pm1(seed, H).astype(np.float32)


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str                 # "f32" | "bf16" : element type of Q/K/V
    B: int
    H: int
    D: int
    grid_h: int
    grid_w: int
    frames: int                # latent frames in the stream
    query_frames: int          # frames per query (1, or 3 in chunk mode)
    pairs: Tuple[int, int, int]  # rotary pairs on the (t, h, w) axes, sum = D/2
    theta0: float = 10000.0
    sigma_t: float = 0.0       # LoL jitter scale on the temporal band
    jitter_seed: int = 0
    t_offset: int = 0          # temporal RoPE index of frame 0
    qkv_scale: float = 1.0     # Q, K, V ~ N(0, 1) * qkv_scale
    seed: int = 0
    n_sink: int = 3
    n_local: int = 9
    layers: int = 1
    recache_every: int = 0     # prompt switch period in frames (0: none)
    cache_dtype: str = ""      # "" => same as dtype; "fp8" => e4m3 + fp32 scales
    d_model: int = 0           # recache hidden width (0: H*D)

    @property
    def N(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def slots(self) -> int:
        return self.n_sink + self.n_local

    @property
    def eps(self) -> Optional[np.ndarray]:
        if self.sigma_t == 0.0:
            return None
        return jitter_eps(self.jitter_seed, self.H)

    @property
    def dm(self) -> int:
        return self.d_model or self.H * self.D


TINY = Workload("tiny", "f32", B=1, H=2, D=64, grid_h=4, grid_w=6, frames=20,
                query_frames=1, pairs=(12, 10, 10), qkv_scale=1.0, seed=0)
WAN = Workload("wan", "bf16", B=1, H=12, D=128, grid_h=30, grid_w=52, frames=120,
               query_frames=1, pairs=(22, 21, 21), qkv_scale=0.5, seed=1)
CHUNK = Workload("chunk", "bf16", B=1, H=12, D=128, grid_h=30, grid_w=52, frames=120,
                 query_frames=3, pairs=(22, 21, 21), qkv_scale=0.5, seed=2,
                 sigma_t=0.8, jitter_seed=2, t_offset=2000)
RECACHE = Workload("recache", "bf16", B=1, H=12, D=128, grid_h=30, grid_w=52, frames=52,
                   query_frames=1, pairs=(22, 21, 21), qkv_scale=0.5, seed=3,
                   layers=30, recache_every=40)
STREAM = Workload("stream", "bf16", B=1, H=12, D=128, grid_h=30, grid_w=52, frames=960,
                  query_frames=1, pairs=(22, 21, 21), qkv_scale=0.5, seed=4,
                  sigma_t=0.8, jitter_seed=4, layers=30, recache_every=40)
STREAM_FP8 = replace(STREAM, name="stream_fp8", cache_dtype="fp8")

WORKLOADS = {w.name: w for w in (TINY, WAN, CHUNK, RECACHE, STREAM, STREAM_FP8)}


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def normal(shape, seed: int, scale: float = 1.0, dtype: torch.dtype = torch.float32,
           device: str = "cpu") -> torch.Tensor:
    """N(0, scale^2) samples from torch's Philox/MT generator seeded with ``seed``,
    drawn in float32 on ``device`` and rounded once to ``dtype``."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & ((1 << 63) - 1))
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype)


def uniform(shape, seed: int, lo: float, hi: float, dtype: torch.dtype = torch.float32,
            device: str = "cpu") -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & ((1 << 63) - 1))
    x = torch.rand(*shape, generator=g, device=device, dtype=torch.float32)
    return (x * (hi - lo) + lo).to(dtype)


def frame_seed(w: Workload, layer: int, frame: int, which: int) -> int:
    """Seed of one (layer, frame, tensor) draw; ``which`` 0/1/2 = Q/K/V."""
    return (w.seed * 1_000_003 + layer * 10_007 + frame * 31 + which) & ((1 << 62) - 1)


def qkv_frames(w: Workload, layer: int, first_frame: int, n_frames: int,
               device: str = "cpu", dtype: Optional[torch.dtype] = None):
    """Q, K, V for frames [first_frame, first_frame + n_frames) of one layer,
    each [B, n_frames*N, H, D] in the workload dtype. Frame f's tokens are
    drawn from seeds that depend only on (layer, f), so any frame range can be
    regenerated independently."""
    dt = dtype or torch_dtype(w.dtype)
    outs = []
    for which in range(3):
        parts = [normal((w.B, w.N, w.H, w.D), frame_seed(w, layer, f, which), w.qkv_scale, dt, device)
                 for f in range(first_frame, first_frame + n_frames)]
        outs.append(torch.cat(parts, dim=1).contiguous())
    return tuple(outs)


def recache_inputs(w: Workload, layer: int, switch_frame: int, device: str = "cpu"):
    """Hidden states X [B, slots*N, Dm] (rows in cache-slot order), projections
    Wk, Wv [Dm, H*D] ~ N(0, 1/Dm) and the RMSNorm scale gamma [H*D] ~ U[0.5, 1.5]."""
    dm, dout = w.dm, w.H * w.D
    base = (w.seed * 7_919 + layer * 104_729 + switch_frame * 13) & ((1 << 62) - 1)
    x = normal((w.B, w.slots * w.N, dm), base + 1, 1.0, torch.bfloat16, device)
    wk = normal((dm, dout), base + 2, 1.0 / float(np.sqrt(dm)), torch.bfloat16, device)
    wv = normal((dm, dout), base + 3, 1.0 / float(np.sqrt(dm)), torch.bfloat16, device)
    gamma = uniform((dout,), base + 4, 0.5, 1.5, torch.float32, device)
    return x, wk, wv, gamma
