"""KV recache at a prompt switch (oracle, float64).

Sources
-------
* LongLive review, section "KV Recache": at a prompt-switch boundary the KV
  cache is rebuilt from the already generated frames together with the new
  prompt — the generated video is encoded as visual context, paired with the
  new prompt, and the cache is recomputed; later steps use the new cache.
* LongLive model card (abstract / framework figure, right panel "KV-recache").

Readings (the pages give no formula for the recompute):
* every cached frame (the sinks included) is re-projected from its hidden
  states X (rows of the frames in the cache): K' = X Wk, V = X Wv, no bias;
* K' is RMS-normalised over its whole row (all heads, d_out wide) with a
  learned scale gamma and eps, then rotated with 3D RoPE at the frame's own
  absolute position; V is stored as is.
"""
from __future__ import annotations

import numpy as np

from .rope import rope_3d, token_positions


def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """y = x / sqrt(mean(x^2 over the last axis) + eps) * gamma."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(gamma, dtype=np.float64)


def recache_frame(x: np.ndarray, wk: np.ndarray, wv: np.ndarray, gamma: np.ndarray,
                  eps: float, frame: int, H: int, D: int, grid_h: int, grid_w: int,
                  omega: np.ndarray, pairs, t_offset: int = 0, t_scale: float = 1.0):
    """Recomputed (rotated K, V) of one frame from its hidden states x [N, Dm].

    Returns k_rot [N, H, D] and v [N, H, D]."""
    x = np.asarray(x, dtype=np.float64)
    kp = x @ np.asarray(wk, dtype=np.float64)
    vp = x @ np.asarray(wv, dtype=np.float64)
    k = rmsnorm(kp, gamma, eps).reshape(-1, H, D)
    t, r, c = token_positions(frame, grid_h, grid_w, t_offset, t_scale)
    return rope_3d(k, t, r, c, omega, pairs), vp.reshape(-1, H, D)
