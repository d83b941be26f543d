"""Rotary position embedding with the LoL multi-head jitter (oracle, float64).

Sources
-------
* LoL review, "Prerequisites: Rotary Position Embedding (RoPE)": a channel pair
  at position t is rotated by R(t, i) = [[cos t*theta_i, -sin t*theta_i],
  [sin t*theta_i, cos t*theta_i]] with theta_i = theta^(-2i/d); the score
  <R(m)q, R(n)k> depends only on n - m.
* LoL review, "Method steps": nu_i = -2i/d_time; per head h draw
  eps_h ~ U[-1, 1]; theta_hat_h = theta0 (1 + sigma_theta eps_h);
  omega_h = [theta_hat_h^nu_0, ...]; rotate Q_h and K_h with omega_h.
  The jitter is applied to the temporal band only (d_time), a reading stated
  for the chunk workload; the spatial bands keep theta0.

* LoL review, "Core innovation": the phase concentration of the RoPE
  components at a relative offset Delta is measured by the phase-coherence
  kernel C(Delta) = (1/K) sum_i exp(j omega_i Delta); it peaks where the sink
  frames collapse. Reading: for the temporal offset between frames the K
  components are the K = pairs_t frequencies of a head's temporal band.
* LoL review, "Motivation" and results table: position interpolation (PI) is
  the baseline that compresses positions; reading: the temporal position
  (t_offset + f) is multiplied by a factor t_scale (1 = plain RoPE).

Layout reading: rotary pairs are adjacent channels (2j, 2j+1) of each head;
the head dimension is split into a temporal band of ``pt`` pairs followed by
``ph`` pairs for the grid row and ``pw`` pairs for the grid column. Inside a
band of P pairs the index i runs 0..P-1 and d_band = 2P.
"""
from __future__ import annotations

import numpy as np


def jittered_base(theta0: float, sigma: float, eps) -> np.ndarray:
    """theta_hat_h = theta0 * (1 + sigma * eps_h)  (LoL "Method steps" (3)-(4))."""
    eps = np.asarray(eps, dtype=np.float64)
    return theta0 * (1.0 + sigma * eps)


def band_frequencies(base: float, pairs: int) -> np.ndarray:
    """omega_i = base^(-2i/d) for i = 0..pairs-1 with d = 2*pairs
    (LoL "RoPE" theta_i = theta^(-2i/d); "Method steps" (2), (5))."""
    d = 2 * pairs
    i = np.arange(pairs, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d)


def head_frequencies(H: int, pairs, theta0: float, sigma: float = 0.0, eps=None) -> np.ndarray:
    """Frequency table omega[h, j] for all D/2 pairs of every head.

    Columns 0..pt-1 use the (jittered) temporal base of head h, then ph columns
    for the row axis and pw for the column axis, both with theta0."""
    pt, ph, pw = pairs
    if eps is None or sigma == 0.0:
        base_t = np.full(H, float(theta0))
    else:
        base_t = jittered_base(theta0, sigma, eps)
    out = np.empty((H, pt + ph + pw), dtype=np.float64)
    for h in range(H):
        out[h, :pt] = band_frequencies(base_t[h], pt)
        out[h, pt:pt + ph] = band_frequencies(theta0, ph)
        out[h, pt + ph:] = band_frequencies(theta0, pw)
    return out


def rotate_pairs(x: np.ndarray, angle: np.ndarray) -> np.ndarray:
    """Apply [[cos, -sin], [sin, cos]] to each adjacent pair (x[..., 2j], x[..., 2j+1]).

    ``angle`` broadcasts against x[..., ::2]."""
    x = np.asarray(x, dtype=np.float64)
    a = x[..., 0::2]
    b = x[..., 1::2]
    c = np.cos(angle)
    s = np.sin(angle)
    out = np.empty(np.broadcast_shapes(x.shape), dtype=np.float64)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def token_positions(frame: int, grid_h: int, grid_w: int, t_offset: int = 0, t_scale: float = 1.0):
    """(t, h, w) of every token of one latent frame, tokens in row-major (h, w)
    order; t = (t_offset + absolute frame index) * t_scale (t_scale != 1: position
    interpolation of the temporal axis)."""
    r = np.repeat(np.arange(grid_h), grid_w)
    c = np.tile(np.arange(grid_w), grid_h)
    t = np.full(grid_h * grid_w, float(t_offset + frame) * float(t_scale))
    return t.astype(np.float64), r.astype(np.float64), c.astype(np.float64)


def phase_coherence(omega: np.ndarray, deltas) -> np.ndarray:
    """C(Delta) = (1/K) * sum_{i<K} exp(j * omega_i * Delta) for every Delta
    (LoL review, "Core innovation"), omega [K] (one head's components).
    Returns complex128 [len(deltas)]."""
    omega = np.asarray(omega, dtype=np.float64)
    deltas = np.asarray(deltas, dtype=np.float64)
    K = omega.shape[0]
    out = np.zeros(deltas.shape[0], dtype=np.complex128)
    for i in range(K):  # one component at a time, as the sum is written
        out += np.exp(1j * omega[i] * deltas)
    return out / K


def rope_3d(x: np.ndarray, pos_t, pos_h, pos_w, omega: np.ndarray, pairs) -> np.ndarray:
    """Factorised 3D RoPE of x [T, H, D] at per-token positions (pos_t, pos_h, pos_w) [T],
    with the per-head frequency table omega [H, D/2]."""
    pt, ph, pw = pairs
    T, H, D = x.shape
    assert D == 2 * (pt + ph + pw) and omega.shape == (H, D // 2)
    pos = np.empty((T, 1, D // 2), dtype=np.float64)
    pos[:, 0, :pt] = np.asarray(pos_t, dtype=np.float64)[:, None]
    pos[:, 0, pt:pt + ph] = np.asarray(pos_h, dtype=np.float64)[:, None]
    pos[:, 0, pt + ph:] = np.asarray(pos_w, dtype=np.float64)[:, None]
    angle = pos * omega[None, :, :]
    return rotate_pairs(x, angle)


def rope_frames(x: np.ndarray, first_frame: int, grid_h: int, grid_w: int, omega, pairs,
                t_offset: int = 0, t_scale: float = 1.0) -> np.ndarray:
    """RoPE of x [B, F*N, H, D] holding consecutive frames first_frame.. first_frame+F-1."""
    x = np.asarray(x, dtype=np.float64)
    B, T, H, D = x.shape
    N = grid_h * grid_w
    F = T // N
    out = np.empty_like(x)
    for fi in range(F):
        t, r, c = token_positions(first_frame + fi, grid_h, grid_w, t_offset, t_scale)
        for b in range(B):
            out[b, fi * N:(fi + 1) * N] = rope_3d(x[b, fi * N:(fi + 1) * N], t, r, c, omega, pairs)
    return out
