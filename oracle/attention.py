"""Attention definitions (oracle, float64).

Sources
-------
* LoL review, "Multi-head attention": per head h,
  Attention(Q_h, K_h, V_h) = softmax(Q_h K_h^T / sqrt(d_k)) V_h.
* LongLive review, "Short-Window Attention": Attn(q, k, v) =
  softmax(q k_[window] / sqrt(d)) v_[window] (the printed formula drops the
  transpose; read as q k^T), window = 12 latent frames.
* LongLive review, "Frame Sink": the window is 9 local + 3 sink frames.

Reading: inside the attended frames there is no token mask — a query token sees
every token of its own frame (or chunk) and of every attended frame; frames
outside A(f) are invisible (frame-level causal attention).
"""
from __future__ import annotations

import numpy as np

from .window import attended_frames


def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Row softmax along the last axis, shifted by the row max."""
    s = np.asarray(s, dtype=np.float64)
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def mha(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float | None = None,
        return_lse: bool = False):
    """Textbook multi-head attention.

    q [Tq, H, D], k [Tk, H, D], v [Tk, H, D] -> o [Tq, H, D] (and the natural-log
    sum-exp of the scaled scores, [H, Tq], when ``return_lse``)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    D = q.shape[-1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    # per-head score matrix Q_h K_h^T (matmul over [H, Tq, D] x [H, D, Tk])
    s = np.matmul(q.transpose(1, 0, 2), k.transpose(1, 2, 0)) * scale   # [H, Tq, Tk]
    p = softmax_rows(s)
    o = np.matmul(p, v.transpose(1, 0, 2)).transpose(1, 0, 2)           # [Tq, H, D]
    if not return_lse:
        return o
    m = np.max(s, axis=-1)
    lse = m + np.log(np.sum(np.exp(s - m[..., None]), axis=-1))
    return o, lse


def attention_probabilities(q, k, scale=None) -> np.ndarray:
    """softmax(q k^T * scale) per head, [H, Tq, Tk]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[-1])
    return softmax_rows(np.einsum("qhd,khd->hqk", q, k) * scale)


def sink_window_attention(q_rot: np.ndarray, k_rot_by_frame: dict, v_by_frame: dict,
                          last_query_frame: int, n_sink: int = 3, n_local: int = 9,
                          scale: float | None = None, return_lse: bool = False):
    """Attention of one query block over the frame-sink + short-window set.

    q_rot            [Tq, H, D] rotated queries (one frame, or a chunk of frames)
    k_rot_by_frame   frame index -> [N, H, D] rotated keys of that frame
    v_by_frame       frame index -> [N, H, D] values of that frame
    last_query_frame f: the key set is every token of every frame in A(f)."""
    frames = attended_frames(last_query_frame, n_sink, n_local)
    k = np.concatenate([np.asarray(k_rot_by_frame[g], dtype=np.float64) for g in frames], axis=0)
    v = np.concatenate([np.asarray(v_by_frame[g], dtype=np.float64) for g in frames], axis=0)
    return mha(q_rot, k, v, scale, return_lse)


def frame_causal_attention(q_rot_frames: np.ndarray, k_rot_frames: np.ndarray,
                           v_frames: np.ndarray, query_frame: int, N: int, scale=None):
    """Full frame-causal attention without any window: the query frame attends
    to every token of frames 0..query_frame. Inputs hold all frames
    [F*N, H, D]; used as the window >= stream-length limit."""
    q = q_rot_frames[query_frame * N:(query_frame + 1) * N]
    k = k_rot_frames[:(query_frame + 1) * N]
    v = v_frames[:(query_frame + 1) * N]
    return mha(q, k, v, scale)
