"""Frame-by-frame stream of the attention hot path (oracle, float64).

It keeps the rotated keys and the values of every frame that can still be
attended to and follows the steps in the pages' order:

* LongLive review, "Short-Window Attention" and "Frame Sink": each query
  frame (or chunk) attends to the 3 sink frames plus the most recent local
  frames, 12 in all;
* LoL review, "Method steps": Q and K of head h are rotated with the head's
  (jittered) frequencies before the scores are formed;
* LongLive review, "KV Recache": at a prompt switch the cached frames' K/V are
  recomputed from their hidden states with the new projections.

No slot map is used here: the key set of a query is A(f) computed from frame
indices, so a cache that stores the wrong frame in a slot disagrees with it.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np

from .attention import sink_window_attention
from .recache import recache_frame
from .rope import rope_3d, token_positions
from .window import attended_frames


class StreamOracle:
    def __init__(self, H: int, D: int, grid_h: int, grid_w: int, omega: np.ndarray, pairs,
                 t_offset: int = 0, n_sink: int = 3, n_local: int = 9, t_scale: float = 1.0):
        self.H, self.D = H, D
        self.grid_h, self.grid_w = grid_h, grid_w
        self.N = grid_h * grid_w
        self.omega = np.asarray(omega, dtype=np.float64)
        self.pairs = tuple(pairs)
        self.t_offset = t_offset
        self.t_scale = t_scale
        self.n_sink, self.n_local = n_sink, n_local
        self.k: Dict[int, np.ndarray] = {}   # frame -> rotated K [N, H, D]
        self.v: Dict[int, np.ndarray] = {}   # frame -> V [N, H, D]
        self.last = -1

    def _rot(self, x: np.ndarray, frame: int) -> np.ndarray:
        t, r, c = token_positions(frame, self.grid_h, self.grid_w, self.t_offset, self.t_scale)
        return rope_3d(x, t, r, c, self.omega, self.pairs)

    def append(self, first_frame: int, k: np.ndarray, v: np.ndarray, replace: bool = False) -> None:
        """Store frames first_frame.. (k, v: [F*N, H, D], K not yet rotated).

        replace=True re-writes the most recent frames instead (first_frame + F
        - 1 == the last frame stored): one denoising pass of the current frame
        or chunk (LongLive review, implementation table: several denoising
        steps per frame) recomputes its K/V, and the next attention sees the
        history plus this pass's K/V. The history itself is unchanged."""
        k = np.asarray(k, dtype=np.float64)
        v = np.asarray(v, dtype=np.float64)
        F = k.shape[0] // self.N
        if replace:
            assert first_frame + F - 1 == self.last, "a pass re-writes the most recent frames"
        else:
            assert first_frame == self.last + 1, "frames must arrive in order"
        for fi in range(F):
            f = first_frame + fi
            sl = slice(fi * self.N, (fi + 1) * self.N)
            self.k[f] = self._rot(k[sl], f)
            self.v[f] = v[sl].copy()
        self.last = first_frame + F - 1
        # A(g) for any later g is contained in A(last) plus frames not yet written
        keep = set(attended_frames(self.last, self.n_sink, self.n_local))
        for f in list(self.k):
            if f not in keep:
                del self.k[f], self.v[f]

    def rotate_queries(self, q: np.ndarray, first_frame: int) -> np.ndarray:
        q = np.asarray(q, dtype=np.float64)
        F = q.shape[0] // self.N
        return np.concatenate([self._rot(q[fi * self.N:(fi + 1) * self.N], first_frame + fi)
                               for fi in range(F)], axis=0)

    def attend(self, q: np.ndarray, first_frame: int, scale: Optional[float] = None,
               rows: Optional[Sequence[int]] = None, return_lse: bool = False):
        """Attention output of query frames first_frame.. (q [F*N, H, D], not rotated).

        ``rows`` restricts the computation to those query rows (all heads)."""
        q = np.asarray(q, dtype=np.float64)
        F = q.shape[0] // self.N
        last = first_frame + F - 1
        qr = self.rotate_queries(q, first_frame)
        if rows is not None:
            qr = qr[np.asarray(rows)]
        return sink_window_attention(qr, self.k, self.v, last, self.n_sink, self.n_local, scale, return_lse)

    def recache(self, switch_frame: int, x_by_frame: Dict[int, np.ndarray], wk, wv, gamma,
                eps: float) -> None:
        """Prompt switch before frame ``switch_frame``: recompute K/V of every frame
        that the next query can attend to, except the one still to be generated."""
        frames = [g for g in attended_frames(switch_frame - 1, self.n_sink, self.n_local)]
        for g in frames:
            k, v = recache_frame(x_by_frame[g], wk, wv, gamma, eps, g, self.H, self.D,
                                 self.grid_h, self.grid_w, self.omega, self.pairs, self.t_offset, self.t_scale)
            self.k[g] = k
            self.v[g] = v
