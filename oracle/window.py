"""Frame sink + short window: which frames a query attends to, and where the
cache keeps them (oracle).

Sources
-------
* LongLive review, section "Short-Window Attention": attention runs over a
  local window of recent latent frames, window size 12 latent frames.
* LongLive review, section "Frame Sink": the KV states of the first frames
  are kept as global anchors; 9 local + 3 sink = 12 effective frames.
* LoL review, "Attention Sink": the initial frames are never evicted.

Readings (the pages do not spell these out):
* the 9 local frames include the query's own frame (12 frames in total);
* while fewer than 12 frames exist, the set is the plain union 0..f;
* in chunk mode the chunk's last frame f decides the set, so the chunk's
  frames count among the 9 local ones;
* the cache has n_sink pinned slots and an n_local ring; frame f < n_sink goes
  to slot f, later frames to n_sink + (f - n_sink) mod n_local.
"""
from __future__ import annotations

from typing import List


def attended_frames(f: int, n_sink: int = 3, n_local: int = 9) -> List[int]:
    """A(f) = {0..n_sink-1} U {max(0, f-n_local+1) .. f}, restricted to frames <= f."""
    if f < 0:
        return []
    sinks = set(range(min(n_sink, f + 1)))
    local = set(range(max(0, f - n_local + 1), f + 1))
    return sorted(sinks | local)


def slot_of(f: int, n_sink: int = 3, n_local: int = 9) -> int:
    """Cache slot of frame f: pinned sinks first, then a ring over the local slots."""
    if f < 0:
        raise ValueError("negative frame index")
    if f < n_sink:
        return f
    return n_sink + (f - n_sink) % n_local


def valid_slots(f: int, n_sink: int = 3, n_local: int = 9) -> int:
    """Number of occupied slots once frames 0..f have been written."""
    return min(f + 1, n_sink + n_local)


def slot_frames(last_frame: int, n_sink: int = 3, n_local: int = 9) -> List[int]:
    """Frame held by each occupied slot after frames 0..last_frame were written
    (-1 for a slot never written)."""
    S = n_sink + n_local
    held = [-1] * S
    for g in range(last_frame + 1):
        held[slot_of(g, n_sink, n_local)] = g
    return held
