"""Pins of the frame-sink / short-window set and the cache slot map.

LongLive review, 'Short-Window Attention' (12 latent frames) and 'Frame Sink'
(9 local + 3 sink = 12 effective); LoL review, 'Attention Sink' (sink frames
are never evicted)."""
import pytest

from oracle import window


def test_attended_golden(golden):
    g = golden("window.json")
    for f, want in g["attended"].items():
        assert window.attended_frames(int(f), g["n_sink"], g["n_local"]) == want
    for f, s in g["slot"].items():
        assert window.slot_of(int(f), g["n_sink"], g["n_local"]) == s
    assert g["n_sink"] + g["n_local"] == g["window"]


def _simulate(n_frames, n_sink, n_local, chunk):
    """Brute-force cache: explicit list of slots, evict the oldest non-sink frame
    when full, write the new frame into the freed slot."""
    S = n_sink + n_local
    slots = [None] * S
    history = []
    f = 0
    while f < n_frames:
        block = list(range(f, min(f + chunk, n_frames)))
        for g in block:
            if None in slots:
                s = slots.index(None)
            else:
                cand = [(slots[i], i) for i in range(S) if slots[i] >= n_sink]
                s = min(cand)[1]            # oldest local frame
            slots[s] = g
            history.append((g, s, list(slots)))
        f += chunk
    return history


@pytest.mark.parametrize("n_sink,n_local,chunk", [(3, 9, 1), (3, 9, 3), (1, 4, 1), (2, 6, 2), (3, 12, 3)])
def test_slot_map_matches_brute_force(n_sink, n_local, chunk):
    for g, s, slots in _simulate(200, n_sink, n_local, chunk):
        assert window.slot_of(g, n_sink, n_local) == s
        held = [x for x in slots if x is not None]
        # after writing frame g the cache holds exactly A(g) ...
        assert sorted(held) == window.attended_frames(g, n_sink, n_local)
        # ... in the slot prefix [0, valid_slots(g))
        nv = window.valid_slots(g, n_sink, n_local)
        assert all(x is not None for x in slots[:nv]) and all(x is None for x in slots[nv:])
        assert window.slot_frames(g, n_sink, n_local)[:nv] == slots[:nv]


def test_chunk_slots_contiguous():
    # 3-frame chunks after the sinks land in 3 consecutive ring slots
    for c in range(1, 60):
        s = [window.slot_of(3 * c + i) for i in range(3)]
        assert s[1] == s[0] + 1 and s[2] == s[0] + 2


def test_window_covers_everything_when_large():
    # with a window at least as long as the stream, A(f) = 0..f (full frame-causal)
    for f in range(50):
        assert window.attended_frames(f, 3, 1000) == list(range(f + 1))


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=150, deadline=None)
@given(n_sink=st.integers(0, 6), n_local=st.integers(1, 14), chunk=st.integers(1, 4), n_frames=st.integers(1, 80))
def test_slot_map_matches_brute_force_random(n_sink, n_local, chunk, n_frames):
    """The brute-force cache simulation above, over random windows, chunk
    sizes (up to the local window) and stream lengths."""
    if chunk > n_local:
        chunk = n_local
    for g, s, slots in _simulate(n_frames, n_sink, n_local, chunk):
        assert window.slot_of(g, n_sink, n_local) == s
        held = [x for x in slots if x is not None]
        assert sorted(held) == window.attended_frames(g, n_sink, n_local)
        nv = window.valid_slots(g, n_sink, n_local)
        assert all(x is not None for x in slots[:nv]) and all(x is None for x in slots[nv:])
