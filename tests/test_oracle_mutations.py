"""The oracle's pins reject plausible mistakes in the oracle.

Each case below plants one mistake in a copy of an oracle function: a flipped
sign, a dropped term or factor, an index off by one, swapped operands or
axes. It runs, on the CPU, the pins that cover that function and requires at
least one of them to fail. monkeypatch swaps the function in for that test
only; the oracle's sources are not changed.

What each mistake contradicts:
- the rotation matrix and its adjacent-pair layout (LoL review, 'Prerequisites:
  RoPE');
- theta_i = theta^(-2i/d) and the per-head temporal jitter
  theta_hat = theta0 (1 + sigma eps) ('Method steps');
- the row-major (h, w) token order and the t, h, w band order of the 3D RoPE;
- C(Delta) = (1/K) sum_i e^{j w_i Delta} ('Core innovation');
- softmax(Q K^T / sqrt(d)) V ('Multi-head attention');
- 3 sink frames + 9 local frames including the current one, the sinks pinned
  and the local frames in a ring (LongLive review, 'Short-Window Attention',
  'Frame Sink'; LoL review, 'Attention Sink');
- RMSNorm over the row (y = x / sqrt(mean x^2 + eps) * gamma) and RoPE at the
  frame's own position ('KV Recache'), on K = X Wk only, V = X Wv stored as
  is (the reading the oracle states for the recompute);
- the OCP E4M3 encoding (bias 7, subnormals without the implicit one,
  round to nearest even, 448 as the largest finite value) and the per-row
  scale that multiplies the decoded codes back.
"""
import json
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import test_oracle_attention as pin_att  # noqa: E402
import test_oracle_recache_fp8 as pin_rf  # noqa: E402
import test_oracle_rope as pin_rope  # noqa: E402
import test_oracle_window as pin_win  # noqa: E402

from oracle import attention, fp8, recache, rope, window  # noqa: E402
from oracle.stream import StreamOracle  # noqa: E402

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def rejected(pins):
    """True when at least one pin fails its assertions."""
    for pin in pins:
        try:
            pin()
        except AssertionError:
            return True
    return False


# ------------------------------------------------------------------ RoPE and jitter
def rot_sign_flipped(x, angle):
    x = np.asarray(x, dtype=np.float64)
    a, b = x[..., 0::2], x[..., 1::2]
    c, s = np.cos(angle), np.sin(angle)
    out = np.empty(x.shape, dtype=np.float64)
    out[..., 0::2] = a * c + b * s
    out[..., 1::2] = -a * s + b * c
    return out


def rot_half_split(x, angle):
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1] // 2
    a, b = x[..., :n], x[..., n:]
    c, s = np.cos(angle), np.sin(angle)
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def freq_d_is_pairs(base, pairs):
    i = np.arange(pairs, dtype=np.float64)
    return np.power(float(base), -2.0 * i / pairs)


def freq_index_from_one(base, pairs):
    i = np.arange(1, pairs + 1, dtype=np.float64)
    return np.power(float(base), -2.0 * i / (2 * pairs))


def jitter_on_every_band(H, pairs, theta0, sigma=0.0, eps=None):
    pt, ph, pw = pairs
    base = np.full(H, float(theta0)) if eps is None or sigma == 0.0 else rope.jittered_base(theta0, sigma, eps)
    out = np.empty((H, pt + ph + pw))
    for h in range(H):
        out[h, :pt] = rope.band_frequencies(base[h], pt)
        out[h, pt:pt + ph] = rope.band_frequencies(base[h], ph)
        out[h, pt + ph:] = rope.band_frequencies(base[h], pw)
    return out


def jitter_sign_flipped(theta0, sigma, eps):
    return theta0 * (1.0 - sigma * np.asarray(eps, dtype=np.float64))


def positions_column_major(frame, grid_h, grid_w, t_offset=0, t_scale=1.0):
    r = np.tile(np.arange(grid_h), grid_w).astype(np.float64)
    c = np.repeat(np.arange(grid_w), grid_h).astype(np.float64)
    t = np.full(grid_h * grid_w, float(t_offset + frame) * float(t_scale))
    return t, r, c


def positions_scaled_on_every_axis(frame, grid_h, grid_w, t_offset=0, t_scale=1.0):
    r = np.repeat(np.arange(grid_h), grid_w) * float(t_scale)
    c = np.tile(np.arange(grid_w), grid_h) * float(t_scale)
    t = np.full(grid_h * grid_w, float(t_offset + frame) * float(t_scale))
    return t, r.astype(np.float64), c.astype(np.float64)


def rope_3d_h_w_bands_swapped(x, pos_t, pos_h, pos_w, omega, pairs):
    pt, ph, pw = pairs
    T, H, D = x.shape
    pos = np.empty((T, 1, D // 2))
    pos[:, 0, :pt] = np.asarray(pos_t, dtype=np.float64)[:, None]
    pos[:, 0, pt:pt + ph] = np.asarray(pos_w, dtype=np.float64)[:, None]
    pos[:, 0, pt + ph:] = np.asarray(pos_h, dtype=np.float64)[:, None]
    return rope.rotate_pairs(x, pos * omega[None])


def coherence_without_mean(omega, deltas):
    omega = np.asarray(omega, dtype=np.float64)
    deltas = np.asarray(deltas, dtype=np.float64)
    return np.exp(1j * omega[None, :] * deltas[:, None]).sum(axis=1)


def jitter_of_head_zero_for_all(H, pairs, theta0, sigma=0.0, eps=None):
    if eps is not None:
        eps = np.full(H, np.asarray(eps, dtype=np.float64)[0])
    return rope.__dict__["_head_freq_orig"](H, pairs, theta0, sigma, eps)


def jitter_added_not_scaled(theta0, sigma, eps):
    return theta0 + sigma * np.asarray(eps, dtype=np.float64)


def rot_half_angle(x, angle):
    return rope.__dict__["_rotate_orig"](x, 0.5 * np.asarray(angle, dtype=np.float64))


def spatial_bands_with_temporal_width(H, pairs, theta0, sigma=0.0, eps=None):
    pt, ph, pw = pairs
    out = rope.__dict__["_head_freq_orig"](H, pairs, theta0, sigma, eps)
    i_h = np.arange(ph, dtype=np.float64)
    i_w = np.arange(pw, dtype=np.float64)
    out[:, pt:pt + ph] = np.power(float(theta0), -2.0 * i_h / (2 * pt))
    out[:, pt + ph:] = np.power(float(theta0), -2.0 * i_w / (2 * pt))
    return out


def coherence_real_part_only(omega, deltas):
    omega = np.asarray(omega, dtype=np.float64)
    deltas = np.asarray(deltas, dtype=np.float64)
    return np.cos(omega[None, :] * deltas[:, None]).mean(axis=1).astype(np.complex128)


def coherence_conjugate_phase(omega, deltas):
    omega = np.asarray(omega, dtype=np.float64)
    deltas = np.asarray(deltas, dtype=np.float64)
    return np.exp(-1j * omega[None, :] * deltas[:, None]).mean(axis=1)


def positions_without_t_offset(frame, grid_h, grid_w, t_offset=0, t_scale=1.0):
    return rope.__dict__["_positions_orig"](frame, grid_h, grid_w, 0, t_scale)


def positions_offset_not_interpolated(frame, grid_h, grid_w, t_offset=0, t_scale=1.0):
    t, r, c = rope.__dict__["_positions_orig"](frame, grid_h, grid_w, 0, t_scale)
    return t + t_offset, r, c


def rope_frames_from_frame_zero(x, first_frame, grid_h, grid_w, omega, pairs, t_offset=0, t_scale=1.0):
    return rope.__dict__["_rope_frames_orig"](x, 0, grid_h, grid_w, omega, pairs, t_offset, t_scale)


ROPE_CASES = {
    "rotation sign flipped": ("rotate_pairs", rot_sign_flipped,
                              [lambda: pin_rope.test_rotation_golden(golden),
                               pin_rope.test_rotation_is_complex_multiplication]),
    "pairs split in halves instead of adjacent": ("rotate_pairs", rot_half_split,
                                                  [lambda: pin_rope.test_rotation_golden(golden),
                                                   pin_rope.test_rotation_is_complex_multiplication,
                                                   pin_rope.test_band_layout_by_hand]),
    "frequency exponent over pairs instead of d": ("band_frequencies", freq_d_is_pairs,
                                                   [lambda: pin_rope.test_frequency_closed_forms(golden),
                                                    pin_rope.test_frequencies_geometric]),
    "frequency index starting at 1": ("band_frequencies", freq_index_from_one,
                                      [lambda: pin_rope.test_frequency_closed_forms(golden),
                                       pin_rope.test_frequencies_geometric]),
    "jitter on the spatial bands too": ("head_frequencies", jitter_on_every_band,
                                        [pin_rope.test_jitter_regenerated_from_seed]),
    "jitter sign flipped": ("jittered_base", jitter_sign_flipped,
                            [lambda: pin_rope.test_jitter_points_and_bounds(golden)]),
    "tokens in column-major order": ("token_positions", positions_column_major,
                                     [pin_rope.test_token_positions_row_major]),
    "position interpolation on h and w too": ("token_positions", positions_scaled_on_every_axis,
                                              [pin_rope.test_position_interpolation_pins]),
    "h and w bands swapped": ("rope_3d", rope_3d_h_w_bands_swapped,
                              [pin_rope.test_band_layout_by_hand]),
    "coherence sum not divided by K": ("phase_coherence", coherence_without_mean,
                                       [pin_rope.test_phase_coherence_special_values,
                                        pin_rope.test_phase_coherence_harmonic_closed_form]),
}


ROPE_CASES.update({
    "t offset dropped": ("token_positions", positions_without_t_offset,
                         [pin_rope.test_token_positions_row_major, pin_rope.test_rope_frames_absolute_positions]),
    "interpolation not applied to the t offset": ("token_positions", positions_offset_not_interpolated,
                                                  [pin_rope.test_rope_frames_absolute_positions]),
    "a block of frames rotated from frame 0": ("rope_frames", rope_frames_from_frame_zero,
                                               [pin_rope.test_rope_frames_absolute_positions]),
    "coherence from the real parts only": ("phase_coherence", coherence_real_part_only,
                                           [pin_rope.test_phase_coherence_special_values,
                                            pin_rope.test_phase_coherence_harmonic_closed_form]),
    "coherence with the conjugate phase": ("phase_coherence", coherence_conjugate_phase,
                                           [pin_rope.test_phase_coherence_special_values,
                                            pin_rope.test_phase_coherence_harmonic_closed_form]),
    "every head given head 0's jitter": ("head_frequencies", jitter_of_head_zero_for_all,
                                         [pin_rope.test_jitter_regenerated_from_seed]),
    "jitter added to theta0 instead of scaling it": ("jittered_base", jitter_added_not_scaled,
                                                     [lambda: pin_rope.test_jitter_points_and_bounds(golden)]),
    "rotation by half the angle": ("rotate_pairs", rot_half_angle,
                                   [lambda: pin_rope.test_rotation_golden(golden)]),
    "spatial bands with the temporal band's width": ("head_frequencies", spatial_bands_with_temporal_width,
                                                      [pin_rope.test_jitter_regenerated_from_seed]),
})


@pytest.mark.parametrize("case", sorted(ROPE_CASES))
def test_rope_pins_reject(case, monkeypatch):
    name, wrong, pins = ROPE_CASES[case]
    assert not rejected(pins), "the pins must pass on the oracle as written"
    monkeypatch.setitem(rope.__dict__, "_positions_orig", rope.token_positions)
    monkeypatch.setitem(rope.__dict__, "_rope_frames_orig", rope.rope_frames)
    monkeypatch.setitem(rope.__dict__, "_head_freq_orig", rope.head_frequencies)
    monkeypatch.setitem(rope.__dict__, "_rotate_orig", rope.rotate_pairs)
    monkeypatch.setattr(rope, name, wrong)
    assert rejected(pins), case


# ------------------------------------------------------------------ attention
def mha_scale_one_over_d(q, k, v, scale=None, return_lse=False):
    return attention.__dict__["_mha_orig"](q, k, v, 1.0 / q.shape[-1] if scale is None else scale, return_lse)


def softmax_over_queries(s):
    s = np.asarray(s, dtype=np.float64)
    e = np.exp(s - np.max(s, axis=-2, keepdims=True))
    return e / np.sum(e, axis=-2, keepdims=True)


def mha_keys_as_values(q, k, v, scale=None, return_lse=False):
    return attention.__dict__["_mha_orig"](q, k, k, scale, return_lse)


def mha_lse_without_max(q, k, v, scale=None, return_lse=False):
    o, lse = attention.__dict__["_mha_orig"](q, k, v, scale, True)
    if not return_lse:
        return o
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    sc = 1.0 / np.sqrt(q.shape[-1]) if scale is None else scale
    s = np.einsum("qhd,khd->hqk", q, k) * sc
    m = np.max(s, axis=-1)
    return o, np.log(np.sum(np.exp(s - m[..., None]), axis=-1))


ATTN_PINS = [lambda: pin_att.test_worked_example(golden), pin_att.test_matches_library_sdpa,
             pin_att.test_rows_sum_to_one_and_degenerate_cases]
ATTN_CASES = {
    "scale 1/d instead of 1/sqrt(d)": ("mha", mha_scale_one_over_d),
    "softmax over the queries": ("softmax_rows", softmax_over_queries),
    "keys used as values": ("mha", mha_keys_as_values),
    "log-sum-exp without the max": ("mha", mha_lse_without_max),
}


@pytest.mark.parametrize("case", sorted(ATTN_CASES))
def test_attention_pins_reject(case, monkeypatch):
    name, wrong = ATTN_CASES[case]
    assert not rejected(ATTN_PINS)
    monkeypatch.setitem(attention.__dict__, "_mha_orig", attention.mha)
    monkeypatch.setattr(attention, name, wrong)
    assert rejected(ATTN_PINS), case


def append_keys_at_their_slot(self, first_frame, k, v, replace=False):
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    F = k.shape[0] // self.N
    for fi in range(F):
        f = first_frame + fi
        sl = slice(fi * self.N, (fi + 1) * self.N)
        self.k[f] = self._rot(k[sl], window.slot_of(f, self.n_sink, self.n_local))
        self.v[f] = v[sl].copy()
    self.last = first_frame + F - 1


def recache_local_frames_only(self, switch_frame, x_by_frame, wk, wv, gamma, eps):
    frames = [g for g in window.attended_frames(switch_frame - 1, self.n_sink, self.n_local) if g >= self.n_sink]
    for g in frames:
        self.k[g], self.v[g] = recache.recache_frame(x_by_frame[g], wk, wv, gamma, eps, g, self.H, self.D,
                                                     self.grid_h, self.grid_w, self.omega, self.pairs,
                                                     self.t_offset, self.t_scale)


def recache_at_slot_positions(self, switch_frame, x_by_frame, wk, wv, gamma, eps):
    for g in window.attended_frames(switch_frame - 1, self.n_sink, self.n_local):
        s = window.slot_of(g, self.n_sink, self.n_local)
        self.k[g], self.v[g] = recache.recache_frame(x_by_frame[g], wk, wv, gamma, eps, s, self.H, self.D,
                                                     self.grid_h, self.grid_w, self.omega, self.pairs,
                                                     self.t_offset, self.t_scale)


@pytest.mark.parametrize("wrong", [recache_local_frames_only, recache_at_slot_positions],
                         ids=["sinks not recomputed", "frames at their slot positions"])
def test_stream_recache_pin_rejects(wrong, monkeypatch):
    pin = [pin_att.test_stream_recache_matches_dense_recomputed]
    assert not rejected(pin)
    monkeypatch.setattr(StreamOracle, "recache", wrong)
    assert rejected(pin)


def append_pass_not_replacing(self, first_frame, k, v, replace=False):
    if replace:
        return  # the pass's K/V never reach the cache
    StreamOracle.__dict__["_append_orig"](self, first_frame, k, v, replace)


def rot_ignoring_interpolation(self, x, frame):
    t, r, c = rope.token_positions(frame, self.grid_h, self.grid_w, self.t_offset)
    return rope.rope_3d(x, t, r, c, self.omega, self.pairs)


def test_stream_pins_reject_lost_denoising_pass_and_lost_interpolation(monkeypatch):
    passes = [lambda: pin_att.test_stream_denoising_passes_match_dense_masked(1)]
    pi = [pin_att.test_stream_position_interpolation_matches_dense]
    assert not rejected(passes) and not rejected(pi)
    with monkeypatch.context() as m:
        m.setattr(StreamOracle, "_append_orig", StreamOracle.append, raising=False)
        m.setattr(StreamOracle, "append", append_pass_not_replacing)
        assert rejected(passes)
    with monkeypatch.context() as m:
        m.setattr(StreamOracle, "_rot", rot_ignoring_interpolation)
        assert rejected(pi)


def attend_window_of_the_first_frame(self, q, first_frame, scale=None, rows=None, return_lse=False):
    qr = self.rotate_queries(q, first_frame)
    if rows is not None:
        qr = qr[np.asarray(rows)]
    return attention.sink_window_attention(qr, self.k, self.v, first_frame, self.n_sink, self.n_local, scale,
                                           return_lse)


def queries_not_rotated(self, q, first_frame):
    return np.asarray(q, dtype=np.float64)


def queries_all_at_the_first_frame(self, q, first_frame):
    q = np.asarray(q, dtype=np.float64)
    F = q.shape[0] // self.N
    return np.concatenate([self._rot(q[fi * self.N:(fi + 1) * self.N], first_frame) for fi in range(F)], axis=0)


STREAM_PINS = [lambda: pin_att.test_stream_matches_dense_masked_brute_force(9, 1),
               lambda: pin_att.test_stream_matches_dense_masked_brute_force(9, 3)]
STREAM_CASES = {
    "a chunk attending with its first frame's window": ("attend", attend_window_of_the_first_frame),
    "queries not rotated": ("rotate_queries", queries_not_rotated),
    "every query frame of a chunk rotated at the first": ("rotate_queries", queries_all_at_the_first_frame),
}


@pytest.mark.parametrize("case", sorted(STREAM_CASES))
def test_stream_pins_reject(case, monkeypatch):
    name, wrong = STREAM_CASES[case]
    assert not rejected(STREAM_PINS)
    monkeypatch.setattr(StreamOracle, name, wrong)
    assert rejected(STREAM_PINS), case


def test_stream_pin_rejects_keys_rotated_at_their_slot(monkeypatch):
    """K must turn with its frame's absolute position, not its cache slot."""
    pin = [lambda: pin_att.test_stream_matches_dense_masked_brute_force(9, 1)]
    assert not rejected(pin)
    monkeypatch.setattr(StreamOracle, "append", append_keys_at_their_slot)
    assert rejected(pin)


def window_attention_without_sinks(q_rot, k_rot_by_frame, v_by_frame, last_query_frame, n_sink=3, n_local=9,
                                   scale=None, return_lse=False):
    frames = [g for g in range(max(0, last_query_frame - n_local - n_sink + 1), last_query_frame + 1)]
    k = np.concatenate([k_rot_by_frame[g] for g in frames], axis=0)
    v = np.concatenate([v_by_frame[g] for g in frames], axis=0)
    return attention.mha(q_rot, k, v, scale, return_lse)


def test_window_attention_pin_rejects_missing_sinks(monkeypatch):
    """The frame-set attention function (sink + window) is pinned against the
    dense masked brute force: a version that attends to the last 12 frames
    without the sinks is rejected."""
    pin = [lambda: pin_att.test_stream_matches_dense_masked_brute_force(9, 1)]
    assert not rejected(pin)
    monkeypatch.setattr(attention, "sink_window_attention", window_attention_without_sinks)
    assert rejected(pin)


def probabilities_scale_one_over_d(q, k, scale=None):
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    return attention.softmax_rows(np.einsum("qhd,khd->hqk", q, k) / q.shape[-1])


def frame_causal_one_frame_short(q_rot_frames, k_rot_frames, v_frames, query_frame, N, scale=None):
    q = q_rot_frames[query_frame * N:(query_frame + 1) * N]
    hi = max(query_frame, 1) * N
    return attention.mha(q, k_rot_frames[:hi], v_frames[:hi], scale)


def test_probability_pin_rejects_wrong_scale(monkeypatch):
    """attention_probabilities is held to the hand-worked example."""
    pin = [lambda: pin_att.test_worked_example(golden)]
    assert not rejected(pin)
    monkeypatch.setattr(attention, "attention_probabilities", probabilities_scale_one_over_d)
    assert rejected(pin)


def test_full_window_pin_rejects_a_short_frame_causal_reference(monkeypatch):
    """With a window longer than the stream the stream oracle must equal full
    frame-causal attention over frames 0..f, the current frame included."""
    pin = [lambda: pin_att.test_stream_matches_dense_masked_brute_force(10_000, 1)]
    assert not rejected(pin)
    monkeypatch.setattr(attention, "frame_causal_attention", frame_causal_one_frame_short)
    assert rejected(pin)


# ------------------------------------------------------------------ window and slots
def attended_local_one_short(f, n_sink=3, n_local=9):
    if f < 0:
        return []
    return sorted(set(range(min(n_sink, f + 1))) | set(range(max(0, f - n_local + 2), f + 1)))


def attended_without_sinks(f, n_sink=3, n_local=9):
    if f < 0:
        return []
    return list(range(max(0, f - n_local - n_sink + 1), f + 1))


def slot_ring_off_by_one(f, n_sink=3, n_local=9):
    return f if f < n_sink else n_sink + (f - n_sink + 1) % n_local


def slot_ring_over_every_slot(f, n_sink=3, n_local=9):
    if f < 0:
        raise ValueError("negative frame index")
    return f % (n_sink + n_local)


def valid_slots_one_short(f, n_sink=3, n_local=9):
    return min(f, n_sink + n_local)


def valid_slots_capped_at_local(f, n_sink=3, n_local=9):
    return min(f + 1, n_local)


def slot_frames_first_writer_kept(last_frame, n_sink=3, n_local=9):
    held = [-1] * (n_sink + n_local)
    for g in range(last_frame + 1):
        s = window.slot_of(g, n_sink, n_local)
        if held[s] < 0:
            held[s] = g
    return held


WINDOW_PINS = [lambda: pin_win.test_attended_golden(golden),
               lambda: pin_win.test_slot_map_matches_brute_force(3, 9, 1),
               lambda: pin_win.test_slot_map_matches_brute_force(3, 9, 3)]
WINDOW_CASES = {
    "local window one frame short": ("attended_frames", attended_local_one_short),
    "no sink frames (last 12 frames)": ("attended_frames", attended_without_sinks),
    "ring slot off by one": ("slot_of", slot_ring_off_by_one),
    "ring over every slot (sinks evicted)": ("slot_of", slot_ring_over_every_slot),
    "valid slot count one short": ("valid_slots", valid_slots_one_short),
    "valid slot count capped at the local window": ("valid_slots", valid_slots_capped_at_local),
    "slot map keeping the first frame written": ("slot_frames", slot_frames_first_writer_kept),
}


@pytest.mark.parametrize("case", sorted(WINDOW_CASES))
def test_window_pins_reject(case, monkeypatch):
    name, wrong = WINDOW_CASES[case]
    assert not rejected(WINDOW_PINS)
    monkeypatch.setattr(window, name, wrong)
    assert rejected(WINDOW_PINS), case


# ------------------------------------------------------------------ recache and FP8
def rms_over_tokens(x, gamma, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=0, keepdims=True) + eps) * gamma


def rms_eps_outside_root(x, gamma, eps):
    x = np.asarray(x, dtype=np.float64)
    return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps) * gamma


def rms_gamma_before_norm(x, gamma, eps):
    y = np.asarray(x, dtype=np.float64) * gamma
    return y / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)


def recache_without_t_offset(x, wk, wv, gamma, eps, frame, H, D, grid_h, grid_w, omega, pairs,
                             t_offset=0, t_scale=1.0):
    return recache.__dict__["_recache_orig"](x, wk, wv, gamma, eps, frame, H, D, grid_h, grid_w, omega, pairs,
                                             0, t_scale)


def decode_bias_8(code):
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** (1 - 8)
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 8)


def decode_subnormal_with_one(code):
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    return sign * (1.0 + m / 8.0) * 2.0 ** (max(e, 1) - 7)


def encode_truncating(mag):
    vals = fp8.e4m3_table()[:0x7F]
    below = np.where(vals[None, :] <= mag[:, None] + 0.0, vals[None, :], -1.0)
    return np.argmax(below, axis=-1).astype(np.int64)


def quantize_to_240(x):
    x = np.asarray(x, dtype=np.float64)
    amax = np.max(np.abs(x), axis=-1)
    scale = np.where(amax > 0, amax / 240.0, 1.0)
    return fp8.e4m3_encode(x / scale[..., None]), scale


def _recache_parts(x, wk, wv):
    x = np.asarray(x, dtype=np.float64)
    return x @ np.asarray(wk, dtype=np.float64), x @ np.asarray(wv, dtype=np.float64)


def recache_wk_wv_swapped(x, wk, wv, gamma, eps, frame, H, D, grid_h, grid_w, omega, pairs,
                          t_offset=0, t_scale=1.0):
    return recache.__dict__["_recache_orig"](x, wv, wk, gamma, eps, frame, H, D, grid_h, grid_w, omega, pairs,
                                             t_offset, t_scale)


def recache_v_rotated_too(x, wk, wv, gamma, eps, frame, H, D, grid_h, grid_w, omega, pairs,
                          t_offset=0, t_scale=1.0):
    k, v = recache.__dict__["_recache_orig"](x, wk, wv, gamma, eps, frame, H, D, grid_h, grid_w, omega, pairs,
                                             t_offset, t_scale)
    t, r, c = rope.token_positions(frame, grid_h, grid_w, t_offset, t_scale)
    return k, rope.rope_3d(v, t, r, c, omega, pairs)


def recache_k_not_normalised(x, wk, wv, gamma, eps, frame, H, D, grid_h, grid_w, omega, pairs,
                             t_offset=0, t_scale=1.0):
    kp, vp = _recache_parts(x, wk, wv)
    t, r, c = rope.token_positions(frame, grid_h, grid_w, t_offset, t_scale)
    k = (kp * np.asarray(gamma, dtype=np.float64)).reshape(-1, H, D)
    return rope.rope_3d(k, t, r, c, omega, pairs), vp.reshape(-1, H, D)


def recache_rotated_one_frame_late(x, wk, wv, gamma, eps, frame, H, D, grid_h, grid_w, omega, pairs,
                                   t_offset=0, t_scale=1.0):
    return recache.__dict__["_recache_orig"](x, wk, wv, gamma, eps, frame + 1, H, D, grid_h, grid_w, omega,
                                             pairs, t_offset, t_scale)


def dequantize_dividing(codes, scale):
    return fp8.e4m3_decode_array(codes) / np.asarray(scale, dtype=np.float64)[..., None]


def dequantize_without_sign(codes, scale):
    return np.abs(fp8.e4m3_decode_array(codes)) * np.asarray(scale, dtype=np.float64)[..., None]


RECACHE_CASES = {
    "RMS over the tokens instead of the row": (recache, "rmsnorm", rms_over_tokens, [pin_rf.test_rmsnorm_textbook]),
    "eps outside the square root": (recache, "rmsnorm", rms_eps_outside_root, [pin_rf.test_rmsnorm_textbook]),
    "gamma applied before the norm": (recache, "rmsnorm", rms_gamma_before_norm, [pin_rf.test_rmsnorm_textbook]),
    "recache RoPE without the t offset": (recache, "recache_frame", recache_without_t_offset,
                                          [pin_rf.test_recache_frame_composition]),
    "E4M3 exponent bias 8": (fp8, "e4m3_decode", decode_bias_8,
                             [lambda: pin_rf.test_e4m3_golden(golden), pin_rf.test_e4m3_decode_matches_library_all_codes]),
    "E4M3 subnormals with an implicit one": (fp8, "e4m3_decode", decode_subnormal_with_one,
                                             [lambda: pin_rf.test_e4m3_golden(golden),
                                              pin_rf.test_e4m3_decode_matches_library_all_codes]),
    "E4M3 encode truncating": (fp8, "_encode_magnitudes", encode_truncating,
                               [lambda: pin_rf.test_e4m3_golden(golden), pin_rf.test_e4m3_encode_roundtrip_and_nearest]),
    "E4M3 row scale for 240 instead of 448": (fp8, "quantize_rows", quantize_to_240, [pin_rf.test_quantize_rows]),
    "recache with Wk and Wv swapped": (recache, "recache_frame", recache_wk_wv_swapped,
                                       [pin_rf.test_recache_frame_composition]),
    "recache rotating V as well": (recache, "recache_frame", recache_v_rotated_too,
                                   [pin_rf.test_recache_frame_composition]),
    "recache K without the RMSNorm": (recache, "recache_frame", recache_k_not_normalised,
                                      [pin_rf.test_recache_frame_composition]),
    "recache RoPE one frame late": (recache, "recache_frame", recache_rotated_one_frame_late,
                                    [pin_rf.test_recache_frame_composition]),
    "E4M3 dequantise dividing by the scale": (fp8, "dequantize_rows", dequantize_dividing,
                                              [pin_rf.test_quantize_rows]),
    "E4M3 dequantise dropping the sign": (fp8, "dequantize_rows", dequantize_without_sign,
                                          [pin_rf.test_quantize_rows]),
}


@pytest.mark.parametrize("case", sorted(RECACHE_CASES))
def test_recache_fp8_pins_reject(case, monkeypatch):
    mod, name, wrong, pins = RECACHE_CASES[case]
    assert not rejected(pins)
    monkeypatch.setitem(recache.__dict__, "_recache_orig", recache.recache_frame)
    monkeypatch.setattr(mod, name, wrong)
    assert rejected(pins), case
