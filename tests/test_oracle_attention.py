"""Pins of the attention oracle.

LoL review, 'Multi-head attention' (softmax(Q K^T / sqrt(d_k)) V per head);
LongLive review, 'Short-Window Attention' and 'Frame Sink'."""
import numpy as np
import pytest
import torch

import swa_workloads as W
from oracle import attention, rope, window
from oracle.stream import StreamOracle


def test_worked_example(golden):
    g = golden("attention_small.json")
    q = np.array(g["q"])[:, None, :]
    k = np.array(g["k"])[:, None, :]
    v = np.array(g["v"])[:, None, :]
    o, lse = attention.mha(q, k, v, return_lse=True)
    assert np.allclose(o[:, 0], g["o"], atol=1e-14)
    assert np.allclose(lse[0], g["lse"], atol=1e-14)
    assert np.allclose(attention.attention_probabilities(q, k)[0], g["p"], atol=1e-15)


def test_matches_library_sdpa():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((9, 3, 16))
    k = rng.standard_normal((21, 3, 16))
    v = rng.standard_normal((21, 3, 16))
    o = attention.mha(q, k, v)
    t = lambda a: torch.from_numpy(a).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v))[0].permute(1, 0, 2).numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)


def test_rows_sum_to_one_and_degenerate_cases():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((5, 2, 8)) * 4
    k = rng.standard_normal((30, 2, 8))
    v = rng.standard_normal((30, 2, 8))
    p = attention.attention_probabilities(q, k)
    assert np.allclose(p.sum(-1), 1.0, atol=1e-14) and np.all(p >= 0)
    # one key: output is that key's value
    assert np.allclose(attention.mha(q, k[:1], v[:1]), np.broadcast_to(v[:1], q.shape), atol=1e-14)
    # zero query: uniform weights, output = mean of V
    assert np.allclose(attention.mha(np.zeros_like(q), k, v), np.broadcast_to(v.mean(0), q.shape), atol=1e-14)
    # permuting the keys (with their values) changes nothing
    perm = rng.permutation(30)
    assert np.allclose(attention.mha(q, k[perm], v[perm]), attention.mha(q, k, v), atol=1e-13)


def _dense_masked(qr, kr, vr, qframe_of_row, kframe_of_col, allowed, scale):
    """Brute force: full score matrix over all frames, -inf where the key's frame
    is not allowed for the query's frame."""
    s = np.einsum("qhd,khd->hqk", qr, kr) * scale
    mask = np.array([[allowed(qf, kf) for kf in kframe_of_col] for qf in qframe_of_row])
    s = np.where(mask[None], s, -np.inf)
    s = s - s.max(-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(-1, keepdims=True)
    return np.einsum("hqk,khd->qhd", p, vr)


@pytest.mark.parametrize("n_local,chunk", [(9, 1), (9, 3), (10_000, 1)])
def test_stream_matches_dense_masked_brute_force(n_local, chunk):
    """The stream oracle (history dict + A(f)) equals one dense masked softmax over
    all frames; with a huge window it is full frame-causal attention."""
    Wl = W.TINY
    H, D, gh, gw = Wl.H, Wl.D, Wl.grid_h, Wl.grid_w
    N = gh * gw
    F = 18
    om = rope.head_frequencies(H, Wl.pairs, 10000.0, 0.8, W.jitter_eps(5, H))
    rng = np.random.default_rng(2)
    Q = rng.standard_normal((F * N, H, D))
    K = rng.standard_normal((F * N, H, D))
    V = rng.standard_normal((F * N, H, D))
    so = StreamOracle(H, D, gh, gw, om, Wl.pairs, t_offset=100, n_local=n_local)
    Qr = rope.rope_frames(Q[None], 0, gh, gw, om, Wl.pairs, 100)[0]
    Kr = rope.rope_frames(K[None], 0, gh, gw, om, Wl.pairs, 100)[0]
    kframe = np.repeat(np.arange(F), N)
    scale = 1 / np.sqrt(D)
    for f0 in range(0, F, chunk):
        so.append(f0, K[f0 * N:(f0 + chunk) * N], V[f0 * N:(f0 + chunk) * N])
        got = so.attend(Q[f0 * N:(f0 + chunk) * N], f0)
        last = f0 + chunk - 1
        A = set(window.attended_frames(last, 3, n_local))
        ref = _dense_masked(Qr[f0 * N:(f0 + chunk) * N], Kr, V, np.repeat(np.arange(f0, f0 + chunk), N),
                            kframe, lambda qf, kf: kf in A, scale)
        assert np.allclose(got, ref, rtol=1e-11, atol=1e-11)
        # the window function itself, fed per-frame rotated keys and values
        kd = {g: Kr[g * N:(g + 1) * N] for g in range(last + 1)}
        vd = {g: V[g * N:(g + 1) * N] for g in range(last + 1)}
        direct = attention.sink_window_attention(Qr[f0 * N:(f0 + chunk) * N], kd, vd, last, 3, n_local)
        assert np.allclose(direct, ref, rtol=1e-11, atol=1e-11)
        if n_local >= F:
            full = attention.frame_causal_attention(Qr, Kr, V, last, N)
            if chunk == 1:
                assert np.allclose(got, full, rtol=1e-11, atol=1e-11)


def test_stream_rows_and_lse():
    Wl = W.TINY
    om = rope.head_frequencies(Wl.H, Wl.pairs, 10000.0)
    rng = np.random.default_rng(3)
    N = Wl.N
    so = StreamOracle(Wl.H, Wl.D, Wl.grid_h, Wl.grid_w, om, Wl.pairs)
    for f in range(4):
        so.append(f, rng.standard_normal((N, Wl.H, Wl.D)), rng.standard_normal((N, Wl.H, Wl.D)))
    q = rng.standard_normal((N, Wl.H, Wl.D))
    full, lse = so.attend(q, 3, return_lse=True)
    part, lse_p = so.attend(q, 3, rows=[0, 5, 23], return_lse=True)
    assert np.allclose(part, full[[0, 5, 23]], atol=1e-14)
    assert np.allclose(lse_p, lse[:, [0, 5, 23]], atol=1e-14)


@pytest.mark.parametrize("chunk", [1, 3])
def test_stream_denoising_passes_match_dense_masked(chunk):
    """Several denoising passes per frame (or chunk): each pass re-writes the
    current frames' K/V (append(..., replace=True)) and attends. Every pass
    equals one dense masked softmax over all frames in which the current
    frames hold that pass's K/V and the earlier frames their last pass's."""
    Wl = W.TINY
    H, D, gh, gw = Wl.H, Wl.D, Wl.grid_h, Wl.grid_w
    N = gh * gw
    F, passes = 15, 3
    om = rope.head_frequencies(H, Wl.pairs, 10000.0, 0.8, W.jitter_eps(6, H))
    rng = np.random.default_rng(7)
    Q = rng.standard_normal((passes, F * N, H, D))
    K = rng.standard_normal((passes, F * N, H, D))
    V = rng.standard_normal((passes, F * N, H, D))
    Qr = [rope.rope_frames(Q[ps][None], 0, gh, gw, om, Wl.pairs, 40)[0] for ps in range(passes)]
    Kr = [rope.rope_frames(K[ps][None], 0, gh, gw, om, Wl.pairs, 40)[0] for ps in range(passes)]
    so = StreamOracle(H, D, gh, gw, om, Wl.pairs, t_offset=40)
    kframe = np.repeat(np.arange(F), N)
    for f0 in range(0, F, chunk):
        cur = slice(f0 * N, (f0 + chunk) * N)
        last = f0 + chunk - 1
        A = set(window.attended_frames(last, 3, 9))
        for ps in range(passes):
            so.append(f0, K[ps][cur], V[ps][cur], replace=ps > 0)
            got = so.attend(Q[ps][cur], f0)
            kk = Kr[passes - 1].copy()
            vv = V[passes - 1].copy()
            kk[cur] = Kr[ps][cur]
            vv[cur] = V[ps][cur]
            ref = _dense_masked(Qr[ps][cur], kk, vv, np.repeat(np.arange(f0, f0 + chunk), N), kframe,
                                lambda qf, kf: kf in A, 1 / np.sqrt(D))
            assert np.allclose(got, ref, rtol=1e-11, atol=1e-11)
    with pytest.raises(AssertionError):  # a pass may only re-write the most recent frames
        so.append(0, K[0][:N], V[0][:N], replace=True)


def test_stream_recache_matches_dense_recomputed():
    """A prompt switch before frame F (LongLive review, 'KV Recache': the cache
    is rebuilt from the generated frames with the new prompt). Afterwards every
    frame the next query can see, sinks included, holds K/V recomputed from its
    own hidden states at its own position; frame F is appended as usual. One
    dense masked softmax over those K/V, built frame by frame from
    recache_frame and rope_frames, must equal the stream oracle's attention."""
    from oracle import recache
    Wl = W.TINY
    H, D, gh, gw = Wl.H, Wl.D, Wl.grid_h, Wl.grid_w
    N, F, dm, t0 = gh * gw, 16, 32, 100
    om = rope.head_frequencies(H, Wl.pairs, 10000.0, 0.8, W.jitter_eps(6, H))
    rng = np.random.default_rng(7)
    K = rng.standard_normal(((F + 1) * N, H, D))
    V = rng.standard_normal(((F + 1) * N, H, D))
    so = StreamOracle(H, D, gh, gw, om, Wl.pairs, t_offset=t0)
    for f in range(F):
        so.append(f, K[f * N:(f + 1) * N], V[f * N:(f + 1) * N])
    X = {g: rng.standard_normal((N, dm)) for g in range(F)}
    wk = rng.standard_normal((dm, H * D)) / np.sqrt(dm)
    wv = rng.standard_normal((dm, H * D)) / np.sqrt(dm)
    gamma = rng.uniform(0.5, 1.5, H * D)
    so.recache(F, X, wk, wv, gamma, 1e-6)
    so.append(F, K[F * N:], V[F * N:])
    q = rng.standard_normal((N, H, D))
    got = so.attend(q, F)
    keys, vals = [], []
    for g in range(F):
        k, v = recache.recache_frame(X[g], wk, wv, gamma, 1e-6, g, H, D, gh, gw, om, Wl.pairs, t_offset=t0)
        keys.append(k)
        vals.append(v)
    keys.append(rope.rope_frames(K[None, F * N:], F, gh, gw, om, Wl.pairs, t0)[0])
    vals.append(V[F * N:])
    A = set(window.attended_frames(F, 3, 9))
    qr = rope.rope_frames(q[None], F, gh, gw, om, Wl.pairs, t0)[0]
    ref = _dense_masked(qr, np.concatenate(keys), np.concatenate(vals), np.full(N, F),
                        np.repeat(np.arange(F + 1), N), lambda qf, kf: kf in A, 1 / np.sqrt(D))
    assert np.allclose(got, ref, rtol=1e-11, atol=1e-11)


def test_stream_position_interpolation_matches_dense():
    """With position interpolation (temporal positions scaled by s, LoL review's
    PI baseline) the stream equals one dense masked softmax over queries and
    keys rotated by rope_frames at the scaled positions, and differs from the
    unscaled stream."""
    Wl = W.TINY
    H, D, gh, gw = Wl.H, Wl.D, Wl.grid_h, Wl.grid_w
    N, F, t0, s = gh * gw, 14, 30, 0.5
    om = rope.head_frequencies(H, Wl.pairs, 10000.0, 0.8, W.jitter_eps(8, H))
    rng = np.random.default_rng(9)
    Q = rng.standard_normal((F * N, H, D))
    K = rng.standard_normal((F * N, H, D))
    V = rng.standard_normal((F * N, H, D))
    so = StreamOracle(H, D, gh, gw, om, Wl.pairs, t_offset=t0, t_scale=s)
    plain = StreamOracle(H, D, gh, gw, om, Wl.pairs, t_offset=t0)
    Qr = rope.rope_frames(Q[None], 0, gh, gw, om, Wl.pairs, t0, s)[0]
    Kr = rope.rope_frames(K[None], 0, gh, gw, om, Wl.pairs, t0, s)[0]
    kframe = np.repeat(np.arange(F), N)
    for f in range(F):
        cur = slice(f * N, (f + 1) * N)
        so.append(f, K[cur], V[cur])
        plain.append(f, K[cur], V[cur])
        got = so.attend(Q[cur], f)
        A = set(window.attended_frames(f, 3, 9))
        ref = _dense_masked(Qr[cur], Kr, V, np.full(N, f), kframe, lambda qf, kf: kf in A, 1 / np.sqrt(D))
        assert np.allclose(got, ref, rtol=1e-11, atol=1e-11)
        if f >= 4:
            assert not np.allclose(got, plain.attend(Q[cur], f), atol=1e-6)
