"""GPU parity of the KV recache (LongLive review, "KV Recache") against the
fp64 oracle: K = RoPE(RMSNorm(X Wk)), V = X Wv for every cached frame, written
into the frame's slot; then attention over the recached cache."""
import numpy as np
import pytest
import torch

import sink_window_attention_b200 as swa
import swa_workloads as W
from oracle import fp8 as ofp8
from oracle import recache as orec
from oracle import rope as orope
from oracle import window as owin
from oracle.stream import StreamOracle
from tests.conftest import assert_parity

pytestmark = pytest.mark.gpu

EPS = 1e-6


@pytest.fixture(scope="module", autouse=True)
def built():
    from sink_window_attention_b200 import build
    build.build()
    swa.lib()
    yield
    assert swa.device_error() == 0


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def setup(w, switch_frame, layer=0, dtype="bf16", t_scale=1.0):
    eps = W.jitter_eps(11, w.H)
    rope = swa.Rope(pairs=w.pairs, grid_h=w.grid_h, grid_w=w.grid_w, theta0=w.theta0, sigma_t=0.8,
                    eps=[float(e) for e in eps], t_offset=w.t_offset, t_scale=t_scale)
    om = orope.head_frequencies(w.H, w.pairs, w.theta0, 0.8, eps.astype(np.float64))
    frames = owin.slot_frames(switch_frame - 1)
    n_slots = sum(1 for f in frames if f >= 0)
    x, wk, wv, gamma = W.recache_inputs(w, layer, switch_frame)
    x = x[:, :n_slots * w.N].contiguous()
    cache = swa.KVCache(w.B, w.H, w.D, w.N, dtype)
    swa.kv_recache(cache, x.cuda(), wk.cuda(), wv.cuda(), gamma.cuda(), EPS, frames[:n_slots], rope)
    torch.cuda.synchronize()
    return rope, om, frames[:n_slots], x, wk, wv, gamma, cache


def check_slots(w, om, frames, x, wk, wv, gamma, cache, rows_per_slot=None, fp8=False, t_scale=1.0):
    X, Wk, Wv, G = np64(x[0]), np64(wk), np64(wv), np64(gamma)
    N = w.N
    for s, f in enumerate(frames):
        if rows_per_slot is None:
            rows = np.arange(N)
            kref, vref = orec.recache_frame(X[s * N:(s + 1) * N], Wk, Wv, G, EPS, f, w.H, w.D, w.grid_h, w.grid_w,
                                            om, w.pairs, w.t_offset, t_scale)
        else:
            rows = np.unique(np.r_[0, N - 1, np.random.default_rng(s).choice(N, rows_per_slot, replace=False)])
            kref, vref = _rows_ref(X, Wk, Wv, G, s, f, rows, w, om)
        if not fp8:
            gk = np64(cache.k[0, s * N:(s + 1) * N])[rows]
            gv = np64(cache.v[0, s * N:(s + 1) * N])[rows]
            # K (unit RMS after the norm) and V (unit variance) are stored in
            # bf16, whose rounding alone is up to 2^-9 of each value: the mean
            # bar is twice that relative to the data, the max bar as everywhere
            assert_parity(gk, kref, mean_abs=2.0 ** -8 * np.abs(kref).mean(), what=f"K slot {s}")
            assert_parity(gv, vref, mean_abs=2.0 ** -8 * np.abs(vref).mean(), what=f"V slot {s}")
        else:
            ks = cache.k_scale[0, s * N:(s + 1) * N].cpu().numpy().astype(np.float64)[rows]
            vs = cache.v_scale[0, s * N:(s + 1) * N].cpu().numpy().astype(np.float64)[rows]
            gk = ofp8.dequantize_rows(cache.k[0, s * N:(s + 1) * N].cpu().numpy()[rows], ks)
            gv = ofp8.dequantize_rows(cache.v[0, s * N:(s + 1) * N].cpu().numpy()[rows], vs)
            for got, ref, sc, nm in ((gk, kref, ks, "K"), (gv, vref, vs, "V")):
                bound = 2.0 ** -4 * np.abs(ref) + 2.0 ** -10 * sc[..., None] + 2e-3 * np.abs(ref).max()
                assert np.all(np.abs(got - ref) <= bound), f"fp8 {nm} slot {s}"


def _rows_ref(X, Wk, Wv, G, s, f, rows, w, om):
    """Oracle recache restricted to some token rows of one frame (RMSNorm and
    RoPE act row by row, so rows are independent)."""
    N = w.N
    xr = X[s * N:(s + 1) * N][rows]
    kp = xr @ Wk
    vp = xr @ Wv
    k = orec.rmsnorm(kp, G, EPS).reshape(-1, w.H, w.D)
    t, r, c = orope.token_positions(f, w.grid_h, w.grid_w, w.t_offset)
    return orope.rope_3d(k, t[rows], r[rows], c[rows], om, w.pairs), vp.reshape(-1, w.H, w.D)


SMALL = W.replace(W.TINY, name="small", dtype="bf16", H=2, D=128, pairs=(22, 21, 21), d_model=256)


@pytest.mark.parametrize("H", [2, 4])
def test_recache_small_every_element(H):
    """Dout = 256 (one CTA per row block) and 512 (a 2-CTA cluster sharing
    the RMSNorm sums); every row of every slot is checked."""
    w = W.replace(SMALL, H=H)
    rope, om, frames, x, wk, wv, gamma, cache = setup(w, 40)
    assert frames == owin.slot_frames(39)
    check_slots(w, om, frames, x, wk, wv, gamma, cache)


def test_recache_small_warmup_slots():
    """A switch during warm-up: only 7 slots are occupied and recomputed."""
    w = W.replace(SMALL, H=4)
    rope, om, frames, x, wk, wv, gamma, cache = setup(w, 7)
    assert len(frames) == 7
    check_slots(w, om, frames, x, wk, wv, gamma, cache)


def test_recache_small_position_interpolation():
    """Position interpolation (t_scale 1/4, temporal offset 300) in the
    recache epilogue's RoPE; every element checked."""
    w = W.replace(SMALL, H=4, t_offset=300)
    rope, om, frames, x, wk, wv, gamma, cache = setup(w, 40, t_scale=0.25)
    check_slots(w, om, frames, x, wk, wv, gamma, cache, t_scale=0.25)


def test_recache_small_fp8():
    w = W.replace(SMALL, H=4)
    rope, om, frames, x, wk, wv, gamma, cache = setup(w, 40, dtype="fp8")
    check_slots(w, om, frames, x, wk, wv, gamma, cache, fp8=True)


def test_recache_wan_sampled_rows():
    """Wan shape: X [18720, 1536], Wk, Wv [1536, 1536]; six column tiles per
    row block form a cluster; sampled rows of every slot."""
    w = W.RECACHE
    rope, om, frames, x, wk, wv, gamma, cache = setup(w, 40)
    check_slots(w, om, frames, x, wk, wv, gamma, cache, rows_per_slot=40)


def test_recache_then_attention():
    """Prompt switch before frame 40, then frames 40..42 attend over the
    recached cache (each frame appended first), against the oracle stream."""
    w = W.RECACHE
    rope, om, frames, x, wk, wv, gamma, cache = setup(w, 40)
    so = StreamOracle(w.H, w.D, w.grid_h, w.grid_w, om, w.pairs, w.t_offset)
    # the oracle's history: frames 0..39 (their K/V are replaced by the recache)
    so.last = 39
    X = np64(x[0])
    so.recache(40, {f: X[s * w.N:(s + 1) * w.N] for s, f in enumerate(frames)}, np64(wk), np64(wv), np64(gamma),
               EPS)
    for f in range(40, 43):
        q, k, v = W.qkv_frames(w, 3, f, 1)
        swa.kvcache_append(cache, k.cuda(), v.cuda(), f, rope)
        out = swa.sink_window_attention(q.cuda(), cache, f, rope)
        so.append(f, np64(k[0]), np64(v[0]))
        rows = np.unique(np.r_[0:4, 1556:1560, np.random.default_rng(f).choice(1560, 24, replace=False)])
        ref = so.attend(np64(q[0]), f, rows=rows)
        assert_parity(np64(out[0])[rows], ref, what=f"attention after recache, frame {f}")
