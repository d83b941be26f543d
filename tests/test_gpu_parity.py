"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle on
the same seeded inputs.

Bars: slots bit-exact; floating point max|err| <= 1e-2 * max|ref| and
mean|err| <= 1e-3 (bf16 inputs, fp32 accumulation; the same bar for the fp32 /
tf32 workload); FP8 cache max|err| <= 5e-2 * max|ref| against the unquantised
reference."""
import numpy as np
import pytest
import torch

import sink_window_attention_b200 as swa
import swa_workloads as W
from oracle import fp8 as ofp8
from oracle import rope as orope
from oracle import window as owin
from oracle.stream import StreamOracle
from tests.conftest import assert_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from sink_window_attention_b200 import build
    build.build()
    swa.lib()
    yield
    assert swa.device_error() == 0


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rope_of(w: W.Workload) -> swa.Rope:
    eps = w.eps
    return swa.Rope(pairs=w.pairs, grid_h=w.grid_h, grid_w=w.grid_w, theta0=w.theta0, sigma_t=w.sigma_t,
                    eps=None if eps is None else [float(e) for e in eps], t_offset=w.t_offset)


def omega_of(w: W.Workload) -> np.ndarray:
    eps = w.eps
    return orope.head_frequencies(w.H, w.pairs, w.theta0, w.sigma_t, None if eps is None else eps.astype(np.float64))


def sample_rows(Tq: int, n: int, seed: int) -> np.ndarray:
    """Sampled query rows: the first and last rows, both sides of every 128-row
    tile boundary, the ragged tail and random rows."""
    rng = np.random.default_rng(seed)
    fixed = {0, 1, Tq - 1, Tq - 2}
    for b in range(128, Tq, 128):
        fixed |= {b - 1, b}
    rows = sorted(fixed | set(rng.choice(Tq, size=min(n, Tq), replace=False).tolist()))
    return np.array([r for r in rows if 0 <= r < Tq])


# ---------------------------------------------------------------------------- RoPE
@pytest.mark.parametrize("name", ["tiny", "wan", "chunk"])
def test_rope_apply(name):
    w = W.WORKLOADS[name]
    F = 3
    x, _, _ = W.qkv_frames(w, 7, 5, F)
    xg = x.cuda()
    swa.rope_apply(xg, 5, rope_of(w))
    ref = orope.rope_frames(np64(x), 5, w.grid_h, w.grid_w, omega_of(w), w.pairs, w.t_offset)
    tol = 1e-5 if w.dtype == "f32" else 1e-2
    assert_parity(np64(xg), ref, max_rel=tol, mean_abs=1e-3 if w.dtype != "f32" else 1e-6, what="rope")


def test_rope_apply_one_head_d8():
    """One head of D = 8 (a single 8-element chunk per token row, so a block
    of the in-place RoPE has fewer threads than token rows), fp32, every
    element checked."""
    w = W.replace(W.TINY, H=1, D=8, pairs=(2, 1, 1), name="tiny_h1_d8")
    x, _, _ = W.qkv_frames(w, 7, 5, 3)
    xg = x.cuda()
    swa.rope_apply(xg, 5, rope_of(w))
    ref = orope.rope_frames(np64(x), 5, w.grid_h, w.grid_w, omega_of(w), w.pairs, w.t_offset)
    assert_parity(np64(xg), ref, max_rel=1e-5, mean_abs=1e-6, what="rope h1 d8")


@pytest.mark.parametrize("name", ["tiny", "chunk"])
def test_rope_position_interpolation(name):
    """Position interpolation (t_scale): against the oracle at scale 1/4, and
    bit-identical to plain RoPE where the positions coincide (scale 1/2 at
    frame 2f is plain RoPE at frame f; the offset is scaled too, so it is 0
    here)."""
    w = W.replace(W.WORKLOADS[name], t_offset=0)
    x, _, _ = W.qkv_frames(w, 8, 3, 2)
    r = rope_of(w)
    r.t_scale = 0.25
    xg = x.cuda()
    swa.rope_apply(xg, 9, r)
    ref = orope.rope_frames(np64(x), 9, w.grid_h, w.grid_w, omega_of(w), w.pairs, 0, t_scale=0.25)
    tol = 1e-5 if w.dtype == "f32" else 1e-2
    assert_parity(np64(xg), ref, max_rel=tol, mean_abs=1e-3 if w.dtype != "f32" else 1e-6, what="rope PI")
    a, b = x[:, :w.N].cuda(), x[:, :w.N].cuda()  # one frame
    r.t_scale = 0.5
    swa.rope_apply(a, 14, r)
    swa.rope_apply(b, 7, rope_of(w))
    assert torch.equal(a, b)


# ---------------------------------------------------------------------------- append
@pytest.mark.parametrize("name,chunk", [("tiny", 1), ("chunk", 3)])
def test_append_slots_and_values(name, chunk):
    w = W.WORKLOADS[name]
    cache = swa.KVCache(w.B, w.H, w.D, w.N, w.dtype)
    rope = rope_of(w)
    om = omega_of(w)
    N = w.N
    frames_seen = []
    for f0 in range(0, 15, chunk):
        _, k, v = W.qkv_frames(w, 1, f0, chunk)
        slots = swa.kvcache_append(cache, k.cuda(), v.cuda(), f0, rope)
        assert slots == [owin.slot_of(f0 + i) for i in range(chunk)]
        kref = orope.rope_frames(np64(k), f0, w.grid_h, w.grid_w, om, w.pairs, w.t_offset)
        for i, s in enumerate(slots):
            got_k = np64(cache.k[:, s * N:(s + 1) * N])
            got_v = cache.v[:, s * N:(s + 1) * N].cpu()
            assert torch.equal(got_v, v[:, i * N:(i + 1) * N])           # a copy: bit-exact
            tol = 1e-5 if w.dtype == "f32" else 1e-2
            assert_parity(got_k, kref[:, i * N:(i + 1) * N], max_rel=tol, what=f"K slot {s}")
        frames_seen += list(range(f0, f0 + chunk))
        # the occupied slots hold exactly A(last frame)
        held = owin.slot_frames(frames_seen[-1])
        assert sorted(x for x in held if x >= 0) == owin.attended_frames(frames_seen[-1])


def test_append_fp8_codes_and_scales():
    """FP8 cache: V codes and scales bit-exact against the oracle's E4M3 encoder
    fed the same fp32 quotient (both sides take the rounding decision on the
    same float32 value); rotated K within the E4M3 error bound."""
    w = W.WAN
    cache = swa.KVCache(1, w.H, w.D, w.N, "fp8")
    _, k, v = W.qkv_frames(w, 2, 0, 1)
    swa.kvcache_append(cache, k.cuda(), v.cuda(), 0, rope_of(w))
    N = w.N
    vv = v[0].float().numpy()                                    # [N, H, D] exact bf16 values
    amax = np.abs(vv).max(-1).astype(np.float32)
    scale32 = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    quot = (vv / scale32[..., None]).astype(np.float32)          # IEEE fp32 division, as on the GPU
    codes = ofp8.e4m3_encode(quot.astype(np.float64))
    got_codes = cache.v[0, :N].cpu().numpy()
    assert np.array_equal(got_codes, codes)
    assert np.array_equal(cache.v_scale[0, :N].cpu().numpy(), scale32)
    # K: dequantised values vs the fp64 rotated K, element by element within the
    # E4M3 rounding bound (half an ulp: 2^-4 of the value for normals, 2^-10 *
    # scale in the subnormal range) plus the fp32 rotation error
    kref = orope.rope_frames(np64(k), 0, w.grid_h, w.grid_w, omega_of(w), w.pairs, w.t_offset)[0]
    ks = cache.k_scale[0, :N].cpu().numpy().astype(np.float64)
    kdeq = ofp8.dequantize_rows(cache.k[0, :N].cpu().numpy(), ks)
    bound = 2.0 ** -4 * np.abs(kref) + 2.0 ** -10 * ks[..., None] + 1e-5 * np.abs(kref).max()
    assert np.all(np.abs(kdeq - kref) <= bound)
    # the row max lands on +-448 * scale up to the rounding of the fp32 quotient
    assert np.allclose(np.abs(kdeq).max(-1), 448.0 * ks, rtol=1e-5)


# ---------------------------------------------------------------------------- attention
def run_stream(w: W.Workload, frames, layer=0, rows_per_step=48, q_scale=1.0, check_lse=True, dtype=None,
               B=None, mean_abs=1e-3, lse_rel=1e-3, max_rel=1e-2, scale=None, k_scale=None, no_rope=False,
               t_scale=1.0, lse_mean=5e-3, n_sink=3, n_local=9, attend=None):
    """Append + attend frame by frame (or chunk by chunk); compare sampled rows
    (all rows when the step is small) with the oracle stream."""
    B = B or w.B
    cache = swa.KVCache(B, w.H, w.D, w.N, dtype or w.dtype, n_sink=n_sink, n_local=n_local)
    # no_rope: Q and K are passed as already rotated (rope descriptor NULL);
    # the oracle then rotates by angle 0 (all frequencies zero)
    rope = None if no_rope else rope_of(w)
    if rope is not None:
        rope.t_scale = t_scale
    om = np.zeros_like(omega_of(w)) if no_rope else omega_of(w)
    oracles = [StreamOracle(w.H, w.D, w.grid_h, w.grid_w, om, w.pairs, w.t_offset, t_scale=t_scale,
                            n_sink=n_sink, n_local=n_local) for _ in range(B)]
    c = w.query_frames
    worst = (0.0, 0.0)
    for f0 in frames:
        parts = [W.qkv_frames(w, layer + 100 * b, f0, c) for b in range(B)]
        q = torch.cat([p[0] for p in parts], 0)
        k = torch.cat([p[1] for p in parts], 0)
        v = torch.cat([p[2] for p in parts], 0)
        if q_scale != 1.0:
            q = (q.float() * q_scale).to(q.dtype)
        if k_scale is not None:
            k = (k.float() * k_scale(f0)).to(k.dtype)
        swa.kvcache_append(cache, k.cuda(), v.cuda(), f0, rope)
        lse = torch.empty(B, w.H, q.shape[1], device="cuda", dtype=torch.float32)
        out = (attend or swa.sink_window_attention)(q.cuda(), cache, f0, rope, lse=lse, softmax_scale=scale or 0.0)
        Tq = q.shape[1]
        rows = np.arange(Tq) if Tq <= 256 else sample_rows(Tq, rows_per_step, f0)
        for b in range(B):
            oracles[b].append(f0, np64(k[b]), np64(v[b]))
            ref, ref_lse = oracles[b].attend(np64(q[b]), f0, scale=scale, rows=rows, return_lse=True)
            got = np64(out[b])[rows]
            r = assert_parity(got, ref, max_rel=max_rel, mean_abs=mean_abs, what=f"{w.name} frame {f0} b {b}")
            worst = (max(worst[0], r[0]), max(worst[1], r[1]))
            if check_lse:
                # natural-log normaliser: 1e-3 of its largest magnitude at most,
                # 5e-3 (0.5 % of the partition function) on average
                assert_parity(lse[b].cpu().numpy()[:, rows], ref_lse, max_rel=lse_rel, mean_abs=lse_mean, what="lse")
    return worst


def test_attention_tiny_full_stream():
    """fp32 / tf32 workload: 20 frames, every output element checked."""
    w = W.TINY
    run_stream(w, range(w.frames))


def test_attention_tiny_bf16_and_peaked():
    """bf16 storage of the tiny workload, then a peaked softmax: Q x 2 gives a
    logit std of about 2 (the tiny inputs are N(0,1), D=64), the same as the
    Wan-shaped workload with Q x 8."""
    w = W.replace(W.TINY, dtype="bf16", name="tiny_bf16")
    run_stream(w, range(16))
    # unit-variance inputs give |O| ~ 1 (4x the Wan-shaped outputs) and the
    # peaked softmax amplifies the bf16 rounding of K and P; the absolute mean
    # bar is scaled with the output magnitude for this variant
    run_stream(w, range(16), q_scale=2.0, mean_abs=2e-3, lse_rel=2e-3)


def test_attention_tiny_d128_batch2():
    w = W.replace(W.TINY, dtype="bf16", D=128, pairs=(22, 21, 21), name="tiny_d128")
    run_stream(w, range(14), B=2)


@pytest.mark.parametrize("n_sink,n_local", [(0, 5), (1, 1), (4, 12)])
def test_attention_other_windows(n_sink, n_local):
    """Other cache shapes: a pure sliding window without sinks, one sink plus
    only the current frame, and a longer window; 20 frames through warm-up
    and several ring wraps, every output element checked."""
    w = W.replace(W.TINY, dtype="bf16", D=128, pairs=(22, 21, 21), name=f"tiny_w{n_sink}_{n_local}")
    run_stream(w, range(20), n_sink=n_sink, n_local=n_local)


def test_attention_max_heads():
    """H = 64 (the largest head count the descriptors carry), with jitter on
    every head; every output element checked. The tiny inputs have unit
    variance, so the logits have unit scale (the Wan frame's 0.25): the LSE
    bar is the sharper-softmax one (2e-3 of its largest magnitude)."""
    w = W.replace(W.TINY, dtype="bf16", H=64, name="tiny_h64", sigma_t=0.8, jitter_seed=9)
    run_stream(w, range(6), lse_rel=2e-3)


def test_attention_wan_warmup_and_steady():
    """Wan-shaped single layer: frames 0..13 cover the warm-up (1..11 valid
    slots), the first ring wrap (frame 12) and steady state."""
    w = W.WAN
    run_stream(w, range(14), rows_per_step=24)


def test_attention_wan_peaked():
    w = W.WAN
    run_stream(w, [0, 1, 2, 3], rows_per_step=24, q_scale=8.0)


def test_attention_wan_growing_logits():
    """Keys of later frames scaled up (K x (1 + f), Q x 4): a row's logit max
    grows by far more than 2^8 (in the exp2 domain) between the first key
    tiles of a piece and the later ones, so the kernel's rescale (O and the
    row sum scaled to the new max, P computed again from S) runs on most rows.
    Q and K go in already rotated (no RoPE in the kernels), so the inputs the
    kernel multiplies are exactly the oracle's: with logits up to ~20, a
    rotation rounded to bf16 would move them by ~2^-9 * |logit|, more than
    the bar allows for a softmax this sharp."""
    w = W.WAN
    run_stream(w, range(5), rows_per_step=24, q_scale=4.0, k_scale=lambda f: 1.0 + f, no_rope=True)


def test_attention_chunk_position_interpolation():
    """3-frame chunks with jitter, temporal offset 2000 and position
    interpolation 1/8 on Q and K (append and attention)."""
    run_stream(W.CHUNK, range(0, 18, 3), rows_per_step=24, t_scale=0.125)


def test_phase_coherence_matches_oracle():
    """ll_phase_coherence against the oracle's C_h(D) for the 12 jittered heads
    of the chunk workload: offsets around 0, far offsets (10^6 frames) and a
    position-interpolated band; fp64 on both sides, fp32 output."""
    w = W.CHUNK
    om = omega_of(w)
    pt = w.pairs[0]
    for delta0, n, ts in [(-64, 4096, 1.0), (10**6, 512, 1.0), (-64, 2048, 0.25)]:
        r = rope_of(w)
        r.t_scale = ts
        got = swa.phase_coherence(r, w.H, delta0, n).cpu().numpy().astype(np.float64)
        d = np.arange(delta0, delta0 + n, dtype=np.float64) * ts
        for h in range(w.H):
            ref = orope.phase_coherence(om[h, :pt], d)
            err = np.abs(got[h, :, 0] + 1j * got[h, :, 1] - ref)
            assert err.max() <= 1e-6, (h, delta0, err.max())


def test_attention_chunk_jitter():
    """3-frame chunks with LoL jitter and temporal offset 2000."""
    w = W.CHUNK
    run_stream(w, range(0, 18, 3), rows_per_step=24)


@pytest.mark.parametrize("name,frames", [("wan", range(14)), ("chunk", range(0, 15, 3))])
def test_attention_fp8_cache(name, frames):
    """E4M3 KV cache (per (token, head) scale): attention against the
    unquantised fp64 reference, max|err| <= 5e-2 * max|ref|."""
    w = W.WORKLOADS[name]
    run_stream(w, frames, dtype="fp8", rows_per_step=24, mean_abs=5e-3, lse_rel=5e-3, max_rel=5e-2)


@pytest.mark.parametrize("name,frames", [("wan", range(14)), ("chunk", range(0, 15, 3))])
def test_attention_fp8_mma(name, frames):
    """E4M3 cache on the FP8 tensor cores (ll_sink_window_attention_fp8_mma:
    Q quantised per tile, S and P' V as kind::f8f6f4 MMAs over the cache's
    codes) through warm-up, the ring wrap and steady state, against the
    unquantised fp64 reference at the FP8 bars."""
    w = W.WORKLOADS[name]
    run_stream(w, frames, dtype="fp8", rows_per_step=24, mean_abs=5e-3, lse_rel=5e-3, max_rel=5e-2,
               attend=swa.sink_window_attention_fp8_mma)


def test_attention_fp8_mma_small_batch2():
    """The FP8 tensor-core attention on two batch entries of a small chunk
    stream (4 heads, 6x10 grid: 60 tokens per frame, so every key count is a
    ragged multiple of the 128-key tile), every output row checked."""
    w = W.replace(W.CHUNK, name="chunk_small_fp8", H=4, grid_h=6, grid_w=10, t_offset=500)
    run_stream(w, range(0, 18, 3), dtype="fp8", B=2, mean_abs=5e-3, lse_rel=5e-3, max_rel=5e-2,
               attend=swa.sink_window_attention_fp8_mma)


def test_attention_fp8_cache_d64_staged():
    """E4M3 cache at D = 64 (dequantised into a bf16 staging copy, then the
    bf16 kernel): 3-frame chunks on a 6x10 grid with the chunk workload's
    input scale, jitter and temporal offset, every output row checked against
    the FP8 bars."""
    w = W.replace(W.CHUNK, name="chunk_d64_fp8", H=3, D=64, pairs=(12, 10, 10), grid_h=6, grid_w=10, t_offset=500)
    run_stream(w, range(0, 18, 3), dtype="fp8", rows_per_step=512, mean_abs=5e-3, lse_rel=5e-3, max_rel=5e-2)


def test_attention_chunk_d64_batch3():
    """3-frame chunks at D = 64 (bf16), three independent streams in one call,
    jitter and a temporal offset: 180 query rows per chunk (a full and a
    ragged 52-row query tile), 720 keys (a ragged 80-key last tile); every
    output row is checked."""
    w = W.replace(W.CHUNK, name="chunk_d64", H=3, D=64, pairs=(12, 10, 10), grid_h=6, grid_w=10, t_offset=500)
    run_stream(w, range(0, 18, 3), B=3)


def test_attention_softmax_scale():
    """A softmax scale other than 1/sqrt(D) reaches the kernel and the oracle."""
    w = W.replace(W.TINY, dtype="bf16", name="tiny_bf16")
    run_stream(w, range(14), scale=0.05)


def test_attention_deterministic():
    """The split of the key range over CTAs and the merge order are fixed, so
    repeated launches on the same inputs give bit-identical outputs."""
    w = W.WAN
    cache = swa.KVCache(w.B, w.H, w.D, w.N, w.dtype)
    rope = rope_of(w)
    for f in range(13):
        _, k, v = W.qkv_frames(w, 0, f, 1)
        swa.kvcache_append(cache, k.cuda(), v.cuda(), f, rope)
    q = W.qkv_frames(w, 0, 12, 1)[0].cuda()
    outs = [swa.sink_window_attention(q, cache, 12, rope).clone() for _ in range(3)]
    torch.cuda.synchronize()
    assert all(torch.equal(outs[0], o) for o in outs[1:])


@pytest.mark.parametrize("chunk", [False, True])
def test_attention_denoising_passes(chunk):
    """Several denoising passes per frame: each pass appends the frame's K/V
    again (the library is stateless, so the frame's slot is simply
    re-written) and attends; every pass is checked against the oracle stream
    with the pass's K/V in place of the current frames'."""
    w = W.replace(W.TINY, dtype="bf16", D=128, pairs=(22, 21, 21), name="tiny_passes", sigma_t=0.8, jitter_seed=3,
                  query_frames=3 if chunk else 1, t_offset=700)
    cache = swa.KVCache(1, w.H, w.D, w.N, "bf16")
    rope = rope_of(w)
    so = StreamOracle(w.H, w.D, w.grid_h, w.grid_w, omega_of(w), w.pairs, w.t_offset)
    c = w.query_frames
    for f0 in range(0, 15, c):
        for ps in range(4):
            q, k, v = W.qkv_frames(w, 10 * ps, f0, c)   # a different draw per pass
            swa.kvcache_append(cache, k.cuda(), v.cuda(), f0, rope)
            out = swa.sink_window_attention(q.cuda(), cache, f0, rope)
            so.append(f0, np64(k[0]), np64(v[0]), replace=ps > 0)
            ref = so.attend(np64(q[0]), f0)
            assert_parity(np64(out[0]), ref, what=f"frame {f0} pass {ps}")


@pytest.mark.parametrize("name", ["wan", "chunk", "tiny", "tiny_d64_b2", "wan_fp8", "chunk_fp8", "tiny_d64_b2_fp8"])
def test_fused_append_attention_matches_separate_calls(name):
    """ll_append_and_attend gives bit-identical outputs, LSE and cache contents
    (codes and scales for an E4M3 cache) to ll_kvcache_append followed by
    ll_sink_window_attention, from the first frame through the ring wrap."""
    fp8 = name.endswith("_fp8")
    base = name[:-4] if fp8 else name
    w = {"wan": W.WAN, "chunk": W.CHUNK, "tiny": W.TINY,
         "tiny_d64_b2": W.replace(W.TINY, dtype="bf16", name="tiny_d64_b2", B=2)}[base]
    rope = rope_of(w)
    c = w.query_frames
    caches = [swa.KVCache(w.B, w.H, w.D, w.N, "fp8" if fp8 else w.dtype) for _ in range(2)]
    frames = range(0, 15, c) if w.N < 100 else [0, 3 * c, 11, 12 * c] if c == 1 else [0, 3, 9, 12]
    for f0 in frames:
        q, k, v = (t.cuda() for t in W.qkv_frames(w, 0, f0, c))   # [w.B, c*N, H, D]
        lse = [torch.empty(w.B, w.H, q.shape[1], device="cuda", dtype=torch.float32) for _ in range(2)]
        swa.kvcache_append(caches[0], k, v, f0, rope)
        o0 = swa.sink_window_attention(q, caches[0], f0, rope, lse=lse[0])
        o1 = swa.append_and_attend(caches[1], k, v, q, f0, rope, lse=lse[1])
        torch.cuda.synchronize()
        assert torch.equal(o0, o1), f"frame {f0}"
        assert torch.equal(lse[0], lse[1]), f"frame {f0}"
        assert torch.equal(caches[0].k, caches[1].k) and torch.equal(caches[0].v, caches[1].v), f"frame {f0}"
        if fp8:
            assert torch.equal(caches[0].k_scale, caches[1].k_scale), f"frame {f0}"
            assert torch.equal(caches[0].v_scale, caches[1].v_scale), f"frame {f0}"


def test_fused_append_attention_stream_parity():
    """The fused call against the oracle stream: chunks with jitter."""
    w = W.CHUNK
    cache = swa.KVCache(w.B, w.H, w.D, w.N, w.dtype)
    rope = rope_of(w)
    so = StreamOracle(w.H, w.D, w.grid_h, w.grid_w, omega_of(w), w.pairs, w.t_offset)
    for f0 in range(0, 18, 3):
        q, k, v = W.qkv_frames(w, 0, f0, 3)
        out = swa.append_and_attend(cache, k.cuda(), v.cuda(), q.cuda(), f0, rope)
        so.append(f0, np64(k[0]), np64(v[0]))
        rows = sample_rows(q.shape[1], 24, f0)
        ref = so.attend(np64(q[0]), f0, rows=rows)
        assert_parity(np64(out[0])[rows], ref, what=f"fused chunk {f0}")


def test_fused_append_attention_fp8_stream_parity():
    """The fused call over an E4M3 cache against the oracle stream: Wan frames
    with jitter through the ring wrap, at the FP8 bars."""
    w = W.replace(W.WAN, sigma_t=0.8, jitter_seed=6, name="wan_jitter")
    cache = swa.KVCache(w.B, w.H, w.D, w.N, "fp8")
    rope = rope_of(w)
    so = StreamOracle(w.H, w.D, w.grid_h, w.grid_w, omega_of(w), w.pairs, w.t_offset)
    for f0 in range(14):
        q, k, v = W.qkv_frames(w, 0, f0, 1)
        out = swa.append_and_attend(cache, k.cuda(), v.cuda(), q.cuda(), f0, rope)
        so.append(f0, np64(k[0]), np64(v[0]))
        rows = sample_rows(q.shape[1], 24, f0)
        ref = so.attend(np64(q[0]), f0, rows=rows)
        assert_parity(np64(out[0])[rows], ref, max_rel=5e-2, mean_abs=5e-3, what=f"fused fp8 frame {f0}")
