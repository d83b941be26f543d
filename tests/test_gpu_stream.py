"""GPU parity of the stream as the benchmark drives it, and of the 30-layer
prompt switch, against the fp64 oracle stream.

LongLive review, "KV Recache": at a prompt switch the cached frames' K/V are
recomputed with the new prompt and later frames attend over the rebuilt
cache; "Frame Sink" and "Short-Window Attention": every frame attends to the
3 sink frames plus the most recent local frames.

* The benchmark's own stream driver (bench.Stream: per frame and layer the
  fused append + attention for a bf16 cache, the append with the bf16
  staging copy then attention for an E4M3 cache, or the append then the FP8
  tensor-core attention; at a switch the recache of every layer) runs frames 12..52 of
  several layers with a prompt switch before frame 40; sampled query rows of
  every layer at frames 28..52 are compared with one oracle stream per layer
  fed the same pooled inputs and the same hidden states and projections.
* The 30-layer switch: every layer is recached before frame 40 (K and V of
  sampled rows of every slot checked), then 12 single-frame steps (frames
  40..51) run through all 30 layers with sampled rows of every step checked.

Bars: bf16 max|err| <= 1e-2 max|ref|, mean|err| <= 1e-3; an E4M3 cache
5e-2 max|ref| and mean 5e-3 against the unquantised reference."""
import numpy as np
import pytest
import torch

import bench
import sink_window_attention_b200 as swa
import swa_workloads as W
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


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def sample_rows(N: int, n: int, seed: int) -> np.ndarray:
    """The first and last rows, both sides of every 128-row tile boundary and
    n random rows."""
    rng = np.random.default_rng(seed)
    fixed = {0, N - 1}
    for b in range(128, N, 128):
        fixed |= {b - 1, b}
    return np.array(sorted(fixed | set(rng.choice(N, size=n, replace=False).tolist())))


def oracle_stream(w: W.Workload) -> StreamOracle:
    eps = w.eps
    om = orope.head_frequencies(w.H, w.pairs, w.theta0, w.sigma_t, None if eps is None else eps.astype(np.float64))
    return StreamOracle(w.H, w.D, w.grid_h, w.grid_w, om, w.pairs, w.t_offset)


@pytest.mark.parametrize("cache", ["bf16", "fp8", "fp8mma"])
def test_bench_stream_across_prompt_switch(cache):
    layers, switch, last, check_from = 3, 40, 53, 28
    w = W.replace(W.STREAM if cache == "bf16" else W.STREAM_FP8, layers=layers)
    # fp8mma: the E4M3 cache read by the FP8 tensor-core attention (fp8_mma_stream of the bench line)
    st = bench.Stream(w, "fp8" if cache == "fp8mma" else cache, "cuda", fp8_mma=cache == "fp8mma")
    N, P = w.N, bench.POOL
    rows = sample_rows(N, 8, 0)
    rows_dev = torch.as_tensor(rows, device="cuda")
    got = {}

    def grab(f, l, out):
        if f >= check_from:
            got[(f, l)] = out[0].index_select(0, rows_dev).clone()

    st.frames(12, switch, on_output=grab)
    st.switch(switch)
    st.frames(switch, last, on_output=grab)
    torch.cuda.synchronize()
    assert swa.device_error() == 0
    assert sorted(got) == [(f, l) for f in range(check_from, last) for l in range(layers)]

    bars = dict(max_rel=5e-2, mean_abs=5e-3) if cache != "bf16" else {}
    # the hidden states are in slot order: slot s holds the frame the oracle's
    # own slot map puts there after frame switch - 1
    held = owin.slot_frames(switch - 1)
    for l in range(layers):
        so = oracle_stream(w)
        qkv = lambda f: (np64(st.q[l][f % P][0]), np64(st.k[l][f % P][0]), np64(st.v[l][f % P][0]))
        for f in range(last):
            if f == switch:
                X = np64(st.rx[l][0])
                so.recache(switch, {g: X[s * N:(s + 1) * N] for s, g in enumerate(held)}, np64(st.rwk[l]),
                           np64(st.rwv[l]), np64(st.rg[l]), EPS)
            q, k, v = qkv(f)
            so.append(f, k, v)
            if f >= check_from:
                ref = so.attend(q, f, rows=rows)
                assert_parity(np64(got[(f, l)]), ref, what=f"{cache} stream layer {l} frame {f}", **bars)


def test_switch_thirty_layers_then_twelve_steps():
    """A prompt switch before frame 40 on the Wan-shaped 30-layer stack: every
    layer's 12 cached frames are recomputed from X [18720, 1536] with its own
    Wk, Wv and gamma, then frames 40..51 run through all 30 layers (fused
    append + attention)."""
    w = W.RECACHE
    switch, steps, N = 40, 12, w.N
    rope = swa.Rope(pairs=w.pairs, grid_h=w.grid_h, grid_w=w.grid_w, theta0=w.theta0, t_offset=w.t_offset)
    held = owin.slot_frames(switch - 1)
    assert min(held) >= 0
    rows = sample_rows(N, 8, 1)
    rows_dev = torch.as_tensor(rows, device="cuda")
    caches, inputs, got = [], [], {}
    for l in range(w.layers):
        x, wk, wv, gamma = W.recache_inputs(w, l, switch, device="cuda")
        cache = swa.KVCache(1, w.H, w.D, N, "bf16")
        swa.kv_recache(cache, x, wk, wv, gamma, EPS, held, rope)
        caches.append(cache)
        inputs.append((x, wk, wv, gamma))
    # recache: sampled rows of every slot of every layer (RMSNorm and RoPE act
    # row by row, so rows are independent)
    rr = sample_rows(N, 6, 2)
    for l in range(w.layers):
        x, wk, wv, gamma = (np64(t) for t in inputs[l])
        x = x[0]
        for s, g in enumerate(held):
            xr = x[s * N:(s + 1) * N][rr]
            k = orec.rmsnorm(xr @ wk, gamma, EPS).reshape(-1, w.H, w.D)
            t, r, c = orope.token_positions(g, w.grid_h, w.grid_w, w.t_offset)
            kref = orope.rope_3d(k, t[rr], r[rr], c[rr], oracle_stream(w).omega, w.pairs)
            vref = (xr @ wv).reshape(-1, w.H, w.D)
            gk = np64(caches[l].k[0, s * N:(s + 1) * N])[rr]
            gv = np64(caches[l].v[0, s * N:(s + 1) * N])[rr]
            assert_parity(gk, kref, mean_abs=2.0 ** -8 * np.abs(kref).mean(), what=f"K layer {l} slot {s}")
            assert_parity(gv, vref, mean_abs=2.0 ** -8 * np.abs(vref).mean(), what=f"V layer {l} slot {s}")
    # 12 single-frame steps through the 30 layers
    out = torch.empty((1, N, w.H, w.D), dtype=torch.bfloat16, device="cuda")
    for f in range(switch, switch + steps):
        for l in range(w.layers):
            q, k, v = W.qkv_frames(w, l, f, 1, device="cuda")
            swa.append_and_attend(caches[l], k, v, q, f, rope, out=out)
            got[(f, l)] = out[0].index_select(0, rows_dev).clone()
    torch.cuda.synchronize()
    assert swa.device_error() == 0
    for l in range(w.layers):
        x, wk, wv, gamma = (np64(t) for t in inputs[l])
        so = oracle_stream(w)
        so.last = switch - 1      # the history before the switch is entirely recomputed
        so.recache(switch, {g: x[0][s * N:(s + 1) * N] for s, g in enumerate(held)}, wk, wv, gamma, EPS)
        for f in range(switch, switch + steps):
            q, k, v = (np64(t[0]) for t in W.qkv_frames(w, l, f, 1, device="cuda"))
            so.append(f, k, v)
            assert_parity(np64(got[(f, l)]), so.attend(q, f, rows=rows), what=f"layer {l} frame {f}")
