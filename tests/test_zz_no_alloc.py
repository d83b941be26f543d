"""The allocation-free attention entry point, ll_sink_window_attention_noalloc.

It is for callers that cannot call cudaMalloc (it may synchronise the whole
device, which a frame-rate loop cannot afford; plugin hosts that own all device
memory forbid allocation outside their pools). It runs the same attention with
the library's static scratch array instead of a caller workspace. This file is
collected last so that a run stopping at the first failure has run every other
test before it; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import sink_window_attention_b200 as swa
import swa_workloads as W
from tests.conftest import assert_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from sink_window_attention_b200 import build
    build.build()
    swa.lib()


def test_noalloc_matches_workspace_entry_point():
    w = W.WAN
    eps = W.jitter_eps(4, w.H)
    rope = swa.Rope(pairs=w.pairs, grid_h=w.grid_h, grid_w=w.grid_w, theta0=w.theta0, sigma_t=0.8,
                    eps=[float(e) for e in eps])
    cache = swa.KVCache(1, w.H, w.D, w.N, "bf16")
    assert swa.attention_workspace_bytes(cache, 1) <= swa.NOALLOC_SCRATCH_BYTES
    for f in range(12):
        _, k, v = W.qkv_frames(w, 5, f, 1, device="cuda")
        swa.kvcache_append(cache, k, v, f, rope)
    for f in (12, 13):
        q, k, v = W.qkv_frames(w, 5, f, 1, device="cuda")
        swa.kvcache_append(cache, k, v, f, rope)
        lse_ref = torch.empty(1, w.H, w.N, device="cuda")
        ref = swa.sink_window_attention(q, cache, f, rope, lse=lse_ref)
        # two calls in a row on the shared static scratch
        for _ in range(2):
            lse = torch.empty_like(lse_ref)
            out = swa.sink_window_attention_noalloc(q, cache, f, rope, lse=lse)
            torch.cuda.synchronize()
            assert_parity(out.double().cpu().numpy(), ref.double().cpu().numpy(), what=f"noalloc frame {f}")
            assert_parity(lse.cpu().numpy(), lse_ref.cpu().numpy(), max_rel=1e-3, mean_abs=5e-3, what="lse")
    assert swa.device_error() == 0


def test_noalloc_rejects_an_fp8_wan_cache():
    """Attention over an E4M3 cache reads a bf16 staging copy of the occupied
    rows (about 115 MB for the Wan-shaped layer) that lives in the scratch:
    far beyond the static array, so the call is refused before any launch."""
    w = W.WAN
    cache = swa.KVCache(1, w.H, w.D, w.N, "fp8")
    assert swa.attention_workspace_bytes(cache, 1) > swa.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(1, w.N, w.H, w.D, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(swa.LLError) as e:
        swa.sink_window_attention_noalloc(q, cache, 20, None)
    assert e.value.status == swa.LL_ERR_INVALID_ARG and "static scratch" in str(e.value)


def test_noalloc_rejects_requests_beyond_the_static_scratch():
    c = swa.KVCacheC()
    c.k, c.v = 4096, 8192            # never dereferenced: the size check comes first
    c.k_scale = c.v_scale = None
    c.dtype, c.B, c.H, c.D = swa.LL_BF16, 8, 64, 128
    c.tokens_per_frame, c.n_sink, c.n_local = 1560, 3, 9
    need = swa.lib().ll_sink_window_attention_workspace_bytes(ctypes.byref(c), 1)
    assert need > swa.NOALLOC_SCRATCH_BYTES
    st = swa.lib().ll_sink_window_attention_noalloc(1 << 20, swa.LL_BF16, ctypes.byref(c), 20, 1, None, 0.0,
                                                    1 << 21, None, None)
    assert st == swa.LL_ERR_INVALID_ARG
    assert "static scratch" in swa.last_error()


def test_noalloc_warm_call_allocates_no_device_memory():
    """The point of the entry point: once the first call on the device has
    looked up the static array, further calls take no device memory at all
    (free memory as reported by cudaMemGetInfo is unchanged across them)."""
    w = W.WAN
    rope = swa.Rope(pairs=w.pairs, grid_h=w.grid_h, grid_w=w.grid_w, theta0=w.theta0)
    cache = swa.KVCache(1, w.H, w.D, w.N, "bf16")
    for f in range(12):
        _, k, v = W.qkv_frames(w, 6, f, 1, device="cuda")
        swa.kvcache_append(cache, k, v, f, rope)
    q = W.qkv_frames(w, 6, 11, 1, device="cuda")[0]
    out = torch.empty_like(q)
    lse = torch.empty(1, w.H, w.N, device="cuda")
    swa.sink_window_attention_noalloc(q, cache, 11, rope, out=out, lse=lse)   # first call: symbol lookup
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        swa.sink_window_attention_noalloc(q, cache, 11, rope, out=out, lse=lse)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert swa.device_error() == 0
