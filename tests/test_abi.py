"""The C ABI without a GPU: the library loads, exports every function that
include/ll_api.h declares, the binding passes each argument with the
header's type and lays out its structures as the C compiler does, frames map
to slots bit-exactly, and bad arguments are rejected on the host before
anything is launched."""
import ctypes
import os
import re

import pytest

import sink_window_attention_b200 as swa
from oracle import window
from tests.conftest import ROOT


@pytest.fixture(scope="module")
def L():
    from sink_window_attention_b200 import build
    build.build()
    return swa.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ll_api.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ll_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(swa.EXPORTED)
    assert swa.abi_version() == swa.ABI_VERSION == 2


@pytest.mark.parametrize("n_sink,n_local", [(3, 9), (0, 5), (2, 1), (4, 12)])
def test_slot_map_bit_exact(L, n_sink, n_local):
    for f in list(range(0, 300)) + [10**6 + 7, 2**40 + 3]:
        assert swa.slot_of_frame(f, n_sink, n_local) == window.slot_of(f, n_sink, n_local)


def test_slot_map_rejects(L):
    with pytest.raises(swa.LLError) as e:
        swa.slot_of_frame(-1)
    assert e.value.status == swa.LL_ERR_INVALID_ARG


def _cache(**kw):
    c = swa.KVCacheC()
    c.k, c.v = 4096, 8192            # fake device addresses: never dereferenced on these paths
    c.k_scale = c.v_scale = None
    c.dtype, c.B, c.H, c.D = swa.LL_BF16, 1, 12, 128
    c.tokens_per_frame, c.n_sink, c.n_local = 1560, 3, 9
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def _rope(**kw):
    r = swa.Rope(pairs=(22, 21, 21), grid_h=30, grid_w=52).to_c()
    for k, v in kw.items():
        setattr(r, k, v)
    return r


def _attn(L, cache, rope=None, first=0, nq=1, scale=0.0, ws=None, ws_bytes=0, q=1 << 20, out=1 << 21,
          qdt=swa.LL_BF16, lse=None):
    return L.ll_sink_window_attention(q, qdt, ctypes.byref(cache), first, nq,
                                      ctypes.byref(rope) if rope is not None else None, scale, out, lse, ws,
                                      ws_bytes, None)


def test_attention_validation(L):
    """Every case fails its own check (the workspace is large enough, so the
    error cannot come from the workspace check), before anything launches."""
    ws = dict(ws=1 << 24, ws_bytes=1 << 40)
    fp8 = dict(dtype=swa.LL_FP8_E4M3, k_scale=1 << 22, v_scale=1 << 23)
    bad = [
        (dict(cache=_cache(k=None)), "NULL"),
        (dict(cache=_cache(D=100)), "multiple of 16"),
        (dict(cache=_cache(H=65)), "exceeds"),
        (dict(cache=_cache(n_local=0)), "n_local"),
        (dict(cache=_cache(tokens_per_frame=1 << 28)), "2^31"),     # cache rows overflow 32 bits
        (dict(cache=_cache(dtype=swa.LL_FP8_E4M3)), "k_scale"),     # FP8 without scales
        (dict(cache=_cache(), first=-1), "first_frame"),
        (dict(cache=_cache(), nq=0), "n_query_frames"),
        (dict(cache=_cache(), nq=10), "n_query_frames"),
        (dict(cache=_cache(), scale=-1.0), "softmax_scale"),
        (dict(cache=_cache(), q=None), "non-NULL"),
        (dict(cache=_cache(), q=(1 << 20) + 2), "aligned"),
        (dict(cache=_cache(), qdt=swa.LL_F32), "q dtype"),
        (dict(cache=_cache(), lse=(1 << 25) + 2), "lse"),
        (dict(cache=_cache(), rope=_rope(pairs_t=10)), "sum to D/2"),
        (dict(cache=_cache(), rope=_rope(grid_w=51)), "does not match"),
        (dict(cache=_cache(), rope=_rope(theta0=0.5)), "theta0"),
        (dict(cache=_cache(), rope=_rope(sigma_t=1.5)), "sigma_t"),
        # an FP8 cache is dequantised by a kernel: a bad rope must be caught first
        (dict(cache=_cache(**fp8), rope=_rope(pairs_t=10)), "sum to D/2"),
    ]
    for kw, msg in bad:
        st = _attn(L, **{**ws, **kw})
        assert st == swa.LL_ERR_INVALID_ARG, (kw, st, swa.last_error())
        assert msg in swa.last_error(), (kw, swa.last_error())
    assert _attn(L, _cache(), ws=1 << 24, ws_bytes=16) == swa.LL_ERR_INVALID_ARG
    assert "workspace" in swa.last_error()


def test_fp8_mma_attention_validation(L):
    """The FP8 tensor-core entry point takes only an E4M3 cache with D = 128 and
    H a multiple of 4, a BF16 q, and the rest as ll_sink_window_attention;
    every case fails on the host before the scale pass is launched."""
    fp8 = dict(dtype=swa.LL_FP8_E4M3, k_scale=1 << 22, v_scale=1 << 23)

    def call(cache, rope=None, first=0, nq=1, scale=0.0, ws=1 << 24, ws_bytes=1 << 40, q=1 << 20, qdt=swa.LL_BF16):
        return L.ll_sink_window_attention_fp8_mma(q, qdt, ctypes.byref(cache), first, nq,
                                                  ctypes.byref(rope) if rope is not None else None, scale,
                                                  1 << 21, None, ws, ws_bytes, None)

    need = L.ll_sink_window_attention_fp8_mma_workspace_bytes(ctypes.byref(_cache(**fp8)), 1)
    assert need > 0
    # larger than the bf16 kernel's scratch for the same frames: + the [B][H] V-scale maxima
    assert need >= L.ll_sink_window_attention_workspace_bytes(ctypes.byref(_cache()), 1) + 12 * 4
    assert L.ll_sink_window_attention_fp8_mma_workspace_bytes(ctypes.byref(_cache()), 1) == 0
    assert L.ll_sink_window_attention_fp8_mma_workspace_bytes(ctypes.byref(_cache(D=64, **fp8)), 1) == 0
    cases = [
        (dict(cache=_cache()), swa.LL_ERR_INVALID_ARG, "FP8_E4M3"),
        (dict(cache=_cache(dtype=swa.LL_FP8_E4M3)), swa.LL_ERR_INVALID_ARG, "k_scale"),
        (dict(cache=_cache(D=64, **fp8)), swa.LL_ERR_UNSUPPORTED, "D = 128"),
        (dict(cache=_cache(H=6, **fp8)), swa.LL_ERR_UNSUPPORTED, "multiple of 4"),
        (dict(cache=_cache(**fp8), qdt=swa.LL_F32), swa.LL_ERR_INVALID_ARG, "BF16"),
        (dict(cache=_cache(**fp8), nq=10), swa.LL_ERR_INVALID_ARG, "n_query_frames"),
        (dict(cache=_cache(**fp8), first=-1), swa.LL_ERR_INVALID_ARG, "first_frame"),
        (dict(cache=_cache(**fp8), scale=float("nan")), swa.LL_ERR_INVALID_ARG, "softmax_scale"),
        (dict(cache=_cache(**fp8), q=(1 << 20) + 2), swa.LL_ERR_INVALID_ARG, "aligned"),
        (dict(cache=_cache(**fp8), ws_bytes=16), swa.LL_ERR_INVALID_ARG, "workspace"),
        (dict(cache=_cache(**fp8), rope=_rope(pairs_t=10)), swa.LL_ERR_INVALID_ARG, "sum to D/2"),
        (dict(cache=_cache(**fp8), rope=_rope(grid_w=51)), swa.LL_ERR_INVALID_ARG, "does not match"),
    ]
    for kw, want, msg in cases:
        st = call(**kw)
        assert st == want, (kw, st, swa.last_error())
        assert msg in swa.last_error(), (kw, swa.last_error())


def test_append_and_rope_validation(L):
    k = v = 1 << 20
    rc = ctypes.byref(_rope())
    c = _cache()
    slots = (ctypes.c_int * 16)()
    assert L.ll_kvcache_append(ctypes.byref(c), None, v, swa.LL_BF16, 0, 1, rc, slots, None) == swa.LL_ERR_INVALID_ARG
    assert L.ll_kvcache_append(ctypes.byref(c), k, v, swa.LL_BF16, 0, 10, rc, slots, None) == swa.LL_ERR_INVALID_ARG
    assert L.ll_kvcache_append(ctypes.byref(c), k, v, swa.LL_F32, 0, 1, rc, slots, None) == swa.LL_ERR_INVALID_ARG
    assert L.ll_kvcache_append(ctypes.byref(c), k, v, swa.LL_BF16, -3, 1, rc, slots, None) == swa.LL_ERR_INVALID_ARG
    eps = (ctypes.c_float * 12)(*([0.0] * 11 + [1.5]))
    r = _rope(sigma_t=0.8)
    r.eps_h = ctypes.cast(eps, ctypes.POINTER(ctypes.c_float))
    assert L.ll_kvcache_append(ctypes.byref(c), k, v, swa.LL_BF16, 0, 1, ctypes.byref(r), slots, None) == swa.LL_ERR_INVALID_ARG
    assert "eps_h[11]" in swa.last_error()
    assert L.ll_rope_apply(None, swa.LL_BF16, 1, 1, 12, 128, 0, rc, None) == swa.LL_ERR_INVALID_ARG
    assert L.ll_rope_apply(k, swa.LL_FP8_E4M3, 1, 1, 12, 128, 0, rc, None) == swa.LL_ERR_INVALID_ARG
    assert L.ll_rope_apply(k, swa.LL_BF16, 1, 1, 12, 128, 0, None, None) == swa.LL_ERR_INVALID_ARG
    # a grid whose token count overflows 32 bits is rejected, not wrapped
    big = ctypes.byref(_rope(grid_h=65536, grid_w=65536))
    assert L.ll_rope_apply(k, swa.LL_BF16, 1, 1, 12, 128, 0, big, None) == swa.LL_ERR_INVALID_ARG
    assert "2^31" in swa.last_error()
    assert L.ll_kvcache_append(ctypes.byref(c), k, v, swa.LL_BF16, 0, 1, big, slots, None) == swa.LL_ERR_INVALID_ARG


def test_recache_validation(L):
    c = _cache()
    frames = (ctypes.c_longlong * 12)(*range(12))
    g = 1 << 22
    def call(cache=c, n=12, dm=1536, fr=frames, x=1 << 20, gamma=g):
        return L.ll_kv_recache(ctypes.byref(cache), x, dm, 1 << 21, 1 << 21, gamma, 1e-6, fr, n, None, None, 0, None)
    assert call(n=0) == swa.LL_ERR_INVALID_ARG
    assert call(n=13) == swa.LL_ERR_INVALID_ARG
    assert call(x=None) == swa.LL_ERR_INVALID_ARG
    assert call(fr=(ctypes.c_longlong * 12)(*([-1] * 12))) == swa.LL_ERR_INVALID_ARG
    assert call(dm=100) == swa.LL_ERR_UNSUPPORTED
    assert call(cache=_cache(H=3)) == swa.LL_ERR_UNSUPPORTED        # H*D = 384 is not a multiple of 256
    assert call(cache=_cache(dtype=swa.LL_F32)) == swa.LL_ERR_UNSUPPORTED
    assert call(gamma=g + 2) == swa.LL_ERR_INVALID_ARG                    # gamma read as floats
    assert "gamma" in swa.last_error()
    assert call(fr=(ctypes.c_longlong * 12)(*([1 << 40] * 12))) == swa.LL_ERR_INVALID_ARG  # frame beyond 32 bits
    assert "slot_frames[0]" in swa.last_error()
    fp8 = _cache(dtype=swa.LL_FP8_E4M3, k_scale=(1 << 22) + 1, v_scale=1 << 23)
    assert call(cache=fp8) == swa.LL_ERR_INVALID_ARG                      # scales written as floats
    assert "4-byte" in swa.last_error()



def _fused(L, cache, rope=None, first=0, nf=1, scale=0.0, ws=1 << 24, ws_bytes=1 << 30, k=1 << 20, v=1 << 21,
           q=1 << 22, out=1 << 23, dt=swa.LL_BF16):
    return L.ll_append_and_attend(ctypes.byref(cache), k, v, q, dt, first, nf,
                                  ctypes.byref(rope) if rope is not None else None, scale, out, None, ws,
                                  ws_bytes, None)


def test_fused_append_attention_validation(L):
    """Every malformed call is rejected on the host, before any launch."""
    fp8 = _cache(dtype=swa.LL_FP8_E4M3, k_scale=1 << 25, v_scale=1 << 26)
    # FP8: the attention scratch and the bf16 staging copy, as for attention alone
    need8 = L.ll_append_and_attend_workspace_bytes(ctypes.byref(fp8), 1)
    assert need8 == L.ll_sink_window_attention_workspace_bytes(ctypes.byref(fp8), 1) > 0
    assert _fused(L, fp8, ws_bytes=need8 - 1) == swa.LL_ERR_INVALID_ARG
    assert _fused(L, fp8, dt=swa.LL_F32) == swa.LL_ERR_INVALID_ARG     # k, v, q are bf16 for an FP8 cache
    assert _fused(L, _cache(dtype=swa.LL_FP8_E4M3, k_scale=1 << 25, v_scale=1 << 26, D=32),
                  ws_bytes=1 << 34) == swa.LL_ERR_UNSUPPORTED           # no kernel for D = 32
    assert _fused(L, _cache(D=96)) == swa.LL_ERR_UNSUPPORTED        # no kernel for D = 96
    need = L.ll_append_and_attend_workspace_bytes(ctypes.byref(_cache()), 1)
    assert need > L.ll_sink_window_attention_workspace_bytes(ctypes.byref(_cache()), 1)  # + the barrier word
    bad = [
        dict(cache=_cache(), dt=swa.LL_F32),                         # not the cache's dtype
        dict(cache=_cache(), k=None),
        dict(cache=_cache(), q=(1 << 22) + 4),                       # misaligned
        dict(cache=_cache(), first=-1),
        dict(cache=_cache(), nf=0),
        dict(cache=_cache(), nf=10),
        dict(cache=_cache(), scale=float("nan")),
        dict(cache=_cache(), ws_bytes=need - 1),
        dict(cache=_cache(), rope=_rope(grid_h=29)),
    ]
    for kw in bad:
        st = _fused(L, **kw)
        assert st == swa.LL_ERR_INVALID_ARG, (kw, st)
        assert swa.last_error() != ""


def test_phase_coherence_and_position_interpolation_validation(L):
    """ll_phase_coherence and the rope descriptor's t_scale are checked on the
    host; every rejected call returns before a launch."""
    out = 1 << 22
    assert L.ll_phase_coherence(None, 12, 0, 16, out, None) == swa.LL_ERR_INVALID_ARG
    r = _rope()
    assert L.ll_phase_coherence(ctypes.byref(r), 12, 0, 16, None, None) == swa.LL_ERR_INVALID_ARG
    assert L.ll_phase_coherence(ctypes.byref(r), 12, 0, 16, out + 4, None) == swa.LL_ERR_INVALID_ARG  # alignment
    assert L.ll_phase_coherence(ctypes.byref(r), 0, 0, 16, out, None) == swa.LL_ERR_INVALID_ARG
    assert L.ll_phase_coherence(ctypes.byref(r), 65, 0, 16, out, None) == swa.LL_ERR_INVALID_ARG
    assert L.ll_phase_coherence(ctypes.byref(r), 12, 0, 0, out, None) == swa.LL_ERR_INVALID_ARG
    assert L.ll_phase_coherence(ctypes.byref(r), 12, 1 << 41, 16, out, None) == swa.LL_ERR_INVALID_ARG
    assert L.ll_phase_coherence(ctypes.byref(_rope(pairs_t=0, pairs_h=32)), 12, 0, 16, out,
                                None) == swa.LL_ERR_INVALID_ARG
    assert L.ll_phase_coherence(ctypes.byref(r), 64, 0, 1 << 26, out, None) == swa.LL_ERR_UNSUPPORTED
    for bad in (-0.5, 1.5, float("nan")):
        rb = _rope(t_scale=bad)
        assert L.ll_phase_coherence(ctypes.byref(rb), 12, 0, 16, out, None) == swa.LL_ERR_INVALID_ARG
        assert "t_scale" in swa.last_error()
        assert _attn(L, _cache(), rope=rb, ws=1 << 24, ws_bytes=1 << 30) == swa.LL_ERR_INVALID_ARG


def test_binding_rejects_host_tensors_and_mismatched_buffers(L):
    """The Python binding hands the library device addresses only: host tensors,
    and buffers whose shape or dtype the kernels would overrun, are refused
    before any call reaches the library."""
    import torch
    B, H, D, N = 1, 2, 64, 24
    cache = swa.KVCache(B, H, D, N, "bf16", device="cpu")
    rope = swa.Rope(pairs=(12, 10, 10), grid_h=4, grid_w=6)
    q = torch.zeros(B, N, H, D, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensors"):
        swa.sink_window_attention(q, cache, 0, rope)
    with pytest.raises(ValueError, match="lse"):
        swa.sink_window_attention(q, cache, 0, rope, lse=torch.zeros(B, H, N + 1))
    with pytest.raises(ValueError, match="out"):
        swa.sink_window_attention(q, cache, 0, rope, out=torch.zeros(B, N, H, D))   # f32 out for bf16 q
    with pytest.raises(ValueError, match="one dtype"):
        swa.kvcache_append(cache, q, q.float(), 0, rope)
    with pytest.raises(ValueError, match="CUDA tensors"):
        swa.kvcache_append(cache, q, q, 0, rope)
    dm, dout = 256, H * D
    x = torch.zeros(B, N, dm, dtype=torch.bfloat16)
    w = torch.zeros(dm, dout, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="gamma"):
        swa.kv_recache(cache, x, w, w, torch.ones(dout, dtype=torch.bfloat16), 1e-6, [0], rope)
    with pytest.raises(ValueError, match="x must be"):
        swa.kv_recache(cache, x, w, w, torch.ones(dout), 1e-6, [0, 1], rope)                  # 2 slots need 2N rows
    with pytest.raises(ValueError, match="whole number"):
        swa.rope_apply(torch.zeros(B, N + 1, H, D, dtype=torch.bfloat16), 0, rope)


def test_workspace_sizes_and_noalloc_limit(L):
    """Workspace = one arrival counter per unit (128 query rows of one head and
    batch entry), then (#SMs + units) partial slots of 128 x D + 2 x 128 floats
    (148 SMs: the count on a B200, and the fallback without a device); an FP8
    cache adds the bf16 staging copy of K and V. The Wan frame (20 MB) and the
    3-frame chunk (39 MB) fit the 48 MiB no-alloc scratch array."""
    def ws(cache, nq):
        return int(L.ll_sink_window_attention_workspace_bytes(ctypes.byref(cache), nq))
    align = lambda x: (x + 255) // 256 * 256
    slot = (128 * 128 + 2 * 128) * 4
    for nq, units in [(1, 13 * 12), (3, 37 * 12)]:
        want = align(align(units * 4) + (148 + units) * slot)
        assert ws(_cache(), nq) == want
        assert want <= 48 * 1024 * 1024
    assert round(ws(_cache(), 1) / 1e6) == 20 and round(ws(_cache(), 3) / 1e6) == 39
    fp8 = _cache(dtype=swa.LL_FP8_E4M3, k_scale=1 << 22, v_scale=1 << 23)
    staging = 2 * align(12 * 1560 * 12 * 128 * 2)
    assert ws(fp8, 1) == ws(_cache(), 1) + staging
    assert ws(_cache(), 0) == 0 and L.ll_sink_window_attention_workspace_bytes(None, 1) == 0


def _prototypes():
    """(return type, name, [parameter types]) of every function in ll_api.h."""
    src = open(os.path.join(ROOT, "include", "ll_api.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    out = []
    for m in re.finditer(r"([A-Za-z_][A-Za-z0-9_ \*]*?)\b(ll_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", src, flags=re.S):
        params = [p.strip() for p in m.group(3).split(",")]
        if params == ["void"]:
            params = []
        # drop the parameter name, keep its type
        types_ = [re.sub(r"\s*\b[A-Za-z_][A-Za-z0-9_]*$", "", p) if not p.endswith("*") else p for p in params]
        out.append((m.group(1).strip(), m.group(2), [" ".join(t.replace("*", " * ").split()) for t in types_]))
    return out


def _ctype_of(c_type: str):
    """The ctypes type the binding must pass for a C parameter type."""
    t = c_type.replace("const ", "").strip()
    if t == "ll_rope_desc *":
        return ctypes.POINTER(swa.RopeDescC)
    if t == "ll_kvcache *":
        return ctypes.POINTER(swa.KVCacheC)
    if t == "long long *":
        return ctypes.POINTER(ctypes.c_longlong)
    if t == "int *":
        return ctypes.POINTER(ctypes.c_int)
    if t.endswith("*"):
        return ctypes.c_void_p                      # device or host buffers, streams
    return {"int": ctypes.c_int, "ll_dtype": ctypes.c_int, "ll_status": ctypes.c_int, "long long": ctypes.c_longlong,
            "float": ctypes.c_float, "double": ctypes.c_double, "size_t": ctypes.c_size_t}[t]


def test_binding_signatures_match_the_header(L):
    """Every argtypes / restype the binding sets agrees with the prototype in
    ll_api.h, parameter by parameter (count, integer widths, float vs double,
    pointers), so the marshalling cannot shift or truncate an argument."""
    protos = _prototypes()
    assert sorted(n for _, n, _ in protos) == sorted(swa.EXPORTED)
    for ret, name, params in protos:
        fn = getattr(L, name)
        want = [_ctype_of(p) for p in params]
        got = fn.argtypes
        if want:
            assert got is not None and len(got) == len(want), (name, got, params)
            for g, w, p in zip(got, want, params):
                if w is ctypes.c_void_p:
                    assert g is ctypes.c_void_p or issubclass(g, ctypes._Pointer), (name, p, g)
                else:
                    assert g is w, (name, p, g, w)
        rt = ctypes.c_char_p if ret == "const char*" else _ctype_of(ret)
        assert fn.restype is rt, (name, ret, fn.restype)


def test_struct_layouts_match_the_header(tmp_path):
    """sizeof and offsetof of every field of ll_rope_desc and ll_kvcache, as
    gcc lays out the header, equal the ctypes structures of the binding."""
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "ll_api.h"', "int main(void) {"]
    for cname, cls in (("ll_rope_desc", swa.RopeDescC), ("ll_kvcache", swa.KVCacheC)):
        lines.append(f'  printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for field, _ in cls._fields_:
            lines.append(f'  printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    import subprocess
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        s, f, v = line.split()
        got[(s, f)] = int(v)
    for cname, cls in (("ll_rope_desc", swa.RopeDescC), ("ll_kvcache", swa.KVCacheC)):
        assert got[(cname, "sizeof")] == ctypes.sizeof(cls), cname
        for field, _ in cls._fields_:
            assert got[(cname, field)] == getattr(cls, field).offset, (cname, field)


def test_plain_c_program_links_and_calls_the_library(L, tmp_path):
    """The boundary is usable from C alone: a program built by gcc against
    ll_api.h and linked with libll_swa.so (no Python, no PyTorch) reads the ABI
    version, maps frames to slots and gets a host-side rejection with its
    message, none of which needs a GPU."""
    import subprocess
    lib_dir = os.path.dirname(swa.LIB_PATH)
    src = tmp_path / "use_abi.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "ll_api.h"
int main(void) {
  if (ll_abi_version() != LL_ABI_VERSION) return 1;
  int slot = -1;
  if (ll_slot_of_frame(100, 3, 9, &slot) != LL_OK || slot != 3 + (100 - 3) % 9) return 2;
  if (ll_slot_of_frame(2, 3, 9, &slot) != LL_OK || slot != 2) return 3;
  ll_rope_desc rope;
  memset(&rope, 0, sizeof(rope));
  rope.pairs_t = 10; rope.pairs_h = 10; rope.pairs_w = 10;   /* sums to 30, not D/2 = 32 */
  rope.theta0 = 10000.0; rope.grid_h = 2; rope.grid_w = 3;
  if (ll_rope_apply((void*)0, LL_BF16, 1, 1, 2, 64, 0, &rope, (void*)0) != LL_ERR_INVALID_ARG) return 4;
  const char* msg = ll_last_error();
  if (msg == NULL || strlen(msg) == 0) return 5;
  printf("%s\n", msg);
  return 0;
}
''')
    exe = tmp_path / "use_abi"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", lib_dir, "-l:" + os.path.basename(swa.LIB_PATH), "-Wl,-rpath," + lib_dir], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.strip()


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=400, deadline=None)
@given(frame=st.integers(0, 2**62), n_sink=st.integers(0, 64), n_local=st.integers(1, 64))
def test_slot_map_bit_exact_random(L, frame, n_sink, n_local):
    """The library's slot map (a host helper; the kernels compute the same
    map on the device) equals the oracle's for any frame index and window."""
    assert swa.slot_of_frame(frame, n_sink, n_local) == window.slot_of(frame, n_sink, n_local)
