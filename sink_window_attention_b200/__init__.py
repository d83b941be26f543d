"""Python binding of libll_swa.so (the B200 sink-window attention library).

Argument marshalling only: torch tensors supply device memory and the CUDA
stream; every step of the computation runs in the library's CUDA kernels.
The shared library must have been built (``python -m
sink_window_attention_b200.build`` or ``__graft_entry__.build()``); importing
this package without it raises, there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libll_swa.so")

LL_OK, LL_ERR_INVALID_ARG, LL_ERR_UNSUPPORTED, LL_ERR_CUDA, LL_ERR_TIMEOUT = range(5)
LL_F32, LL_BF16, LL_FP8_E4M3 = 0, 1, 2
MAX_HEADS = 64
ABI_VERSION = 2

EXPORTED = (
    "ll_abi_version", "ll_last_error", "ll_slot_of_frame", "ll_device_error", "ll_rope_apply",
    "ll_kvcache_append", "ll_sink_window_attention_workspace_bytes", "ll_sink_window_attention",
    "ll_kv_recache_workspace_bytes", "ll_kv_recache", "ll_sink_window_attention_noalloc",
    "ll_append_and_attend_workspace_bytes", "ll_append_and_attend", "ll_phase_coherence",
    "ll_selftest_bounded_waits", "ll_sink_window_attention_fp8_mma_workspace_bytes",
    "ll_sink_window_attention_fp8_mma",
)
NOALLOC_SCRATCH_BYTES = 48 * 1024 * 1024


class LLError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"ll status {status}: {message}")
        self.status = status


class RopeDescC(ctypes.Structure):
    _fields_ = [("pairs_t", ctypes.c_int), ("pairs_h", ctypes.c_int), ("pairs_w", ctypes.c_int),
                ("theta0", ctypes.c_double), ("sigma_t", ctypes.c_double),
                ("eps_h", ctypes.POINTER(ctypes.c_float)), ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
                ("t_offset", ctypes.c_longlong), ("t_scale", ctypes.c_double)]


class KVCacheC(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("v_scale", ctypes.c_void_p), ("dtype", ctypes.c_int), ("B", ctypes.c_int), ("H", ctypes.c_int),
                ("D", ctypes.c_int), ("tokens_per_frame", ctypes.c_int), ("n_sink", ctypes.c_int),
                ("n_local", ctypes.c_int)]


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with sink_window_attention_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, ll_, f, d, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_double, ctypes.c_size_t
        rp, cp = ctypes.POINTER(RopeDescC), ctypes.POINTER(KVCacheC)
        L.ll_abi_version.restype = i
        L.ll_last_error.restype = ctypes.c_char_p
        L.ll_slot_of_frame.argtypes = [ll_, i, i, ctypes.POINTER(i)]
        L.ll_device_error.argtypes = [ctypes.POINTER(i), vp]
        L.ll_rope_apply.argtypes = [vp, i, i, i, i, i, ll_, rp, vp]
        L.ll_kvcache_append.argtypes = [cp, vp, vp, i, ll_, i, rp, ctypes.POINTER(i), vp]
        L.ll_sink_window_attention_workspace_bytes.argtypes = [cp, i]
        L.ll_sink_window_attention_workspace_bytes.restype = sz
        L.ll_sink_window_attention.argtypes = [vp, i, cp, ll_, i, rp, f, vp, vp, vp, sz, vp]
        L.ll_sink_window_attention_noalloc.argtypes = [vp, i, cp, ll_, i, rp, f, vp, vp, vp]
        L.ll_sink_window_attention_fp8_mma_workspace_bytes.argtypes = [cp, i]
        L.ll_sink_window_attention_fp8_mma_workspace_bytes.restype = sz
        L.ll_sink_window_attention_fp8_mma.argtypes = [vp, i, cp, ll_, i, rp, f, vp, vp, vp, sz, vp]
        L.ll_kv_recache_workspace_bytes.argtypes = [cp, i, i]
        L.ll_kv_recache_workspace_bytes.restype = sz
        L.ll_kv_recache.argtypes = [cp, vp, i, vp, vp, vp, f, ctypes.POINTER(ll_), i, rp, vp, sz, vp]
        L.ll_append_and_attend_workspace_bytes.argtypes = [cp, i]
        L.ll_append_and_attend_workspace_bytes.restype = sz
        L.ll_append_and_attend.argtypes = [cp, vp, vp, vp, i, ll_, i, rp, f, vp, vp, vp, sz, vp]
        L.ll_phase_coherence.argtypes = [rp, i, ll_, i, vp, vp]
        L.ll_selftest_bounded_waits.argtypes = [vp]
        for name in EXPORTED[2:]:
            if not name.endswith("_workspace_bytes"):
                getattr(L, name).restype = i
        _lib = L
    return _lib


def last_error() -> str:
    return lib().ll_last_error().decode()


def _check(status: int) -> None:
    if status != LL_OK:
        raise LLError(status, last_error())


def _stream(stream=None) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return LL_F32
    if t == torch.bfloat16:
        return LL_BF16
    raise ValueError(f"unsupported tensor dtype {t}")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    """Device address of a contiguous CUDA tensor on the current device (the
    library's kernels dereference it there)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"tensors must be CUDA tensors, got one on {t.device}")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensors must be on the current CUDA device (cuda:{torch.cuda.current_device()}), "
                         f"got one on {t.device}")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _expect(t: Optional[torch.Tensor], shape, dtype: torch.dtype, what: str) -> None:
    """Shape and dtype of a buffer the kernels read or write in full."""
    if t is not None and (tuple(t.shape) != tuple(shape) or t.dtype != dtype):
        raise ValueError(f"{what} must be a {dtype} tensor of shape {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def _cache_c(cache: "KVCache") -> "KVCacheC":
    """The cache descriptor for a launch: its tensors checked like any other."""
    for t in (cache.k, cache.v, cache.k_scale, cache.v_scale):
        _ptr(t)
    return cache.to_c()


@dataclass
class Rope:
    """3D RoPE with the LoL per-head jittered temporal base (mirrors ll_rope_desc)."""
    pairs: Sequence[int]
    grid_h: int
    grid_w: int
    theta0: float = 10000.0
    sigma_t: float = 0.0
    eps: Optional[Sequence[float]] = None
    t_offset: int = 0
    t_scale: float = 1.0   # position interpolation of the temporal axis (1: plain RoPE)

    def to_c(self) -> RopeDescC:
        r = RopeDescC()
        r.pairs_t, r.pairs_h, r.pairs_w = (int(x) for x in self.pairs)
        r.theta0 = float(self.theta0)
        r.sigma_t = float(self.sigma_t)
        if self.eps is not None:
            arr = (ctypes.c_float * len(self.eps))(*[float(e) for e in self.eps])
            r._eps_keepalive = arr  # noqa: keep the host array alive with the struct
            r.eps_h = ctypes.cast(arr, ctypes.POINTER(ctypes.c_float))
        r.grid_h, r.grid_w, r.t_offset = int(self.grid_h), int(self.grid_w), int(self.t_offset)
        r.t_scale = float(self.t_scale)
        return r


def _rope_ref(rope: Optional[Rope]):
    return ctypes.byref(rope.to_c()) if rope is not None else None


class KVCache:
    """One layer's sink + ring KV cache in device memory (mirrors ll_kvcache)."""

    def __init__(self, B: int, H: int, D: int, tokens_per_frame: int, dtype: str = "bf16",
                 n_sink: int = 3, n_local: int = 9, device: str = "cuda"):
        self.B, self.H, self.D, self.N = B, H, D, tokens_per_frame
        self.n_sink, self.n_local = n_sink, n_local
        self.S = n_sink + n_local
        self.dtype = dtype
        shape = (B, self.S * tokens_per_frame, H, D)
        if dtype == "fp8":
            self.k = torch.zeros(shape, dtype=torch.uint8, device=device)
            self.v = torch.zeros(shape, dtype=torch.uint8, device=device)
            self.k_scale = torch.ones(shape[:3], dtype=torch.float32, device=device)
            self.v_scale = torch.ones(shape[:3], dtype=torch.float32, device=device)
            self.code = LL_FP8_E4M3
        else:
            tdt = {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]
            self.k = torch.zeros(shape, dtype=tdt, device=device)
            self.v = torch.zeros(shape, dtype=tdt, device=device)
            self.k_scale = self.v_scale = None
            self.code = _dtype_code(tdt)

    def to_c(self) -> KVCacheC:
        c = KVCacheC()
        c.k, c.v = self.k.data_ptr(), self.v.data_ptr()
        c.k_scale = self.k_scale.data_ptr() if self.k_scale is not None else None
        c.v_scale = self.v_scale.data_ptr() if self.v_scale is not None else None
        c.dtype, c.B, c.H, c.D = self.code, self.B, self.H, self.D
        c.tokens_per_frame, c.n_sink, c.n_local = self.N, self.n_sink, self.n_local
        return c


def abi_version() -> int:
    return lib().ll_abi_version()


def slot_of_frame(frame: int, n_sink: int = 3, n_local: int = 9) -> int:
    s = ctypes.c_int(-1)
    _check(lib().ll_slot_of_frame(frame, n_sink, n_local, ctypes.byref(s)))
    return s.value


def device_error(stream=None) -> int:
    """Synchronise and read (then clear) the library's device error word."""
    code = ctypes.c_int(0)
    st = lib().ll_device_error(ctypes.byref(code), _stream(stream))
    if st not in (LL_OK, LL_ERR_TIMEOUT):
        _check(st)
    return code.value


def rope_apply(x: torch.Tensor, first_frame: int, rope: Rope, stream=None) -> torch.Tensor:
    """In-place 3D RoPE of x [B, F*N, H, D]."""
    if x.dim() != 4:
        raise ValueError(f"x must be [B, F*N, H, D], got shape {tuple(x.shape)}")
    B, T, H, D = x.shape
    N = rope.grid_h * rope.grid_w
    if T % N != 0:
        raise ValueError(f"x holds {T} tokens, not a whole number of {N}-token frames")
    _check(lib().ll_rope_apply(_ptr(x), _dtype_code(x.dtype), B, T // N, H, D, first_frame, _rope_ref(rope),
                               _stream(stream)))
    return x


def _check_shape(cache: "KVCache", t: torch.Tensor, what: str) -> int:
    """[B, F*N, H, D] on the cache's batch, heads and head dim; returns F."""
    if t.dim() != 4 or t.shape[0] != cache.B or t.shape[2] != cache.H or t.shape[3] != cache.D or \
            t.shape[1] % cache.N != 0 or not t.is_contiguous():
        raise ValueError(f"{what} must be a contiguous [B={cache.B}, F*{cache.N}, {cache.H}, {cache.D}] tensor, "
                         f"got {tuple(t.shape)}")
    return t.shape[1] // cache.N


def kvcache_append(cache: KVCache, k: torch.Tensor, v: torch.Tensor, first_frame: int,
                   rope: Optional[Rope], stream=None):
    """Write frames first_frame.. of k, v [B, F*N, H, D] into their slots; returns the slots."""
    F = _check_shape(cache, k, "k")
    if _check_shape(cache, v, "v") != F:
        raise ValueError("k and v must cover the same frames")
    if v.dtype != k.dtype:
        raise ValueError("k and v must have one dtype")
    slots = (ctypes.c_int * F)()
    _check(lib().ll_kvcache_append(ctypes.byref(_cache_c(cache)), _ptr(k), _ptr(v), _dtype_code(k.dtype), first_frame,
                                   F, _rope_ref(rope), slots, _stream(stream)))
    return list(slots)


def attention_workspace_bytes(cache: KVCache, n_query_frames: int) -> int:
    return int(lib().ll_sink_window_attention_workspace_bytes(ctypes.byref(cache.to_c()), n_query_frames))


_workspaces = {}


def workspace_for(nbytes: int, device) -> torch.Tensor:
    """A device scratch buffer of at least nbytes, cached per device. Calls that
    share it must be ordered (one stream); pass your own workspace to run
    attention concurrently on several streams."""
    key = torch.device(device)
    t = _workspaces.get(key)
    if t is None or t.numel() < nbytes:
        t = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=key)
        _workspaces[key] = t
    return t


def sink_window_attention(q: torch.Tensor, cache: KVCache, first_frame: int, rope: Optional[Rope],
                          softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                          lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """Attention of query frames first_frame.. (q [B, F*N, H, D]) over the cache."""
    F = _check_shape(cache, q, "q")
    if out is None:
        out = torch.empty_like(q)
    _expect(out, q.shape, q.dtype, "out")
    _expect(lse, (cache.B, cache.H, q.shape[1]), torch.float32, "lse")
    if workspace is None:
        workspace = workspace_for(attention_workspace_bytes(cache, F), q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().ll_sink_window_attention(_ptr(q), _dtype_code(q.dtype), ctypes.byref(_cache_c(cache)), first_frame, F,
                                          _rope_ref(rope), float(softmax_scale), _ptr(out), _ptr(lse),
                                          _ptr(workspace), ws_bytes, _stream(stream)))
    return out


def attention_fp8_mma_workspace_bytes(cache: KVCache, n_query_frames: int) -> int:
    return int(lib().ll_sink_window_attention_fp8_mma_workspace_bytes(ctypes.byref(cache.to_c()), n_query_frames))


def sink_window_attention_fp8_mma(q: torch.Tensor, cache: KVCache, first_frame: int, rope: Optional[Rope],
                                  softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                                  lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                                  stream=None) -> torch.Tensor:
    """Attention over an E4M3 cache on the FP8 tensor cores (ll_sink_window_attention_fp8_mma)."""
    F = _check_shape(cache, q, "q")
    if out is None:
        out = torch.empty_like(q)
    _expect(out, q.shape, q.dtype, "out")
    _expect(lse, (cache.B, cache.H, q.shape[1]), torch.float32, "lse")
    if workspace is None:
        workspace = workspace_for(max(attention_fp8_mma_workspace_bytes(cache, F), 256), q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().ll_sink_window_attention_fp8_mma(_ptr(q), _dtype_code(q.dtype), ctypes.byref(_cache_c(cache)),
                                                  first_frame, F, _rope_ref(rope), float(softmax_scale), _ptr(out),
                                                  _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream)))
    return out


def append_and_attend_workspace_bytes(cache: KVCache, n_frames: int) -> int:
    return int(lib().ll_append_and_attend_workspace_bytes(ctypes.byref(cache.to_c()), n_frames))


def append_and_attend(cache: KVCache, k: torch.Tensor, v: torch.Tensor, q: torch.Tensor, first_frame: int,
                      rope: Optional[Rope], softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                      lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """ll_append_and_attend: append frames first_frame.. (k, v [B, F*N, H, D])
    and attend with their queries q (one kernel for BF16 / F32 caches; for an
    E4M3 cache the append with the bf16 staging copy, then attention)."""
    F = _check_shape(cache, q, "q")
    if _check_shape(cache, k, "k") != F or _check_shape(cache, v, "v") != F:
        raise ValueError("k, v and q must cover the same frames")
    if not (k.dtype == v.dtype == q.dtype):
        raise ValueError("k, v and q must have one dtype")
    if out is None:
        out = torch.empty_like(q)
    _expect(out, q.shape, q.dtype, "out")
    _expect(lse, (cache.B, cache.H, q.shape[1]), torch.float32, "lse")
    if workspace is None:
        workspace = workspace_for(append_and_attend_workspace_bytes(cache, F), q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().ll_append_and_attend(ctypes.byref(_cache_c(cache)), _ptr(k), _ptr(v), _ptr(q), _dtype_code(q.dtype),
                                      first_frame, F, _rope_ref(rope), float(softmax_scale), _ptr(out), _ptr(lse),
                                      _ptr(workspace), ws_bytes, _stream(stream)))
    return out


def sink_window_attention_noalloc(q: torch.Tensor, cache: KVCache, first_frame: int, rope: Optional[Rope],
                                  softmax_scale: float = 0.0, out: Optional[torch.Tensor] = None,
                                  lse: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """ll_sink_window_attention_noalloc: the same attention with the library's
    static scratch array instead of a caller workspace (allocates nothing)."""
    F = _check_shape(cache, q, "q")
    if out is None:
        out = torch.empty_like(q)
    _expect(out, q.shape, q.dtype, "out")
    _expect(lse, (cache.B, cache.H, q.shape[1]), torch.float32, "lse")
    _check(lib().ll_sink_window_attention_noalloc(_ptr(q), _dtype_code(q.dtype), ctypes.byref(_cache_c(cache)),
                                                  first_frame, F, _rope_ref(rope), float(softmax_scale), _ptr(out),
                                                  _ptr(lse), _stream(stream)))
    return out


def recache_workspace_bytes(cache: KVCache, d_model: int, n_slots: int) -> int:
    return int(lib().ll_kv_recache_workspace_bytes(ctypes.byref(cache.to_c()), d_model, n_slots))


def kv_recache(cache: KVCache, x: torch.Tensor, wk: torch.Tensor, wv: torch.Tensor, gamma: torch.Tensor,
               rms_eps: float, slot_frames: Sequence[int], rope: Rope,
               workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Recompute K/V of slots 0..len(slot_frames)-1 from hidden states x [B, n*N, d_model]."""
    n = len(slot_frames)
    if x.dim() != 3:
        raise ValueError(f"x must be [B, n_slots*N, d_model], got shape {tuple(x.shape)}")
    dm, dout = x.shape[-1], cache.H * cache.D
    _expect(x, (cache.B, n * cache.N, dm), torch.bfloat16, "x")
    _expect(wk, (dm, dout), torch.bfloat16, "wk")
    _expect(wv, (dm, dout), torch.bfloat16, "wv")
    _expect(gamma, (dout,), torch.float32, "gamma")
    frames = (ctypes.c_longlong * n)(*[int(f) for f in slot_frames])
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().ll_kv_recache(ctypes.byref(_cache_c(cache)), _ptr(x), dm, _ptr(wk), _ptr(wv), _ptr(gamma),
                               float(rms_eps), frames, n, _rope_ref(rope), _ptr(workspace), ws_bytes,
                               _stream(stream)))


def phase_coherence(rope: Rope, H: int, delta0: int, n_delta: int, out: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """C_h(D) of the temporal RoPE band for D = delta0 .. delta0 + n_delta - 1
    (ll_phase_coherence): float32 [H, n_delta, 2] (real, imaginary) on the
    current CUDA device."""
    if out is None:
        out = torch.empty((H, n_delta, 2), dtype=torch.float32, device="cuda")
    _expect(out, (H, n_delta, 2), torch.float32, "out")
    _check(lib().ll_phase_coherence(ctypes.byref(rope.to_c()), H, int(delta0), int(n_delta), _ptr(out),
                                    _stream(stream)))
    return out


def selftest_bounded_waits(stream=None) -> int:
    """Launch the bounded-wait self-test (ll_selftest_bounded_waits) and return
    the device error code it leaves (read and cleared by ll_device_error)."""
    _check(lib().ll_selftest_bounded_waits(_stream(stream)))
    return device_error(stream)
