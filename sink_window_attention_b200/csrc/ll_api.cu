// ll_api.cu — host side of libll_swa.so: argument validation, TMA tensor-map
// encoding and kernel launches behind the C ABI declared in include/ll_api.h.
// The library allocates no device memory and keeps no state between calls.
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <string>

#include "../../include/ll_api.h"
#include "ll_attention.cuh"
#include "ll_common.cuh"
#include "ll_recache.cuh"
#include "ll_rope_append.cuh"

namespace {

thread_local std::string g_last_error;

ll_status fail(ll_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

ll_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(LL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return LL_OK;
}

int element_size(ll_dtype t) {
  switch (t) {
    case LL_F32: return 4;
    case LL_BF16: return 2;
    case LL_FP8_E4M3: return 1;
  }
  return 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Validates a rope descriptor for heads H and head dim D and converts it.
ll_status make_rope(const ll_rope_desc* r, int H, int D, long long t_first, ll::RopeParams* out) {
  std::memset(out, 0, sizeof(*out));
  if (r == nullptr) return LL_OK;  // disabled
  if (r->pairs_t < 0 || r->pairs_h < 0 || r->pairs_w < 0 || r->pairs_t + r->pairs_h + r->pairs_w != D / 2)
    return fail(LL_ERR_INVALID_ARG, "rope pairs (%d, %d, %d) must be >= 0 and sum to D/2 = %d", r->pairs_t,
                r->pairs_h, r->pairs_w, D / 2);
  if (!(r->theta0 > 1.0) || !std::isfinite(r->theta0))
    return fail(LL_ERR_INVALID_ARG, "rope theta0 must be a finite value > 1");
  if (!(r->sigma_t >= 0.0 && r->sigma_t < 1.0))
    return fail(LL_ERR_INVALID_ARG, "rope sigma_t must lie in [0, 1) so every base stays positive");
  if (r->grid_h < 1 || r->grid_w < 1) return fail(LL_ERR_INVALID_ARG, "rope grid must be at least 1x1");
  if (static_cast<long long>(r->grid_h) * r->grid_w > INT_MAX)
    return fail(LL_ERR_INVALID_ARG, "rope grid %dx%d has more than 2^31 - 1 tokens", r->grid_h, r->grid_w);
  if (H > ll::kMaxHeads) return fail(LL_ERR_INVALID_ARG, "H = %d exceeds %d", H, ll::kMaxHeads);
  if (r->t_offset < 0) return fail(LL_ERR_INVALID_ARG, "rope t_offset must be >= 0");
  if (!(r->t_scale >= 0.0 && r->t_scale <= 1.0))
    return fail(LL_ERR_INVALID_ARG, "rope t_scale must lie in [0, 1] (0 and 1: no interpolation)");
  out->enabled = 1;
  out->pt = r->pairs_t;
  out->ph = r->pairs_h;
  out->pw = r->pairs_w;
  out->grid_w = r->grid_w;
  out->t_first = r->t_offset + t_first;
  out->t_scale = r->t_scale > 0.0 ? static_cast<float>(r->t_scale) : 1.0f;
  out->theta0 = r->theta0;
  out->sigma = r->eps_h ? r->sigma_t : 0.0;
  for (int h = 0; h < H; ++h) {
    const float e = r->eps_h ? r->eps_h[h] : 0.f;
    if (!(e >= -1.f && e <= 1.f)) return fail(LL_ERR_INVALID_ARG, "eps_h[%d] = %g is outside [-1, 1]", h, e);
    out->eps[h] = e;
  }
  return LL_OK;
}

ll_status check_cache(const ll_kvcache* c) {
  if (c == nullptr) return fail(LL_ERR_INVALID_ARG, "cache is NULL");
  if (c->k == nullptr || c->v == nullptr) return fail(LL_ERR_INVALID_ARG, "cache k/v pointer is NULL");
  if (!aligned16(c->k) || !aligned16(c->v)) return fail(LL_ERR_INVALID_ARG, "cache k/v must be 16-byte aligned");
  if (element_size(c->dtype) == 0) return fail(LL_ERR_INVALID_ARG, "unknown cache dtype %d", (int)c->dtype);
  if (c->dtype == LL_FP8_E4M3 && (c->k_scale == nullptr || c->v_scale == nullptr))
    return fail(LL_ERR_INVALID_ARG, "an FP8 cache needs k_scale and v_scale");
  if (c->dtype == LL_FP8_E4M3 && (!aligned4(c->k_scale) || !aligned4(c->v_scale)))
    return fail(LL_ERR_INVALID_ARG, "k_scale and v_scale must be 4-byte aligned");
  if (c->B < 1 || c->H < 1 || c->D < 2 || c->tokens_per_frame < 1)
    return fail(LL_ERR_INVALID_ARG, "cache sizes must be positive (B=%d H=%d D=%d N=%d)", c->B, c->H, c->D,
                c->tokens_per_frame);
  if (c->D % 16 != 0) return fail(LL_ERR_INVALID_ARG, "D = %d must be a multiple of 16", c->D);
  if (c->dtype == LL_FP8_E4M3) {  // a row's max|x| is reduced over its D / 8 lanes: a power of two up to 32
    const int lanes = c->D / 8;
    if ((lanes & (lanes - 1)) != 0 || lanes > 32)
      return fail(LL_ERR_UNSUPPORTED, "an FP8 cache needs D = 16 * 2^k <= 256 (got D = %d)", c->D);
  }
  if (c->H > ll::kMaxHeads) return fail(LL_ERR_INVALID_ARG, "H = %d exceeds %d", c->H, ll::kMaxHeads);
  if (c->n_sink < 0 || c->n_local < 1) return fail(LL_ERR_INVALID_ARG, "need n_sink >= 0 and n_local >= 1");
  if ((static_cast<long long>(c->n_sink) + c->n_local) * c->tokens_per_frame > INT_MAX)
    return fail(LL_ERR_INVALID_ARG, "(n_sink + n_local) x tokens_per_frame = %lld cache rows exceed 2^31 - 1",
                (static_cast<long long>(c->n_sink) + c->n_local) * c->tokens_per_frame);
  return LL_OK;
}

ll_status check_grid(const ll_rope_desc* r, int N) {
  if (r && static_cast<long long>(r->grid_h) * r->grid_w != N)
    return fail(LL_ERR_INVALID_ARG, "rope grid %dx%d does not match %d tokens per frame", r->grid_h, r->grid_w, N);
  return LL_OK;
}

constexpr int kDeviceSlots = 64;  // device ordinals with cached per-device state

// SM count of the current device (looked up once per device).
int num_sms() {
  static std::atomic<int> cached[kDeviceSlots];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) dev = 0;
  if (dev < kDeviceSlots) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
  if (dev < kDeviceSlots) cached[dev].store(sms, std::memory_order_relaxed);
  return sms;
}

// Runs `setup` (kernel attributes: they are per device) the first time it is
// reached on the current device; later calls on that device skip it. Only a
// successful setup is remembered.
template <class F>
ll_status once_per_device(std::atomic<unsigned long long>& done, F&& setup) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return check_launch("cudaGetDevice");
  if (dev < 0 || dev >= kDeviceSlots) return fail(LL_ERR_UNSUPPORTED, "device ordinal %d is out of range", dev);
  const unsigned long long bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return LL_OK;
  const ll_status st = setup();
  if (st == LL_OK) done.fetch_or(bit, std::memory_order_acq_rel);
  return st;
}

// ---------------------------------------------------------------------------
// TMA tensor maps (driver entry point fetched through the runtime, so the
// library does not link libcuda directly).
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 4D map over a [B][rows][H][D] tensor whose batch stride is batch_rows rows:
// dims (D, H, rows, B), box (128 bytes of D, 1 head, box_rows, 1), 128-byte
// swizzle, rows >= `rows` read as zeros.
ll_status encode_rows_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int es, int D, int H,
                          long long rows, long long batch_rows, int B, int box_rows,
                          CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(LL_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * es, (cuuint64_t)H * D * es, (cuuint64_t)batch_rows * H * D * es};
  const cuuint32_t box[4] = {(cuuint32_t)(128 / es), 1u, (cuuint32_t)box_rows, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  const CUresult r = fn(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LL_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return LL_OK;
}

// 3D map over an E4M3 cache's fp32 scales [B][batch_rows][H]: dims (H, rows,
// B), box (4 heads, box_rows, 1), 16 bytes wide, so its x coordinate (the
// first head) is always a multiple of 4; heads >= H and rows >= `rows` read as
// 0. The row stride H * 4 bytes must be a multiple of 16 (H % 4 == 0).
ll_status encode_scale_map(CUtensorMap* map, const void* base, int H, long long rows, long long batch_rows, int B,
                           int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(LL_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[3] = {(cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)H * 4, (cuuint64_t)batch_rows * H * 4};
  const cuuint32_t box[3] = {4u, (cuuint32_t)box_rows, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LL_ERR_CUDA, "cuTensorMapEncodeTiled (scales) failed (%d)", (int)r);
  return LL_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of one attention call: per-unit arrival counters, then
// (#SMs + units) partial slots of SLOT_FLOATS floats.
template <class TR>
size_t attention_workspace(int units) {
  return align256(static_cast<size_t>(units) * sizeof(int)) +
         static_cast<size_t>(num_sms() + units) * TR::SLOT_FLOATS * sizeof(float);
}

template <class TR>
ll_status launch_attention(ll::AttnParams p, const ll_kvcache* c, long long S, void* workspace, size_t ws_bytes,
                           cudaStream_t stream, bool cooperative = false) {
  p.q_tiles = (p.Tq + TR::BM - 1) / TR::BM;
  p.nkv = (p.Nk + TR::BN - 1) / TR::BN;
  p.units = p.q_tiles * c->H * c->B;
  p.total = static_cast<long long>(p.units) * p.nkv;
  p.grid = static_cast<int>(p.total < num_sms() ? p.total : num_sms());
  const size_t need = attention_workspace<TR>(p.units);
  if (workspace == nullptr || ws_bytes < need)
    return fail(LL_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu required", ws_bytes, need);
  p.counters = static_cast<int*>(workspace);
  p.partials = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(p.units * sizeof(int)));
  CUtensorMap tmQ, tmK, tmV, tmKS, tmVS;
  // Q (and O) are bf16 in the E4M3 variant; its K and V are 1-byte codes
  const CUtensorMapDataType dq =
      TR::FP8 || TR::ES == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const CUtensorMapDataType dkv = TR::FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : dq;
  const int qes = TR::FP8 ? 2 : TR::ES;
  const long long batch_rows = S * c->tokens_per_frame;
  ll_status st = encode_rows_map(&tmQ, p.q, dq, qes, TR::D, c->H, p.Tq, p.Tq, c->B, TR::BM);
  if (st != LL_OK) return st;
  st = encode_rows_map(&tmK, c->k, dkv, TR::ES, TR::D, c->H, p.Nk, batch_rows, c->B, TR::BN);
  if (st != LL_OK) return st;
  st = encode_rows_map(&tmV, c->v, dkv, TR::ES, TR::D, c->H, p.Nk, batch_rows, c->B, TR::BN,
                       TR::ES <= 2 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B);
  if (st != LL_OK) return st;
  tmKS = tmK;  // read only by the E4M3 variant
  tmVS = tmK;
  if constexpr (TR::FP8) {
    if ((st = encode_scale_map(&tmKS, c->k_scale, c->H, p.Nk, batch_rows, c->B, TR::BN)) != LL_OK) return st;
    if ((st = encode_scale_map(&tmVS, c->v_scale, c->H, p.Nk, batch_rows, c->B, TR::BN)) != LL_OK) return st;
  }
  auto kern = ll::sink_window_attention_kernel<TR>;
  static std::atomic<unsigned long long> attr_set{0};
  st = once_per_device(attr_set, [&]() -> ll_status {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TR::SMEM_BYTES) != cudaSuccess)
      return check_launch("cudaFuncSetAttribute(attention)");
    return LL_OK;
  });
  if (st != LL_OK) return st;
  if (cudaMemsetAsync(p.counters, 0, p.units * sizeof(int), stream) != cudaSuccess)
    return check_launch("cudaMemsetAsync(attention counters)");
  if (!cooperative) {
    kern<<<p.grid, TR::THREADS, TR::SMEM_BYTES, stream>>>(tmQ, tmK, tmV, tmKS, tmVS, p);
    return check_launch("sink_window_attention_kernel");
  }
  // fused append: the CTAs meet at a grid barrier, so they must all be
  // resident at once (the launch fails instead of running otherwise)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid, 1, 1);
  cfg.blockDim = dim3(TR::THREADS, 1, 1);
  cfg.dynamicSmemBytes = TR::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tmQ, tmK, tmV, tmKS, tmVS, p) != cudaSuccess)
    return check_launch("sink_window_attention_kernel (cooperative, fused append)");
  return check_launch("sink_window_attention_kernel (cooperative, fused append)");
}

// Launch generation of the fused append's grid barrier word (never 0, so a
// zero-filled word never matches).
unsigned int next_generation() {
  static std::atomic<unsigned int> gen{0};
  unsigned int g = ++gen;
  if (g == 0) g = ++gen;
  return g;
}

// Bytes of the bf16 copy of an FP8 cache that attention over an FP8 cache
// dequantises into (placed after the attention scratch in the workspace).
size_t fp8_staging_half(const ll_kvcache* c) {  // one of K / V, bf16, 256-byte aligned
  const size_t S = static_cast<size_t>(c->n_sink + c->n_local);
  return align256(static_cast<size_t>(c->B) * S * c->tokens_per_frame * c->H * c->D * sizeof(__nv_bfloat16));
}
size_t fp8_staging_bytes(const ll_kvcache* c) { return c->dtype == LL_FP8_E4M3 ? 2 * fp8_staging_half(c) : 0; }

size_t attention_scratch_bytes(const ll_kvcache* cache, int n_query_frames) {
  const int units = ((n_query_frames * cache->tokens_per_frame + 127) / 128) * cache->H * cache->B;
  if (cache->D == 128) return align256(attention_workspace<ll::AttnTraits<128, __nv_bfloat16>>(units));
  if (cache->dtype == LL_F32) return align256(attention_workspace<ll::AttnTraits<64, float>>(units));
  return align256(attention_workspace<ll::AttnTraits<64, __nv_bfloat16>>(units));
}

ll_status launch_bf16_attention_on(const ll_kvcache* staged, const void* q, long long first_frame, int n_query_frames,
                                   const ll_rope_desc* rope, float softmax_scale, void* out, float* lse,
                                   void* workspace, size_t workspace_bytes, cudaStream_t s);

// The fused append + attention over an E4M3 cache: one kernel appends the new
// frames (codes and scales into their slots, their dequantised values into
// the bf16 staging rows) and dequantises every other occupied row into the
// staging copy; the bf16 attention kernel then reads the staging copy. The
// results equal those of ll_kvcache_append followed by
// ll_sink_window_attention.
ll_status append_stage_and_attend(const ll_kvcache* cache, const ll::AppendParams& ap, const void* q,
                                  long long first_frame, int n_frames, const ll_rope_desc* rope, float softmax_scale,
                                  void* out, float* lse, void* workspace, size_t workspace_bytes, cudaStream_t s) {
  const long long S = cache->n_sink + cache->n_local;
  const long long last = first_frame + n_frames - 1;
  const long long valid_slots = last + 1 < S ? last + 1 : S;
  const size_t half = fp8_staging_half(cache);
  char* stage = static_cast<char*>(workspace) + attention_scratch_bytes(cache, n_frames);
  ll::AppendStageParams q8{};
  q8.ap = ap;
  q8.ap.stage_k = reinterpret_cast<__nv_bfloat16*>(stage);
  q8.ap.stage_v = reinterpret_cast<__nv_bfloat16*>(stage + half);
  ll::DequantParams& dp = q8.dq;
  dp.src[0] = static_cast<const uint8_t*>(cache->k);
  dp.src[1] = static_cast<const uint8_t*>(cache->v);
  dp.scale[0] = cache->k_scale;
  dp.scale[1] = cache->v_scale;
  dp.dst[0] = q8.ap.stage_k;
  dp.dst[1] = q8.ap.stage_v;
  dp.B = cache->B;
  dp.rows = static_cast<int>(valid_slots * cache->tokens_per_frame);
  dp.batch_rows = static_cast<int>(S * cache->tokens_per_frame);
  dp.H = cache->H;
  dp.D = cache->D;
  dp.cshift = cache->D == 128 ? 3 : 2;
  // the appended frames' slots as runs of consecutive slots (a ring wrap
  // splits them; a sink and a local frame can join): their (token, head) rows
  // are written by the append blocks and skipped by the staging blocks
  {
    bool is_new[ll::kMaxSlots] = {};
    for (int i = 0; i < n_frames; ++i) {
      int slot = 0;
      ll_slot_of_frame(first_frame + i, cache->n_sink, cache->n_local, &slot);
      is_new[slot] = true;
    }
    const int per_slot = cache->tokens_per_frame * cache->H;
    for (int sl = 0; sl < S;) {
      if (!is_new[sl]) { ++sl; continue; }
      int e = sl;
      while (e < S && is_new[e]) ++e;
      if (dp.nskip == 3) return fail(LL_ERR_UNSUPPORTED, "the appended frames' slots form more than 3 runs");
      dp.skip_lo[dp.nskip] = sl * per_slot;
      dp.skip_hi[dp.nskip] = e * per_slot;
      ++dp.nskip;
      sl = e;
    }
  }
  const long long threads = ll::append_items(ap);
  const long long want_a = (threads + 255) / 256;
  q8.append_blocks = static_cast<int>(want_a < 8LL * num_sms() ? want_a : 8LL * num_sms());
  const long long chunks = static_cast<long long>(dp.B) * dp.rows * dp.H * (dp.D / 16);
  const long long want_d = (chunks + 255) / 256;
  q8.dequant_blocks = static_cast<int>(want_d < 4LL * num_sms() ? want_d : 4LL * num_sms());
  const size_t smem = ll::append_smem_bytes(n_frames, cache->H, cache->D, ap.rp.pt);
  if (smem > 48 * 1024)
    return fail(LL_ERR_UNSUPPORTED, "frequency tables of %zu bytes exceed 48 KiB (n_frames x H x pairs_t too large)",
                smem);
  ll::append_stage_e4m3_kernel<<<q8.append_blocks + 2 * q8.dequant_blocks, 256, smem, s>>>(q8);
  ll_status st = check_launch("append_stage_e4m3_kernel");
  if (st != LL_OK) return st;
  ll_kvcache staged = *cache;
  staged.k = q8.ap.stage_k;
  staged.v = q8.ap.stage_v;
  staged.k_scale = staged.v_scale = nullptr;
  staged.dtype = LL_BF16;
  return launch_bf16_attention_on(&staged, q, first_frame, n_frames, rope, softmax_scale, out, lse, workspace,
                                  workspace_bytes, s);
}

}  // namespace

extern "C" {

int ll_abi_version(void) { return LL_ABI_VERSION; }

const char* ll_last_error(void) { return g_last_error.c_str(); }

ll_status ll_slot_of_frame(long long frame, int n_sink, int n_local, int* slot) {
  if (slot == nullptr) return fail(LL_ERR_INVALID_ARG, "slot is NULL");
  if (frame < 0 || n_sink < 0 || n_local < 1)
    return fail(LL_ERR_INVALID_ARG, "need frame >= 0, n_sink >= 0, n_local >= 1");
  *slot = frame < n_sink ? static_cast<int>(frame) : n_sink + static_cast<int>((frame - n_sink) % n_local);
  return LL_OK;
}

ll_status ll_device_error(int* code, void* stream) {
  if (code == nullptr) return fail(LL_ERR_INVALID_ARG, "code is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return check_launch("cudaStreamSynchronize");
  unsigned int w = 0;
  if (cudaMemcpyFromSymbol(&w, ll::g_error_word, sizeof(w)) != cudaSuccess) return check_launch("read error word");
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(ll::g_error_word, &zero, sizeof(zero)) != cudaSuccess)
    return check_launch("clear error word");
  *code = static_cast<int>(w);
  if (w != 0) return fail(LL_ERR_TIMEOUT, "a device-side wait gave up (error word 0x%x)", w);
  return LL_OK;
}

ll_status ll_rope_apply(void* x, ll_dtype dtype, int B, int n_frames, int H, int D, long long first_frame,
                        const ll_rope_desc* rope, void* stream) {
  g_last_error.clear();
  if (x == nullptr || rope == nullptr) return fail(LL_ERR_INVALID_ARG, "x and rope must be non-NULL");
  if (!aligned16(x)) return fail(LL_ERR_INVALID_ARG, "x must be 16-byte aligned");
  if (B < 1 || n_frames < 1 || H < 1 || D < 2) return fail(LL_ERR_INVALID_ARG, "sizes must be positive");
  if (D % 8 != 0) return fail(LL_ERR_INVALID_ARG, "D = %d must be a multiple of 8", D);
  if (first_frame < 0) return fail(LL_ERR_INVALID_ARG, "first_frame must be >= 0");
  if (dtype != LL_F32 && dtype != LL_BF16) return fail(LL_ERR_INVALID_ARG, "rope_apply takes F32 or BF16");
  ll::RopeApplyParams p{};
  ll_status st = make_rope(rope, H, D, first_frame, &p.rp);
  if (st != LL_OK) return st;
  p.x = x;
  p.B = B;
  p.F = n_frames;
  p.N = rope->grid_h * rope->grid_w;
  p.H = H;
  p.D = D;
  const long long chunks = static_cast<long long>(B) * n_frames * p.N * H * (D / 8);
  if (chunks >= (1LL << 31)) return fail(LL_ERR_UNSUPPORTED, "tensor too large for one call (%lld chunks)", chunks);
  if (H * (D / 8) > 1024) return fail(LL_ERR_UNSUPPORTED, "H * D / 8 = %d exceeds 1024", H * (D / 8));
  const long long rows = static_cast<long long>(B) * n_frames * p.N;
  const int grid = static_cast<int>((rows + ll::kRopeTokens - 1) / ll::kRopeTokens);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == LL_BF16)
    ll::rope_apply_kernel<__nv_bfloat16><<<grid, H * (D / 8), 0, s>>>(p);
  else
    ll::rope_apply_kernel<float><<<grid, H * (D / 8), 0, s>>>(p);
  return check_launch("rope_apply_kernel");
}

ll_status ll_kvcache_append(const ll_kvcache* cache, const void* k, const void* v, ll_dtype in_dtype,
                            long long first_frame, int n_frames, const ll_rope_desc* rope, int* slots_out,
                            void* stream) {
  g_last_error.clear();
  ll_status st = check_cache(cache);
  if (st != LL_OK) return st;
  if (k == nullptr || v == nullptr) return fail(LL_ERR_INVALID_ARG, "k and v must be non-NULL");
  if (!aligned16(k) || !aligned16(v)) return fail(LL_ERR_INVALID_ARG, "k and v must be 16-byte aligned");
  if (first_frame < 0) return fail(LL_ERR_INVALID_ARG, "first_frame must be >= 0");
  if (n_frames < 1 || n_frames > cache->n_local)
    return fail(LL_ERR_INVALID_ARG, "n_frames = %d must lie in [1, n_local = %d]", n_frames, cache->n_local);
  if (in_dtype != LL_F32 && in_dtype != LL_BF16) return fail(LL_ERR_INVALID_ARG, "k/v must be F32 or BF16");
  if (cache->dtype == LL_FP8_E4M3 ? in_dtype != LL_BF16 : in_dtype != cache->dtype)
    return fail(LL_ERR_INVALID_ARG, "input dtype does not match the cache dtype");
  if ((st = check_grid(rope, cache->tokens_per_frame)) != LL_OK) return st;
  ll::AppendParams p{};
  if ((st = make_rope(rope, cache->H, cache->D, first_frame, &p.rp)) != LL_OK) return st;
  p.k_in = k;
  p.v_in = v;
  p.k_cache = cache->k;
  p.v_cache = cache->v;
  p.k_scale = cache->k_scale;
  p.v_scale = cache->v_scale;
  p.B = cache->B;
  p.F = n_frames;
  p.N = cache->tokens_per_frame;
  p.H = cache->H;
  p.D = cache->D;
  p.n_sink = cache->n_sink;
  p.n_local = cache->n_local;
  p.first_frame = first_frame;
  if (slots_out)
    for (int i = 0; i < n_frames; ++i) ll_slot_of_frame(first_frame + i, cache->n_sink, cache->n_local, &slots_out[i]);
  // one thread per (head, 8-element chunk) of a token row, kAppendTokens rows per block
  const long long chunks = static_cast<long long>(p.B) * n_frames * p.N * p.H * (p.D / 8);
  if (chunks >= (1LL << 31)) return fail(LL_ERR_UNSUPPORTED, "tensor too large for one call (%lld chunks)", chunks);
  if (p.H * (p.D / 8) > 1024) return fail(LL_ERR_UNSUPPORTED, "H * D / 8 = %d exceeds 1024", p.H * (p.D / 8));
  const long long rows = static_cast<long long>(p.B) * n_frames * p.N;
  const int grid = static_cast<int>((rows + ll::kAppendTokens - 1) / ll::kAppendTokens);
  const int threads = (p.H * (p.D / 8) + 31) / 32 * 32;  // whole warps (the E4M3 row max shuffles)
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cache->dtype == LL_BF16)
    ll::append_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, threads, 0, s>>>(p);
  else if (cache->dtype == LL_F32)
    ll::append_kernel<float, float><<<grid, threads, 0, s>>>(p);
  else
    ll::append_kernel<__nv_bfloat16, uint8_t><<<grid, threads, 0, s>>>(p);
  return check_launch("append_kernel");
}

size_t ll_sink_window_attention_workspace_bytes(const ll_kvcache* cache, int n_query_frames) {
  if (cache == nullptr || n_query_frames < 1 || cache->tokens_per_frame < 1 || cache->H < 1 || cache->B < 1)
    return 0;
  return attention_scratch_bytes(cache, n_query_frames) + fp8_staging_bytes(cache);
}

ll_status ll_sink_window_attention(const void* q, ll_dtype q_dtype, const ll_kvcache* cache, long long first_frame,
                                   int n_query_frames, const ll_rope_desc* rope, float softmax_scale, void* out,
                                   float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  g_last_error.clear();
  ll_status st = check_cache(cache);
  if (st != LL_OK) return st;
  if (q == nullptr || out == nullptr) return fail(LL_ERR_INVALID_ARG, "q and out must be non-NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(LL_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
  if (!aligned4(lse)) return fail(LL_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  if (first_frame < 0) return fail(LL_ERR_INVALID_ARG, "first_frame must be >= 0");
  if (n_query_frames < 1 || n_query_frames > cache->n_local)
    return fail(LL_ERR_INVALID_ARG, "n_query_frames = %d must lie in [1, n_local = %d]", n_query_frames,
                cache->n_local);
  if (!(softmax_scale >= 0.f) || !std::isfinite(softmax_scale))
    return fail(LL_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  const size_t need = ll_sink_window_attention_workspace_bytes(cache, n_query_frames);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(LL_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu required", workspace_bytes, need);
  if (!aligned16(workspace)) return fail(LL_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if ((st = check_grid(rope, cache->tokens_per_frame)) != LL_OK) return st;
  const bool f32 = cache->dtype == LL_F32;
  if (f32 ? q_dtype != LL_F32 : q_dtype != LL_BF16)
    return fail(LL_ERR_INVALID_ARG, "q dtype must be F32 for an F32 cache and BF16 otherwise");
  const long long S = cache->n_sink + cache->n_local;
  const long long last = first_frame + n_query_frames - 1;
  const long long valid_slots = last + 1 < S ? last + 1 : S;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ll::AttnParams p{};
  if ((st = make_rope(rope, cache->H, cache->D, first_frame, &p.rp)) != LL_OK) return st;  // before any launch
  ll_kvcache staged;
  if (cache->dtype == LL_FP8_E4M3) {
    // E4M3 cache: the occupied rows are dequantised into bf16 staging inside
    // the workspace, then the bf16 kernel runs on the staged copy
    if (cache->D != 128 && cache->D != 64)
      return fail(LL_ERR_UNSUPPORTED, "attention supports D = 64 or 128; got D = %d", cache->D);
    const size_t half = fp8_staging_half(cache);
    char* stage = static_cast<char*>(workspace) + attention_scratch_bytes(cache, n_query_frames);
    ll::DequantParams dp{};
    dp.src[0] = static_cast<const uint8_t*>(cache->k);
    dp.src[1] = static_cast<const uint8_t*>(cache->v);
    dp.scale[0] = cache->k_scale;
    dp.scale[1] = cache->v_scale;
    dp.dst[0] = reinterpret_cast<__nv_bfloat16*>(stage);
    dp.dst[1] = reinterpret_cast<__nv_bfloat16*>(stage + half);
    dp.B = cache->B;
    dp.rows = static_cast<int>(valid_slots * cache->tokens_per_frame);
    dp.batch_rows = static_cast<int>(S * cache->tokens_per_frame);
    dp.H = cache->H;
    dp.D = cache->D;
    dp.cshift = cache->D == 128 ? 3 : 2;
    const long long chunks = static_cast<long long>(dp.B) * dp.rows * dp.H * (dp.D / 16);
    const long long want = (chunks + 255) / 256;
    const dim3 grid(static_cast<unsigned>(want < 8LL * num_sms() ? want : 8LL * num_sms()), 2);
    ll::dequant_e4m3_kernel<<<grid, 256, 0, s>>>(dp);
    if ((st = check_launch("dequant_e4m3_kernel")) != LL_OK) return st;
    staged = *cache;
    staged.k = dp.dst[0];
    staged.v = dp.dst[1];
    staged.k_scale = staged.v_scale = nullptr;
    staged.dtype = LL_BF16;
    cache = &staged;
  }
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.B = cache->B;
  p.H = cache->H;
  p.Tq = n_query_frames * cache->tokens_per_frame;
  p.Nk = static_cast<int>(valid_slots * cache->tokens_per_frame);
  p.softmax_scale = softmax_scale;
  p.N = cache->tokens_per_frame;
  if (!f32 && cache->D == 128)
    return launch_attention<ll::AttnTraits<128, __nv_bfloat16>>(p, cache, S, workspace, workspace_bytes, s);
  if (!f32 && cache->D == 64)
    return launch_attention<ll::AttnTraits<64, __nv_bfloat16>>(p, cache, S, workspace, workspace_bytes, s);
  if (f32 && cache->D == 64)
    return launch_attention<ll::AttnTraits<64, float>>(p, cache, S, workspace, workspace_bytes, s);
  return fail(LL_ERR_UNSUPPORTED, "attention supports D = 64 or 128 (bf16) and D = 64 (f32); got D = %d", cache->D);
}

size_t ll_sink_window_attention_fp8_mma_workspace_bytes(const ll_kvcache* cache, int n_query_frames) {
  if (cache == nullptr || n_query_frames < 1 || cache->tokens_per_frame < 1 || cache->H < 1 || cache->B < 1 ||
      cache->dtype != LL_FP8_E4M3 || cache->D != 128)
    return 0;
  const int units = ((n_query_frames * cache->tokens_per_frame + 127) / 128) * cache->H * cache->B;
  return align256(attention_workspace<ll::AttnTraits<128, ll::E4M3Kv>>(units)) +
         align256(static_cast<size_t>(cache->B) * cache->H * sizeof(float));  // + the V-scale maxima
}

ll_status ll_sink_window_attention_fp8_mma(const void* q, ll_dtype q_dtype, const ll_kvcache* cache,
                                           long long first_frame, int n_query_frames, const ll_rope_desc* rope,
                                           float softmax_scale, void* out, float* lse, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  g_last_error.clear();
  ll_status st = check_cache(cache);
  if (st != LL_OK) return st;
  if (cache->dtype != LL_FP8_E4M3)
    return fail(LL_ERR_INVALID_ARG, "ll_sink_window_attention_fp8_mma reads an FP8_E4M3 cache");
  if (cache->D != 128 || cache->H % 4 != 0)
    return fail(LL_ERR_UNSUPPORTED, "the FP8 tensor-core attention needs D = 128 and H a multiple of 4 (D = %d, H = %d)",
                cache->D, cache->H);
  if (q_dtype != LL_BF16) return fail(LL_ERR_INVALID_ARG, "q dtype must be BF16");
  if (q == nullptr || out == nullptr) return fail(LL_ERR_INVALID_ARG, "q and out must be non-NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(LL_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
  if (!aligned4(lse)) return fail(LL_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  if (first_frame < 0) return fail(LL_ERR_INVALID_ARG, "first_frame must be >= 0");
  if (n_query_frames < 1 || n_query_frames > cache->n_local)
    return fail(LL_ERR_INVALID_ARG, "n_query_frames = %d must lie in [1, n_local = %d]", n_query_frames,
                cache->n_local);
  if (!(softmax_scale >= 0.f) || !std::isfinite(softmax_scale))
    return fail(LL_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  const size_t need = ll_sink_window_attention_fp8_mma_workspace_bytes(cache, n_query_frames);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(LL_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu required", workspace_bytes, need);
  if (!aligned16(workspace)) return fail(LL_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if ((st = check_grid(rope, cache->tokens_per_frame)) != LL_OK) return st;
  const long long S = cache->n_sink + cache->n_local;
  const long long last = first_frame + n_query_frames - 1;
  const long long valid_slots = last + 1 < S ? last + 1 : S;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ll::AttnParams p{};
  if ((st = make_rope(rope, cache->H, cache->D, first_frame, &p.rp)) != LL_OK) return st;  // before any launch
  // the largest V scale of each (batch, head) over the valid keys
  const int units = ((n_query_frames * cache->tokens_per_frame + 127) / 128) * cache->H * cache->B;
  float* v_scale_max = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                                align256(attention_workspace<ll::AttnTraits<128, ll::E4M3Kv>>(units)));
  if (cudaMemsetAsync(v_scale_max, 0, static_cast<size_t>(cache->B) * cache->H * sizeof(float), s) != cudaSuccess)
    return check_launch("cudaMemsetAsync(V scale maxima)");
  ll::ScaleMaxParams sp{};
  sp.scale = cache->v_scale;
  sp.out = reinterpret_cast<unsigned int*>(v_scale_max);
  sp.rows = static_cast<int>(valid_slots * cache->tokens_per_frame);
  sp.batch_rows = static_cast<int>(S * cache->tokens_per_frame);
  sp.H = cache->H;
  const int per = 256 / cache->H;
  const long long want = (sp.rows + per - 1) / per;
  const dim3 grid(static_cast<unsigned>(want < num_sms() ? want : num_sms()), static_cast<unsigned>(cache->B));
  ll::scale_max_kernel<<<grid, 256, 0, s>>>(sp);
  if ((st = check_launch("scale_max_kernel")) != LL_OK) return st;
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.B = cache->B;
  p.H = cache->H;
  p.Tq = n_query_frames * cache->tokens_per_frame;
  p.Nk = static_cast<int>(valid_slots * cache->tokens_per_frame);
  p.softmax_scale = softmax_scale;
  p.N = cache->tokens_per_frame;
  p.v_scale_max = v_scale_max;
  return launch_attention<ll::AttnTraits<128, ll::E4M3Kv>>(p, cache, S, workspace, workspace_bytes, s);
}

}  // extern "C"

namespace {
// The bf16 attention kernel over a bf16 cache descriptor (validated by the caller).
ll_status launch_bf16_attention_on(const ll_kvcache* staged, const void* q, long long first_frame, int n_query_frames,
                                   const ll_rope_desc* rope, float softmax_scale, void* out, float* lse,
                                   void* workspace, size_t workspace_bytes, cudaStream_t s) {
  const long long S = staged->n_sink + staged->n_local;
  const long long last = first_frame + n_query_frames - 1;
  const long long valid_slots = last + 1 < S ? last + 1 : S;
  ll::AttnParams p{};
  ll_status st = make_rope(rope, staged->H, staged->D, first_frame, &p.rp);
  if (st != LL_OK) return st;
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.B = staged->B;
  p.H = staged->H;
  p.Tq = n_query_frames * staged->tokens_per_frame;
  p.Nk = static_cast<int>(valid_slots * staged->tokens_per_frame);
  p.softmax_scale = softmax_scale;
  p.N = staged->tokens_per_frame;
  if (staged->D == 128)
    return launch_attention<ll::AttnTraits<128, __nv_bfloat16>>(p, staged, S, workspace, workspace_bytes, s);
  return launch_attention<ll::AttnTraits<64, __nv_bfloat16>>(p, staged, S, workspace, workspace_bytes, s);
}
}  // namespace

extern "C" {

size_t ll_append_and_attend_workspace_bytes(const ll_kvcache* cache, int n_frames) {
  if (cache == nullptr || n_frames < 1 || cache->tokens_per_frame < 1 || cache->H < 1 || cache->B < 1) return 0;
  // + the grid barrier word; an FP8 cache: + the bf16 staging copy instead
  return attention_scratch_bytes(cache, n_frames) + (cache->dtype == LL_FP8_E4M3 ? fp8_staging_bytes(cache) : 256);
}

ll_status ll_append_and_attend(const ll_kvcache* cache, const void* k, const void* v, const void* q, ll_dtype dtype,
                               long long first_frame, int n_frames, const ll_rope_desc* rope, float softmax_scale,
                               void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  g_last_error.clear();
  ll_status st = check_cache(cache);
  if (st != LL_OK) return st;
  const bool fp8 = cache->dtype == LL_FP8_E4M3;
  if (fp8 ? dtype != LL_BF16 : dtype != cache->dtype)
    return fail(LL_ERR_INVALID_ARG, "k, v and q must have the cache's dtype (BF16 for an FP8 cache)");
  if (fp8 && cache->D != 128 && cache->D != 64)
    return fail(LL_ERR_UNSUPPORTED, "attention supports D = 64 or 128; got D = %d", cache->D);
  if (fp8 && cache->n_sink + cache->n_local > 64)
    return fail(LL_ERR_UNSUPPORTED, "the fused append over an FP8 cache takes at most 64 slots");
  if (k == nullptr || v == nullptr || q == nullptr || out == nullptr)
    return fail(LL_ERR_INVALID_ARG, "k, v, q and out must be non-NULL");
  if (!aligned16(k) || !aligned16(v) || !aligned16(q) || !aligned16(out))
    return fail(LL_ERR_INVALID_ARG, "k, v, q and out must be 16-byte aligned");
  if (!aligned4(lse)) return fail(LL_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  if (first_frame < 0) return fail(LL_ERR_INVALID_ARG, "first_frame must be >= 0");
  if (n_frames < 1 || n_frames > cache->n_local)
    return fail(LL_ERR_INVALID_ARG, "n_frames = %d must lie in [1, n_local = %d]", n_frames, cache->n_local);
  if (!(softmax_scale >= 0.f) || !std::isfinite(softmax_scale))
    return fail(LL_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  const size_t need = ll_append_and_attend_workspace_bytes(cache, n_frames);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(LL_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu required", workspace_bytes, need);
  if (!aligned16(workspace)) return fail(LL_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if ((st = check_grid(rope, cache->tokens_per_frame)) != LL_OK) return st;
  const bool f32 = cache->dtype == LL_F32;
  if (!((!f32 && (cache->D == 128 || cache->D == 64)) || (f32 && cache->D == 64)))
    return fail(LL_ERR_UNSUPPORTED, "attention supports D = 64 or 128 (bf16) and D = 64 (f32); got D = %d", cache->D);
  // the append part, exactly as ll_kvcache_append sets it up
  ll::AttnParams p{};
  ll::AppendParams& ap = p.ap;
  if ((st = make_rope(rope, cache->H, cache->D, first_frame, &ap.rp)) != LL_OK) return st;
  ap.k_in = k;
  ap.v_in = v;
  ap.k_cache = cache->k;
  ap.v_cache = cache->v;
  ap.k_scale = cache->k_scale;
  ap.v_scale = cache->v_scale;
  ap.B = cache->B;
  ap.F = n_frames;
  ap.N = cache->tokens_per_frame;
  ap.H = cache->H;
  ap.D = cache->D;
  ap.n_sink = cache->n_sink;
  ap.n_local = cache->n_local;
  ap.first_frame = first_frame;
  if (ll::append_items(ap) >= (1LL << 31))
    return fail(LL_ERR_UNSUPPORTED, "tensor too large for one call (%lld items)", ll::append_items(ap));
  if (fp8) return append_stage_and_attend(cache, ap, q, first_frame, n_frames, rope, softmax_scale, out, lse,
                                          workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
  // the append's frequency tables are built in the kernel's K stages
  const size_t tables = ll::append_smem_bytes(n_frames, cache->H, cache->D, ap.rp.pt);
  // the tables live in the kernel's second Q buffer during the append
  const size_t qbuf = cache->D == 128 ? ll::AttnTraits<128, __nv_bfloat16>::Q_BYTES
                                      : (f32 ? ll::AttnTraits<64, float>::Q_BYTES
                                             : ll::AttnTraits<64, __nv_bfloat16>::Q_BYTES);
  if (tables > qbuf)
    return fail(LL_ERR_UNSUPPORTED, "frequency tables of %zu bytes exceed %zu", tables, qbuf);
  // the attention part, exactly as ll_sink_window_attention sets it up
  const long long S = cache->n_sink + cache->n_local;
  const long long last = first_frame + n_frames - 1;
  const long long valid_slots = last + 1 < S ? last + 1 : S;
  if ((st = make_rope(rope, cache->H, cache->D, first_frame, &p.rp)) != LL_OK) return st;
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.B = cache->B;
  p.H = cache->H;
  p.Tq = n_frames * cache->tokens_per_frame;
  p.Nk = static_cast<int>(valid_slots * cache->tokens_per_frame);
  p.softmax_scale = softmax_scale;
  p.N = cache->tokens_per_frame;
  p.fuse_append = 1;
  p.gen = next_generation();
  p.grid_bar = reinterpret_cast<unsigned long long*>(static_cast<char*>(workspace) +
                                                     attention_scratch_bytes(cache, n_frames));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!f32 && cache->D == 128)
    return launch_attention<ll::AttnTraits<128, __nv_bfloat16>>(p, cache, S, workspace, workspace_bytes, s, true);
  if (!f32)
    return launch_attention<ll::AttnTraits<64, __nv_bfloat16>>(p, cache, S, workspace, workspace_bytes, s, true);
  return launch_attention<ll::AttnTraits<64, float>>(p, cache, S, workspace, workspace_bytes, s, true);
}

ll_status ll_phase_coherence(const ll_rope_desc* rope, int H, long long delta0, int n_delta, float* out,
                             void* stream) {
  g_last_error.clear();
  if (rope == nullptr || out == nullptr) return fail(LL_ERR_INVALID_ARG, "rope and out must be non-NULL");
  if ((reinterpret_cast<uintptr_t>(out) & 7u) != 0) return fail(LL_ERR_INVALID_ARG, "out must be 8-byte aligned");
  if (H < 1 || H > ll::kMaxHeads) return fail(LL_ERR_INVALID_ARG, "H = %d must lie in [1, %d]", H, ll::kMaxHeads);
  if (n_delta < 1) return fail(LL_ERR_INVALID_ARG, "n_delta must be >= 1");
  if (rope->pairs_t < 1) return fail(LL_ERR_INVALID_ARG, "the temporal band needs pairs_t >= 1");
  const long long lim = 1LL << 40;  // offsets far beyond any stream; keeps delta * t_scale exact in fp64
  if (delta0 < -lim || delta0 > lim - n_delta)
    return fail(LL_ERR_INVALID_ARG, "offsets must lie within +-2^40 frames");
  if (static_cast<long long>(H) * n_delta >= (1LL << 31))
    return fail(LL_ERR_UNSUPPORTED, "H * n_delta too large for one call");
  ll::PhaseParams p{};
  const int D = 2 * (rope->pairs_t + rope->pairs_h + rope->pairs_w);
  ll_status st = make_rope(rope, H, D, 0, &p.rp);
  if (st != LL_OK) return st;
  p.t_scale = rope->t_scale > 0.0 ? rope->t_scale : 1.0;
  p.delta0 = delta0;
  p.H = H;
  p.n = n_delta;
  p.out = reinterpret_cast<float2*>(out);
  const long long threads = static_cast<long long>(H) * n_delta;
  ll::phase_coherence_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0,
                               static_cast<cudaStream_t>(stream)>>>(p);
  return check_launch("phase_coherence_kernel");
}

ll_status ll_selftest_bounded_waits(void* stream) {
  g_last_error.clear();
  ll::selftest_bounded_waits_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(next_generation());
  return check_launch("selftest_bounded_waits_kernel");
}

}  // extern "C"

// Scratch of ll_sink_window_attention_noalloc: one copy per device that loads
// the library, alive until the process exits. In host code the symbol is only
// a handle; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LL_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = kDeviceSlots;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array of the device that `stream` belongs to,
// which must be the current device (the address is looked up once per device,
// with that device current).
ll_status noalloc_scratch(cudaStream_t stream, void** ptr) {
  int dev = -1, sdev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return check_launch("cudaGetDevice");
  if (cudaStreamGetDevice(stream, &sdev) != cudaSuccess) return check_launch("cudaStreamGetDevice");
  if (sdev != dev)
    return fail(LL_ERR_INVALID_ARG, "the stream belongs to device %d but device %d is current; make the stream's "
                                    "device current first", sdev, dev);
  if (dev < 0 || dev >= kMaxDevices) return fail(LL_ERR_UNSUPPORTED, "device ordinal %d is out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(LL_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return LL_OK;
}
}  // namespace

extern "C" {

ll_status ll_sink_window_attention_noalloc(const void* q, ll_dtype q_dtype, const ll_kvcache* cache,
                                           long long first_frame, int n_query_frames, const ll_rope_desc* rope,
                                           float softmax_scale, void* out, float* lse, void* stream) {
  g_last_error.clear();
  if (cache == nullptr) return fail(LL_ERR_INVALID_ARG, "cache is NULL");
  const size_t need = ll_sink_window_attention_workspace_bytes(cache, n_query_frames);
  if (need > LL_NOALLOC_SCRATCH_BYTES)
    return fail(LL_ERR_INVALID_ARG,
                "this call needs %zu bytes of scratch; the static scratch array holds %u "
                "(use ll_sink_window_attention with a caller workspace)",
                need, LL_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  const ll_status st = noalloc_scratch(static_cast<cudaStream_t>(stream), &scratch);
  if (st != LL_OK) return st;
  return ll_sink_window_attention(q, q_dtype, cache, first_frame, n_query_frames, rope, softmax_scale, out, lse,
                                  scratch, LL_NOALLOC_SCRATCH_BYTES, stream);
}

size_t ll_kv_recache_workspace_bytes(const ll_kvcache* cache, int d_model, int n_slots) {
  (void)cache;
  (void)d_model;
  (void)n_slots;
  return 0;  // the recache kernel needs no scratch
}

ll_status ll_kv_recache(const ll_kvcache* cache, const void* x, int d_model, const void* wk, const void* wv,
                        const float* gamma, float rms_eps, const long long* slot_frames, int n_slots,
                        const ll_rope_desc* rope, void* workspace, size_t workspace_bytes, void* stream) {
  g_last_error.clear();
  (void)workspace;
  (void)workspace_bytes;
  ll_status st = check_cache(cache);
  if (st != LL_OK) return st;
  if (x == nullptr || wk == nullptr || wv == nullptr || gamma == nullptr || slot_frames == nullptr)
    return fail(LL_ERR_INVALID_ARG, "x, wk, wv, gamma and slot_frames must be non-NULL");
  if (!aligned16(x) || !aligned16(wk) || !aligned16(wv))
    return fail(LL_ERR_INVALID_ARG, "x, wk and wv must be 16-byte aligned");
  if (!aligned4(gamma)) return fail(LL_ERR_INVALID_ARG, "gamma must be 4-byte aligned");
  const int S = cache->n_sink + cache->n_local;
  if (n_slots < 1 || n_slots > S || n_slots > ll::kMaxSlots)
    return fail(LL_ERR_INVALID_ARG, "n_slots = %d must lie in [1, %d]", n_slots, S < ll::kMaxSlots ? S : ll::kMaxSlots);
  for (int i = 0; i < n_slots; ++i)
    if (slot_frames[i] < 0 || slot_frames[i] > INT_MAX)
      return fail(LL_ERR_INVALID_ARG, "slot_frames[%d] = %lld lies outside [0, 2^31 - 1]", i, slot_frames[i]);
  if (!(rms_eps >= 0.f) || !std::isfinite(rms_eps)) return fail(LL_ERR_INVALID_ARG, "rms_eps must be finite, >= 0");
  if ((st = check_grid(rope, cache->tokens_per_frame)) != LL_OK) return st;
  if (cache->dtype != LL_BF16 && cache->dtype != LL_FP8_E4M3)
    return fail(LL_ERR_UNSUPPORTED, "kv recache writes BF16 or FP8 caches");
  const int Dout = cache->H * cache->D;
  if (d_model < 64 || d_model % 64 != 0)
    return fail(LL_ERR_UNSUPPORTED, "d_model = %d must be a positive multiple of 64", d_model);
  if (Dout % 256 != 0 || Dout / 256 > 8 || (cache->D != 64 && cache->D != 128))
    return fail(LL_ERR_UNSUPPORTED, "H*D = %d must be a multiple of 256 up to 2048 with D = 64 or 128", Dout);
  using TR = ll::RecacheTraits;
  ll::RecacheParams p{};
  if ((st = make_rope(rope, cache->H, cache->D, 0, &p.rp)) != LL_OK) return st;
  p.k_cache = cache->k;
  p.v_cache = cache->v;
  p.k_scale = cache->k_scale;
  p.v_scale = cache->v_scale;
  p.gamma = gamma;
  p.eps = rms_eps;
  p.M = n_slots * cache->tokens_per_frame;
  p.B = cache->B;
  p.Din = d_model;
  p.Dout = Dout;
  p.H = cache->H;
  p.D = cache->D;
  p.N = cache->tokens_per_frame;
  p.S = S;
  p.fp8 = cache->dtype == LL_FP8_E4M3;
  for (int i = 0; i < n_slots; ++i) p.slot_frame[i] = static_cast<int>(slot_frames[i]);
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(LL_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  CUtensorMap tmX, tmWk, tmWv;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)d_model, (cuuint64_t)p.M, (cuuint64_t)cache->B};
    const cuuint64_t strides[2] = {(cuuint64_t)d_model * 2, (cuuint64_t)p.M * d_model * 2};
    const cuuint32_t box[3] = {64u, 128u, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    if (fn(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return fail(LL_ERR_CUDA, "cuTensorMapEncodeTiled(x) failed");
  }
  for (int w = 0; w < 2; ++w) {
    const cuuint64_t dims[2] = {(cuuint64_t)Dout, (cuuint64_t)d_model};
    const cuuint64_t strides[1] = {(cuuint64_t)Dout * 2};
    const cuuint32_t box[2] = {64u, 64u};
    const cuuint32_t estr[2] = {1u, 1u};
    if (fn(w ? &tmWv : &tmWk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w ? wv : wk), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return fail(LL_ERR_CUDA, "cuTensorMapEncodeTiled(w) failed");
  }
  static std::atomic<unsigned long long> attr_set{0};
  const ll_status ast = once_per_device(attr_set, []() -> ll_status {
    if (cudaFuncSetAttribute(ll::kv_recache_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TR::SMEM_BYTES) !=
        cudaSuccess)
      return check_launch("cudaFuncSetAttribute(recache)");
    if (cudaFuncSetAttribute(ll::kv_recache_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0) != cudaSuccess)
      return check_launch("cudaFuncSetAttribute(recache cluster)");
    return LL_OK;
  });
  if (ast != LL_OK) return ast;
  // persistent clusters of Dout/256 CTAs (one per column tile), as many as
  // fit one CTA per SM, each walking every G-th (row block, K or V) tile
  const int C = Dout / TR::BN;
  const long long ntiles = 2LL * ((p.M + TR::BM - 1) / TR::BM) * cache->B;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(TR::THREADS, 1, 1);
  cfg.dynamicSmemBytes = TR::SMEM_BYTES;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // as many clusters as can be resident at once (a cluster's CTAs must share
  // one GPC), each walking a contiguous range of tiles
  int G = 0;
  cfg.gridDim = dim3(C, 1, 1);
  if (cudaOccupancyMaxActiveClusters(&G, ll::kv_recache_kernel, &cfg) != cudaSuccess || G < 1) {
    cudaGetLastError();
    G = num_sms() / C;
  }
  if (G < 1) G = 1;
  if (G > ntiles) G = static_cast<int>(ntiles);
  cfg.gridDim = dim3(C, G, 1);
  if (cudaLaunchKernelEx(&cfg, ll::kv_recache_kernel, tmX, tmWk, tmWv, p) != cudaSuccess)
    return check_launch("kv_recache_kernel");
  return check_launch("kv_recache_kernel");
}

}  // extern "C"
