// ll_rope_append.cuh — 3D RoPE with per-head jittered temporal base (LoL:
// Longer than Longer, review, "Prerequisites: RoPE" and "Method steps"), and
// the sink + ring KV-cache append (LongLive review, "Frame Sink",
// "Short-Window Attention"). Both are HBM-bound streaming kernels: every
// thread moves one 8-element chunk of a (token, head) row with 128-bit
// accesses; the frequency table of every head is built once per CTA in
// shared memory.
#pragma once

#include "ll_common.cuh"
#include <cuda_fp16.h>

namespace ll {

constexpr int kMaxHeads = 64;

// RoPE parameters as the kernels receive them. Position of token n of the
// i-th frame in a tensor: ((t_first + i) * t_scale, n / grid_w, n % grid_w).
struct RopeParams {
  int enabled;
  int pt, ph, pw;          // pairs per band (t, h, w); pt + ph + pw = D/2
  int grid_w;
  float t_scale;           // temporal position factor (position interpolation; 1 = plain RoPE)
  long long t_first;       // index of the tensor's first frame, t_offset included
  double theta0;
  double sigma;
  float eps[kMaxHeads];    // per-head jitter draws (0 when there is no jitter)
};

// omega_i = base^(-2i/d) for pair j = 0..P-1 of head h (P = D/2): the temporal
// band (j < pt) uses base theta0 (1 + sigma eps_h), the row and column bands
// theta0; inside a band of `pairs` pairs, d = 2 * pairs. Evaluated in fp32 as
// exp2(-(i/pairs) * log2(base)) (base itself in fp32: 6e-8 relative): the
// relative error of omega is below 1e-6, i.e. under 3e-4 rad of angle at
// position 3000, far below bf16 resolution.
__device__ __forceinline__ float omega_of(const RopeParams& rp, int h, int j) {
  const float theta0 = static_cast<float>(rp.theta0);
  float base = theta0;
  int i = j, pairs = rp.pt;
  if (j < rp.pt) {
    base = theta0 * fmaf(static_cast<float>(rp.sigma), rp.eps[h], 1.0f);
  } else if (j < rp.pt + rp.ph) {
    i = j - rp.pt;
    pairs = rp.ph;
  } else {
    i = j - rp.pt - rp.ph;
    pairs = rp.pw;
  }
  return exp2f(-(static_cast<float>(i) / static_cast<float>(pairs)) * log2f(base));
}

// Temporal position of the i-th frame of a tensor: (t_first + i) * t_scale
// (the frame index is exact in fp32 below 2^24; t_scale = 1 leaves it exact).
__device__ __forceinline__ float temporal_pos(const RopeParams& rp, long long i) {
  return static_cast<float>(rp.t_first + i) * rp.t_scale;
}

// omega[hh * P + j] for heads h0 .. h0+nh-1, built by the whole block.
__device__ __forceinline__ void build_omega(float* omega, const RopeParams& rp, int h0, int nh, int P) {
  for (int idx = threadIdx.x; idx < nh * P; idx += blockDim.x) {
    const int hh = idx / P;
    omega[idx] = omega_of(rp, h0 + hh, idx - hh * P);
  }
}

// omega[j] of one head, built by threads tid = 0..nthreads-1.
__device__ __forceinline__ void build_omega_one_head(float* omega, const RopeParams& rp, int h, int P, int tid,
                                                     int nthreads) {
  for (int j = tid; j < P; j += nthreads) omega[j] = omega_of(rp, h, j);
}

// sin and cos of x for |x| up to ~1e5: Cody and Waite's two-constant
// reduction x = k 2pi + r (k = rint(x / 2pi); 2pi split into its float
// rounding and the remainder, each product taken in one FMA) brings r into
// [-pi, pi], where the hardware approximation is accurate to ~4e-7 absolute.
// (The fp32 angle pos * omega itself carries ~1e-4 rad of rounding at frame
// indices in the thousands, far above either error.)
__device__ __forceinline__ void sincos_reduced(float x, float& s, float& c) {
  const float k = rintf(x * 0.15915494309189535f);
  float r = fmaf(-k, 6.28318548202514648f, x);
  r = fmaf(k, 1.7484555314695172e-7f, r);
  __sincosf(r, &s, &c);
}

// Rotate the 4 pairs (x[0],x[1]) .. (x[6],x[7]) whose first pair index is j0
// with [[cos, -sin], [sin, cos]] at angle pos_axis * omega_j.
__device__ __forceinline__ void rotate_chunk8(float (&x)[8], int j0, float pos_t, float pos_r, float pos_c,
                                              const float* omega_h, int pt, int pth) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int j = j0 + q;
    const float pos = j < pt ? pos_t : (j < pth ? pos_r : pos_c);
    float s, c;
    sincos_reduced(pos * omega_h[j], s, c);
    const float a = x[2 * q], b = x[2 * q + 1];
    x[2 * q] = a * c - b * s;
    x[2 * q + 1] = a * s + b * c;
  }
}

template <typename T>
__device__ __forceinline__ void load_chunk8(const T* p, float (&x)[8]);
template <>
__device__ __forceinline__ void load_chunk8<__nv_bfloat16>(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
    const float2 f = __bfloat1622float2(b);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
template <>
__device__ __forceinline__ void load_chunk8<float>(const float* p, float (&x)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

template <typename T>
__device__ __forceinline__ void store_chunk8(T* p, const float (&x)[8]);
template <>
__device__ __forceinline__ void store_chunk8<__nv_bfloat16>(__nv_bfloat16* p, const float (&x)[8]) {
  uint4 u;
  u.x = pack_bf16(x[0], x[1]);
  u.y = pack_bf16(x[2], x[3]);
  u.z = pack_bf16(x[4], x[5]);
  u.w = pack_bf16(x[6], x[7]);
  *reinterpret_cast<uint4*>(p) = u;
}
template <>
__device__ __forceinline__ void store_chunk8<float>(float* p, const float (&x)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
}

// E4M3 codes of x / scale for one chunk of 8 values (IEEE fp32 quotient,
// round to nearest even, saturating at +-448).
__device__ __forceinline__ uint2 encode_chunk8_e4m3(const float (&x)[8], float scale) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = make_float2(__fdiv_rn(x[2 * i], scale), __fdiv_rn(x[2 * i + 1], scale));
    const __nv_fp8x2_storage_t q = __nv_cvt_float2_to_fp8x2(v, __NV_SATFINITE, __NV_E4M3);
    w[i] = static_cast<uint32_t>(q);
  }
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// ---------------------------------------------------------------------------
// Phase-coherence kernel of a head's temporal band (LoL review, "Core
// innovation"): C_h(D) = (1/K) sum_{i<K} exp(j omega_{h,i} s D) with
// K = pt, omega_{h,i} = base_h^(-i/pt), base_h = theta0 (1 + sigma eps_h),
// s = t_scale, for the frame offsets D = delta0 .. delta0 + n - 1. One thread
// per (head, offset); frequencies, angles and the sum in fp64 (angles reach
// 1e5 rad and more), stored as fp32 (re, im).
// ---------------------------------------------------------------------------
struct PhaseParams {
  RopeParams rp;
  double t_scale;
  long long delta0;
  int H, n;
  float2* out;  // [H][n]
};

__global__ void __launch_bounds__(256) phase_coherence_kernel(const PhaseParams p) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(p.H) * p.n) return;
  const int h = static_cast<int>(idx / p.n);
  const int k = static_cast<int>(idx - static_cast<long long>(h) * p.n);
  const double lb = log2(p.rp.theta0 * (1.0 + p.rp.sigma * static_cast<double>(p.rp.eps[h])));
  const double d = static_cast<double>(p.delta0 + k) * p.t_scale;
  double re = 0.0, im = 0.0;
  for (int i = 0; i < p.rp.pt; ++i) {
    const double w = exp2(-(static_cast<double>(i) / p.rp.pt) * lb);
    double sn, cs;
    sincos(w * d, &sn, &cs);
    re += cs;
    im += sn;
  }
  p.out[idx] = make_float2(static_cast<float>(re / p.rp.pt), static_cast<float>(im / p.rp.pt));
}

// ---------------------------------------------------------------------------
// K0: in-place RoPE of x [B][F*N][H][D].
// ---------------------------------------------------------------------------
struct RopeApplyParams {
  void* x;
  int B, F, N, H, D;
  RopeParams rp;
};

// One thread per (head, 8-element chunk) of a token row (blockDim = H * D/8),
// kRopeTokens token rows per block: a thread's head and pairs, hence its 4
// frequencies, are the same for every row it rotates, so they are evaluated
// once per thread; the rows' positions once per row; the loads of all rows
// are issued before any rotation.
constexpr int kRopeTokens = 4;

template <typename T>
__global__ void __launch_bounds__(1024) rope_apply_kernel(const RopeApplyParams p) {
  __shared__ float s_pos[kRopeTokens][3];  // temporal, row and column position of each token row
  const int cpr = p.D / 8;
  const int h = threadIdx.x / cpr, c = threadIdx.x - h * cpr;
  const int rows = p.B * p.F * p.N;
  const int r0 = blockIdx.x * kRopeTokens;
  const int nt = min(kRopeTokens, rows - r0);
  for (int k = threadIdx.x; k < nt; k += blockDim.x) {  // blockDim may be below kRopeTokens (H * D / 8 < 4)
    const int tok = (r0 + k) % (p.F * p.N);
    const int fi = tok / p.N, n = tok - fi * p.N;
    const int r = n / p.rp.grid_w;
    s_pos[k][0] = temporal_pos(p.rp, fi);
    s_pos[k][1] = static_cast<float>(r);
    s_pos[k][2] = static_cast<float>(n - r * p.rp.grid_w);
  }
  const int pth = p.rp.pt + p.rp.ph;
  float om[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) om[q] = omega_of(p.rp, h, c * 4 + q);
  T* x = static_cast<T*>(p.x) + (static_cast<size_t>(r0) * p.H + h) * p.D + c * 8;
  float v[kRopeTokens][8];
#pragma unroll
  for (int k = 0; k < kRopeTokens; ++k)
    if (k < nt) load_chunk8<T>(x + static_cast<size_t>(k) * p.H * p.D, v[k]);
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kRopeTokens; ++k) {
    if (k >= nt) break;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = c * 4 + q;
      const float pos = j < p.rp.pt ? s_pos[k][0] : (j < pth ? s_pos[k][1] : s_pos[k][2]);
      float sn, cs;
      sincos_reduced(pos * om[q], sn, cs);
      const float a = v[k][2 * q], b = v[k][2 * q + 1];
      v[k][2 * q] = a * cs - b * sn;
      v[k][2 * q + 1] = a * sn + b * cs;
    }
    store_chunk8<T>(x + static_cast<size_t>(k) * p.H * p.D, v[k]);
  }
}

// ---------------------------------------------------------------------------
// K1: append F frames of K (rotated here unless rp.enabled == 0) and V to
// their cache slots. Cache element type C: bf16, f32, or uint8_t (E4M3 codes
// with per-(token, head) fp32 scales).
// ---------------------------------------------------------------------------
struct AppendParams {
  const void* k_in;
  const void* v_in;
  void* k_cache;
  void* v_cache;
  float* k_scale;
  float* v_scale;
  int B, F, N, H, D;
  int n_sink, n_local;     // cache slots S = n_sink + n_local
  long long first_frame;   // absolute index of the first appended frame
  RopeParams rp;
  // E4M3 cache only, optional: bf16 rows [B][S*N][H][D] that also receive the
  // dequantised value (code * scale) of every code written
  __nv_bfloat16* stage_k;
  __nv_bfloat16* stage_v;
};

// Slot of frame f: pinned sink slots first, then a ring over the local slots
// (LongLive review, "Frame Sink": 3 sink frames stay; the short window keeps
// the most recent frames).
__device__ __forceinline__ int cache_slot(long long f, int n_sink, int n_local) {
  return f < n_sink ? static_cast<int>(f) : n_sink + static_cast<int>((f - n_sink) % n_local);
}

// One thread: one 8-element chunk position c of one token, for a group of
// `hg` heads. The angles of the chunk's 4 pairs are shared: a pair of the row
// or column band has the same angle in every head (no jitter there), and a
// pair of the temporal band has the same angle for every token of a frame,
// so its cos/sin come from a per-block table [F][H][pt]. Consecutive threads
// take consecutive chunks of a (token, head) row, so every access is a
// coalesced 16 bytes.
__host__ __device__ __forceinline__ int append_heads_per_thread(int H) {
  return (H % 4 == 0) ? 4 : (H % 3 == 0 ? 3 : (H % 2 == 0 ? 2 : 1));
}
constexpr int kAppendMaxHg = 4;

__host__ __device__ __forceinline__ size_t append_smem_bytes(int F, int H, int D, int pt) {
  return (static_cast<size_t>(H) * (D / 2) + 2 * static_cast<size_t>(F) * H * pt) * sizeof(float);
}

// Frequency table [H][D/2] and the temporal band's cos/sin [F][H][pt][2] in
// shared memory, built by the whole block (two block barriers).
__device__ __forceinline__ void build_append_tables(float* s_omega, float* s_tcs, const AppendParams& p) {
  const int P = p.D / 2;
  build_omega(s_omega, p.rp, 0, p.H, P);
  __syncthreads();
  const int nt = p.F * p.H * p.rp.pt;
  for (int idx = threadIdx.x; idx < nt; idx += blockDim.x) {
    const int f = idx / (p.H * p.rp.pt), rem = idx - f * (p.H * p.rp.pt);
    const int h = rem / p.rp.pt, j = rem - h * p.rp.pt;
    float sn, cs;
    sincos_reduced(temporal_pos(p.rp, f) * s_omega[h * P + j], sn, cs);
    s_tcs[2 * idx] = cs;
    s_tcs[2 * idx + 1] = sn;
  }
  __syncthreads();
}

// Number of append work items: (token, 8-element chunk position, group of
// append_heads_per_thread(H) heads).
__host__ __device__ __forceinline__ long long append_items(const AppendParams& p) {
  return static_cast<long long>(p.B) * p.F * p.N * (p.D / 8) * (p.H / append_heads_per_thread(p.H));
}

// One work item: where its chunks come from and go to.
struct AppendItem {
  int c, h0, fi, n;
  size_t src0, dst0;  // element offsets of the group's first head in the input and in the cache
};

__device__ __forceinline__ AppendItem append_item(const AppendParams& p, int i) {
  const int cpr = p.D / 8;
  const int hg = append_heads_per_thread(p.H);
  const int ngroups = p.H / hg;
  AppendItem it;
  const int grow = i / cpr;  // (b * F*N + tok) * ngroups + group
  it.c = i - grow * cpr;
  const int bt = grow / ngroups;
  it.h0 = (grow - bt * ngroups) * hg;
  const int FN = p.F * p.N;
  const int b = bt / FN;
  const int tok = bt - b * FN;
  it.fi = tok / p.N;
  it.n = tok - it.fi * p.N;
  const int S = p.n_sink + p.n_local;
  const int slot = cache_slot(p.first_frame + it.fi, p.n_sink, p.n_local);
  it.src0 = (static_cast<size_t>(bt) * p.H + it.h0) * p.D + it.c * 8;
  it.dst0 = ((static_cast<size_t>(b) * S * p.N + static_cast<size_t>(slot) * p.N + it.n) * p.H + it.h0) * p.D +
            it.c * 8;
  return it;
}

template <typename Tin>
__device__ __forceinline__ void append_load(const AppendParams& p, const AppendItem& it, bool active,
                                            float (&kx)[kAppendMaxHg][8], float (&vx)[kAppendMaxHg][8]) {
  const int hg = append_heads_per_thread(p.H);
  const Tin* kin = static_cast<const Tin*>(p.k_in);
  const Tin* vin = static_cast<const Tin*>(p.v_in);
#pragma unroll
  for (int k = 0; k < kAppendMaxHg; ++k) {
    if (active && k < hg) {
      load_chunk8<Tin>(kin + it.src0 + static_cast<size_t>(k) * p.D, kx[k]);
      load_chunk8<Tin>(vin + it.src0 + static_cast<size_t>(k) * p.D, vx[k]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) kx[k][e] = vx[k][e] = 0.f;
    }
  }
}

// Rotate the K chunks of an item: a row- or column-band pair has one angle for
// all heads; a temporal-band pair takes its head's cos/sin from the table.
__device__ __forceinline__ void append_rotate(const AppendParams& p, const AppendItem& it, const float* s_omega,
                                              const float* s_tcs, float (&kx)[kAppendMaxHg][8]) {
  const int hg = append_heads_per_thread(p.H);
  const int pth = p.rp.pt + p.rp.ph;
  const float pos_r = static_cast<float>(it.n / p.rp.grid_w), pos_c = static_cast<float>(it.n % p.rp.grid_w);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int j = it.c * 4 + q;
    float cs[kAppendMaxHg], sn[kAppendMaxHg];
    if (j < p.rp.pt) {
#pragma unroll
      for (int k = 0; k < kAppendMaxHg; ++k) {
        const int e = k < hg ? ((it.fi * p.H + it.h0 + k) * p.rp.pt + j) : 0;
        cs[k] = s_tcs[2 * e];
        sn[k] = s_tcs[2 * e + 1];
      }
    } else {
      float s1, c1;
      sincos_reduced((j < pth ? pos_r : pos_c) * s_omega[j], s1, c1);
#pragma unroll
      for (int k = 0; k < kAppendMaxHg; ++k) {
        cs[k] = c1;
        sn[k] = s1;
      }
    }
#pragma unroll
    for (int k = 0; k < kAppendMaxHg; ++k) {
      const float x0 = kx[k][2 * q], x1 = kx[k][2 * q + 1];
      kx[k][2 * q] = x0 * cs[k] - x1 * sn[k];
      kx[k][2 * q + 1] = x0 * sn[k] + x1 * cs[k];
    }
  }
}

template <typename C>
__device__ __forceinline__ void append_store_plain(const AppendParams& p, const AppendItem& it,
                                                   const float (&kx)[kAppendMaxHg][8],
                                                   const float (&vx)[kAppendMaxHg][8]) {
  const int hg = append_heads_per_thread(p.H);
#pragma unroll
  for (int k = 0; k < kAppendMaxHg; ++k)
    if (k < hg) {
      store_chunk8<C>(static_cast<C*>(p.k_cache) + it.dst0 + static_cast<size_t>(k) * p.D, kx[k]);
      store_chunk8<C>(static_cast<C*>(p.v_cache) + it.dst0 + static_cast<size_t>(k) * p.D, vx[k]);
    }
}

// bf16 of code * scale for 8 E4M3 codes (the exact code value times the fp32
// scale, rounded once): the values attention reads from the staging copy.
__device__ __forceinline__ uint4 decode_chunk8_e4m3_bf16(uint2 codes, float scale) {
  const uint32_t w[2] = {codes.x, codes.y};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const __nv_fp8x2_storage_t q = static_cast<__nv_fp8x2_storage_t>((w[i] >> (16 * half)) & 0xFFFFu);
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(q, __NV_E4M3);
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
      o[2 * i + half] = pack_bf16(f.x * scale, f.y * scale);
    }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// The append over blocks blk = 0..nblk-1 of 256 threads (the whole grid of
// append_kernel, or the append share of the fused E4M3 append + staging).
template <typename Tin, typename C>
__device__ __forceinline__ void append_blocks(const AppendParams& p, int blk, int nblk) {
  extern __shared__ float s_tab[];      // omega [H][D/2], then cos, sin of the temporal band [F][H][pt][2]
  float* s_omega = s_tab;
  float* s_tcs = s_tab + p.H * (p.D / 2);
  const int cpr = p.D / 8;                        // chunks per (token, head) row
  const int hg = append_heads_per_thread(p.H);    // heads per thread
  const int total = static_cast<int>(append_items(p));  // < 2^31, checked on the host
  const int stride = nblk * blockDim.x;
  float kx[kAppendMaxHg][8], vx[kAppendMaxHg][8];
  // the first chunks' loads go out before the tables are built, so the
  // table work overlaps their latency
  int base = blk * blockDim.x;
  {
    const int idx = base + threadIdx.x;
    append_load<Tin>(p, append_item(p, idx < total ? idx : 0), idx < total, kx, vx);
  }
  if (p.rp.enabled) build_append_tables(s_omega, s_tcs, p);
  // All threads of the block run the same number of iterations, so the
  // shuffles of the FP8 path always see full warps.
  for (; base < total; base += stride) {
    const int idx = base + threadIdx.x;
    const bool active = idx < total;
    const AppendItem it = append_item(p, active ? idx : 0);
    if (active && p.rp.enabled) append_rotate(p, it, s_omega, s_tcs, kx);
    if constexpr (sizeof(C) == 1) {
      // per (token, head) row: scale = max|x| / 448 over the row's D values,
      // which lie in the cpr consecutive lanes of this chunk position's group
      uint8_t* kc = static_cast<uint8_t*>(p.k_cache) + it.dst0;
      uint8_t* vc = static_cast<uint8_t*>(p.v_cache) + it.dst0;
#pragma unroll
      for (int k = 0; k < kAppendMaxHg; ++k) {
        if (k >= hg) break;  // hg is uniform across the grid
        float ka = 0.f, va = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          ka = fmaxf(ka, fabsf(kx[k][e]));
          va = fmaxf(va, fabsf(vx[k][e]));
        }
        for (int off = cpr >> 1; off > 0; off >>= 1) {
          ka = fmaxf(ka, __shfl_xor_sync(0xffffffffu, ka, off));
          va = fmaxf(va, __shfl_xor_sync(0xffffffffu, va, off));
        }
        const float ks = ka > 0.f ? __fdiv_rn(ka, 448.0f) : 1.0f;
        const float vs = va > 0.f ? __fdiv_rn(va, 448.0f) : 1.0f;
        if (active) {
          const uint2 kq = encode_chunk8_e4m3(kx[k], ks), vq = encode_chunk8_e4m3(vx[k], vs);
          *reinterpret_cast<uint2*>(kc + static_cast<size_t>(k) * p.D) = kq;
          *reinterpret_cast<uint2*>(vc + static_cast<size_t>(k) * p.D) = vq;
          if (p.stage_k != nullptr) {
            *reinterpret_cast<uint4*>(p.stage_k + it.dst0 + static_cast<size_t>(k) * p.D) = decode_chunk8_e4m3_bf16(kq, ks);
            *reinterpret_cast<uint4*>(p.stage_v + it.dst0 + static_cast<size_t>(k) * p.D) = decode_chunk8_e4m3_bf16(vq, vs);
          }
          if (it.c == 0) {
            const size_t srow = it.dst0 / p.D + k;
            p.k_scale[srow] = ks;
            p.v_scale[srow] = vs;
          }
        }
      }
    } else {
      if (active) append_store_plain<C>(p, it, kx, vx);
    }
    if (base + stride < total) {  // uniform condition
      const int nidx = base + stride + threadIdx.x;
      append_load<Tin>(p, append_item(p, nidx < total ? nidx : 0), nidx < total, kx, vx);
    }
  }
}

// ll_kvcache_append: one thread per (head, 8-element chunk) of a token row
// (blockDim = H * D/8) and kAppendTokens token rows per block, as in the
// in-place RoPE: a thread's 4 frequencies are evaluated once; each row's
// position and cache row once per block (shared memory); the K and V loads of
// all rows are issued before any rotation. The angles are the same products
// position x frequency as append_blocks forms (which the fused E4M3 staging
// kernel uses), so the cache rows are the same bits. E4M3: the D/8 lanes of a
// (token, head) row reduce its max|x| by shuffles; blockDim is rounded up to
// whole warps and the lanes past H * D/8 only take part in the shuffles.
constexpr int kAppendTokens = 2;

template <typename Tin, typename C>
__global__ void __launch_bounds__(1024) append_kernel(const AppendParams p) {
  __shared__ float s_pos[kAppendTokens][3];      // temporal, row and column position
  __shared__ long long s_dst[kAppendTokens];     // cache token row (batch entry, slot, token)
  const int cpr = p.D / 8;
  const bool live = static_cast<int>(threadIdx.x) < p.H * cpr;
  const int h = live ? threadIdx.x / cpr : 0, c = threadIdx.x - (threadIdx.x / cpr) * cpr;
  const int FN = p.F * p.N, rows = p.B * FN;
  const int r0 = blockIdx.x * kAppendTokens;
  const int nt = min(kAppendTokens, rows - r0);
  for (int k = threadIdx.x; k < nt; k += blockDim.x) {
    const int b = (r0 + k) / FN, tok = (r0 + k) - b * FN;
    const int fi = tok / p.N, n = tok - fi * p.N;
    const int gw = p.rp.grid_w > 0 ? p.rp.grid_w : 1;
    const int r = n / gw;
    s_pos[k][0] = temporal_pos(p.rp, fi);
    s_pos[k][1] = static_cast<float>(r);
    s_pos[k][2] = static_cast<float>(n - r * gw);
    const int S = p.n_sink + p.n_local;
    s_dst[k] = (static_cast<long long>(b) * S + cache_slot(p.first_frame + fi, p.n_sink, p.n_local)) * p.N + n;
  }
  float om[4];
  if (p.rp.enabled) {
#pragma unroll
    for (int q = 0; q < 4; ++q) om[q] = omega_of(p.rp, h, c * 4 + q);
  }
  const Tin* kin = static_cast<const Tin*>(p.k_in) + (static_cast<size_t>(r0) * p.H + h) * p.D + c * 8;
  const Tin* vin = static_cast<const Tin*>(p.v_in) + (static_cast<size_t>(r0) * p.H + h) * p.D + c * 8;
  float kx[kAppendTokens][8], vx[kAppendTokens][8];
#pragma unroll
  for (int k = 0; k < kAppendTokens; ++k) {
    if (live && k < nt) {
      load_chunk8<Tin>(kin + static_cast<size_t>(k) * p.H * p.D, kx[k]);
      load_chunk8<Tin>(vin + static_cast<size_t>(k) * p.H * p.D, vx[k]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) kx[k][e] = vx[k][e] = 0.f;
    }
  }
  __syncthreads();
  const int pth = p.rp.pt + p.rp.ph;
#pragma unroll
  for (int k = 0; k < kAppendTokens; ++k) {
    if (k >= nt) break;  // uniform across the block
    if (p.rp.enabled) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = c * 4 + q;
        const float pos = j < p.rp.pt ? s_pos[k][0] : (j < pth ? s_pos[k][1] : s_pos[k][2]);
        float sn, cs;
        sincos_reduced(pos * om[q], sn, cs);
        const float x0 = kx[k][2 * q], x1 = kx[k][2 * q + 1];
        kx[k][2 * q] = x0 * cs - x1 * sn;
        kx[k][2 * q + 1] = x0 * sn + x1 * cs;
      }
    }
    const size_t dst = (static_cast<size_t>(s_dst[k]) * p.H + h) * p.D + c * 8;
    if constexpr (sizeof(C) == 1) {
      // per (token, head) row: scale = max|x| / 448 over the row's D values,
      // held by the cpr consecutive lanes of this head
      float ka = 0.f, va = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        ka = fmaxf(ka, fabsf(kx[k][e]));
        va = fmaxf(va, fabsf(vx[k][e]));
      }
      for (int off = cpr >> 1; off > 0; off >>= 1) {
        ka = fmaxf(ka, __shfl_xor_sync(0xffffffffu, ka, off));
        va = fmaxf(va, __shfl_xor_sync(0xffffffffu, va, off));
      }
      const float ks = ka > 0.f ? __fdiv_rn(ka, 448.0f) : 1.0f;
      const float vs = va > 0.f ? __fdiv_rn(va, 448.0f) : 1.0f;
      if (!live) continue;
      const uint2 kq = encode_chunk8_e4m3(kx[k], ks), vq = encode_chunk8_e4m3(vx[k], vs);
      *reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.k_cache) + dst) = kq;
      *reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.v_cache) + dst) = vq;
      if (p.stage_k != nullptr) {
        *reinterpret_cast<uint4*>(p.stage_k + dst) = decode_chunk8_e4m3_bf16(kq, ks);
        *reinterpret_cast<uint4*>(p.stage_v + dst) = decode_chunk8_e4m3_bf16(vq, vs);
      }
      if (c == 0) {
        p.k_scale[dst / p.D] = ks;
        p.v_scale[dst / p.D] = vs;
      }
    } else if (live) {
      store_chunk8<C>(static_cast<C*>(p.k_cache) + dst, kx[k]);
      store_chunk8<C>(static_cast<C*>(p.v_cache) + dst, vx[k]);
    }
  }
}

// ---------------------------------------------------------------------------
// Largest scale of each (batch, head) over the first `rows` tokens of an E4M3
// cache's scale array [B][batch_rows][H]: out[b * H + h], zeroed before the
// launch (scales are positive, so their bits order as unsigned integers and
// atomicMax on the bits is the float maximum). Grid (x: row blocks, y: batch);
// H <= kMaxHeads.
// ---------------------------------------------------------------------------
struct ScaleMaxParams {
  const float* scale;
  unsigned int* out;
  int rows, batch_rows, H;
};

__global__ void __launch_bounds__(256) scale_max_kernel(const ScaleMaxParams p) {
  __shared__ unsigned int smax[kMaxHeads];
  for (int i = threadIdx.x; i < p.H; i += blockDim.x) smax[i] = 0u;
  __syncthreads();
  const int b = blockIdx.y;
  const int per = blockDim.x / p.H;  // tokens a pass of the block reads
  const int h = threadIdx.x % p.H, r0 = threadIdx.x / p.H;
  if (r0 < per) {
    float m = 0.f;
    for (int r = blockIdx.x * per + r0; r < p.rows; r += gridDim.x * per)
      m = fmaxf(m, p.scale[(static_cast<size_t>(b) * p.batch_rows + r) * p.H + h]);
    atomicMax(&smax[h], __float_as_uint(m));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < p.H; i += blockDim.x) atomicMax(&p.out[b * p.H + i], smax[i]);
}

// ---------------------------------------------------------------------------
// E4M3 cache rows -> bf16: value = decode(code) * scale for the first `rows`
// token rows of every batch entry, K and V (blockIdx.y = 0 / 1). 16 codes
// (16 bytes) per thread.
// ---------------------------------------------------------------------------
struct DequantParams {
  const uint8_t* src[2];
  const float* scale[2];
  __nv_bfloat16* dst[2];
  int B, rows, batch_rows, H, D;
  int cshift;                   // log2(D / 16): 16-code chunks per (token, head) row
  int nskip;                    // rows left alone: (token, head) rows [skip_lo[i], skip_hi[i]) of every batch entry
  int skip_lo[3], skip_hi[3];
};

// K (isv false) or V rows of every batch entry over blocks blk = 0..nblk-1.
// The first `rows` token rows of a batch entry are contiguous ([rows][H][D]
// codes, [rows][H] scales), so chunk i of a batch entry (16 codes) starts at
// code 16 i and belongs to (token, head) row i >> cshift: no division in the
// index arithmetic.
// U: chunks per thread per pass, their loads in flight together.
template <int U>
__device__ __forceinline__ void dequant_blocks(const DequantParams& p, bool isv, int blk, int nblk) {
  const uint8_t* src = isv ? p.src[1] : p.src[0];  // selected, not indexed, to keep the params out of local memory
  const float* scale = isv ? p.scale[1] : p.scale[0];
  __nv_bfloat16* dst = isv ? p.dst[1] : p.dst[0];
  const int per_batch = (p.rows * p.H) << p.cshift;
  const int stride = nblk * blockDim.x;
  for (int b = 0; b < p.B; ++b) {
    const size_t row0 = static_cast<size_t>(b) * p.batch_rows * p.H;  // first (token, head) row of the entry
    const uint4* srcb = reinterpret_cast<const uint4*>(src + row0 * p.D);
    const float* scb = scale + row0;
    uint4* dstb = reinterpret_cast<uint4*>(dst + row0 * p.D);
    for (int base = blk * blockDim.x + threadIdx.x; base < per_batch; base += U * stride) {
      uint4 u[U];
      float sc[U];
      bool go[U];
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const int idx = base + k * stride;
        const int th = idx >> p.cshift;
        bool g = idx < per_batch;
#pragma unroll
        for (int i = 0; i < 3; ++i)  // constant indices keep the params out of local memory
          if (i < p.nskip) g = g && !(th >= p.skip_lo[i] && th < p.skip_hi[i]);
        go[k] = g;
        sc[k] = g ? scb[th] : 0.f;
        u[k] = g ? srcb[idx] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int k = 0; k < U; ++k) {
        if (!go[k]) continue;
        const uint32_t w[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
        uint32_t o[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const __nv_fp8x2_storage_t q = static_cast<__nv_fp8x2_storage_t>((w[i] >> (16 * half)) & 0xFFFFu);
            const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(q, __NV_E4M3);
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
            o[2 * i + half] = pack_bf16(f.x * sc[k], f.y * sc[k]);
          }
        }
        const int idx = base + k * stride;
        dstb[2 * idx] = make_uint4(o[0], o[1], o[2], o[3]);
        dstb[2 * idx + 1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
    }
  }
}

// blockIdx.y = 0 / 1: K / V rows.
__global__ void __launch_bounds__(256) dequant_e4m3_kernel(const DequantParams p) {
  dequant_blocks<4>(p, blockIdx.y != 0, blockIdx.x, gridDim.x);
}

// E4M3 cache: the append of the new frames (RoPE on K, per (token, head)
// quantisation, codes and scales into their slots, and the dequantised values
// into the bf16 staging rows) and the dequantisation of every other occupied
// row into the staging copy, in one launch. Blocks [0, append_blocks) append;
// the rest are split evenly between the K and V rows of the slots the append
// does not write (dq's skip ranges). The staging rows equal those of
// ll_kvcache_append followed by the dequantisation pass.
struct AppendStageParams {
  AppendParams ap;
  DequantParams dq;              // with the rows of the appended frames' slots skipped
  int append_blocks;
  int dequant_blocks;            // per K and per V
};

__global__ void __launch_bounds__(256) append_stage_e4m3_kernel(const AppendStageParams q) {
  const int blk = blockIdx.x;
  if (blk < q.append_blocks) {
    append_blocks<__nv_bfloat16, uint8_t>(q.ap, blk, q.append_blocks);
  } else {
    const int d = blk - q.append_blocks;
    const bool isv = d >= q.dequant_blocks;
    // the append's register allocation leaves few blocks per SM: more loads in flight per thread
    dequant_blocks<8>(q.dq, isv, isv ? d - q.dequant_blocks : d, q.dequant_blocks);
  }
}

}  // namespace ll
