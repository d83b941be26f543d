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
// i-th frame in a tensor: (t_first + i, n / grid_w, n % grid_w).
struct RopeParams {
  int enabled;
  int pt, ph, pw;          // pairs per band (t, h, w); pt + ph + pw = D/2
  int grid_w;
  long long t_first;       // temporal position of the tensor's first frame (t_offset included)
  double theta0;
  double sigma;
  float eps[kMaxHeads];    // per-head jitter draws (0 when there is no jitter)
};

// omega_i = base^(-2i/d) for pair j = 0..P-1 of head h (P = D/2): the temporal
// band (j < pt) uses base theta0 (1 + sigma eps_h), the row and column bands
// theta0; inside a band of `pairs` pairs, d = 2 * pairs. Evaluated in fp32 as
// exp2(-(i/pairs) * log2(base)): the relative error of omega is below 1e-6,
// i.e. under 3e-4 rad of angle at position 3000, far below bf16 resolution.
__device__ __forceinline__ float omega_of(const RopeParams& rp, int h, int j) {
  float base;
  int i, pairs;
  if (j < rp.pt) {
    base = static_cast<float>(rp.theta0 * (1.0 + rp.sigma * static_cast<double>(rp.eps[h])));
    i = j;
    pairs = rp.pt;
  } else if (j < rp.pt + rp.ph) {
    base = static_cast<float>(rp.theta0);
    i = j - rp.pt;
    pairs = rp.ph;
  } else {
    base = static_cast<float>(rp.theta0);
    i = j - rp.pt - rp.ph;
    pairs = rp.pw;
  }
  return exp2f(-(static_cast<float>(i) / static_cast<float>(pairs)) * log2f(base));
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

// Rotate the 4 pairs (x[0],x[1]) .. (x[6],x[7]) whose first pair index is j0
// with [[cos, -sin], [sin, cos]] at angle pos_axis * omega_j.
__device__ __forceinline__ void rotate_chunk8(float (&x)[8], int j0, float pos_t, float pos_r, float pos_c,
                                              const float* omega_h, int pt, int pth) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int j = j0 + q;
    const float pos = j < pt ? pos_t : (j < pth ? pos_r : pos_c);
    float s, c;
    sincosf(pos * omega_h[j], &s, &c);
    const float a = x[2 * q], b = x[2 * q + 1];
    x[2 * q] = a * c - b * s;
    x[2 * q + 1] = a * s + b * c;
  }
}

// sin and cos of x for |x| up to ~1e5: Cody and Waite's two-constant
// reduction x = k 2pi + r (k = rint(x / 2pi); 2pi split into its float
// rounding and the remainder, each product taken in one FMA) brings r into
// [-pi, pi], where the hardware approximation is accurate to ~4e-7 absolute.
__device__ __forceinline__ void sincos_reduced(float x, float& s, float& c) {
  const float k = rintf(x * 0.15915494309189535f);
  float r = fmaf(-k, 6.28318548202514648f, x);
  r = fmaf(k, 1.7484555314695172e-7f, r);
  __sincosf(r, &s, &c);
}

// rotate_chunk8 with sincos_reduced (query tiles staged by the attention kernel)
__device__ __forceinline__ void rotate_chunk8_fast(float (&x)[8], int j0, float pos_t, float pos_r, float pos_c,
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

// E4M3 codes of x / scale for one chunk; the (token, head) row of D values is
// spread over `group` consecutive lanes, which reduce max|x| with shuffles.
__device__ __forceinline__ uint2 quantize_chunk8_e4m3(const float (&x)[8], int group, float* scale_out) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
  for (int off = group >> 1; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  *scale_out = scale;
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
// K0: in-place RoPE of x [B][F*N][H][D].
// ---------------------------------------------------------------------------
struct RopeApplyParams {
  void* x;
  int B, F, N, H, D;
  RopeParams rp;
};

template <typename T>
__global__ void __launch_bounds__(256) rope_apply_kernel(const RopeApplyParams p) {
  extern __shared__ float s_omega[];  // [H][D/2]
  const int P = p.D / 2;
  build_omega(s_omega, p.rp, 0, p.H, P);
  __syncthreads();
  const int cpr = p.D / 8;  // chunks per (token, head) row
  const int total = p.B * p.F * p.N * p.H * cpr;  // < 2^31, checked on the host
  const int FN = p.F * p.N;
  T* x = static_cast<T*>(p.x);
  const int pth = p.rp.pt + p.rp.ph;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += gridDim.x * blockDim.x) {
    const int row = idx / cpr;
    const int c = idx - row * cpr;
    const int bt = row / p.H;
    const int h = row - bt * p.H;
    const int tok = bt % FN;
    const int fi = tok / p.N;
    const int n = tok - fi * p.N;
    const int r = n / p.rp.grid_w, col = n - r * p.rp.grid_w;
    float v[8];
    T* ptr = x + static_cast<size_t>(row) * p.D + c * 8;
    load_chunk8<T>(ptr, v);
    rotate_chunk8(v, c * 4, static_cast<float>(p.rp.t_first + fi), static_cast<float>(r),
                  static_cast<float>(col), s_omega + h * P, p.rp.pt, pth);
    store_chunk8<T>(ptr, v);
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
};

// Slot of frame f: pinned sink slots first, then a ring over the local slots
// (LongLive review, "Frame Sink": 3 sink frames stay; the short window keeps
// the most recent frames).
__device__ __forceinline__ int cache_slot(long long f, int n_sink, int n_local) {
  return f < n_sink ? static_cast<int>(f) : n_sink + static_cast<int>((f - n_sink) % n_local);
}

template <typename Tin, typename C>
__global__ void __launch_bounds__(256) append_kernel(const AppendParams p) {
  extern __shared__ float s_omega[];  // [H][D/2]
  const int P = p.D / 2;
  if (p.rp.enabled) build_omega(s_omega, p.rp, 0, p.H, P);
  __syncthreads();
  const int cpr = p.D / 8;
  const int total = p.B * p.F * p.N * p.H * cpr;  // < 2^31, checked on the host
  const int FN = p.F * p.N;
  const int S = p.n_sink + p.n_local;
  const int pth = p.rp.pt + p.rp.ph;
  const Tin* kin = static_cast<const Tin*>(p.k_in);
  const Tin* vin = static_cast<const Tin*>(p.v_in);
  // All threads of the block run the same number of iterations, so the
  // shuffles of the FP8 path always see full warps.
  for (int base = blockIdx.x * blockDim.x; base < total; base += gridDim.x * blockDim.x) {
    const int idx = base + threadIdx.x;
    const bool active = idx < total;
    const int i = active ? idx : 0;
    const int row = i / cpr;
    const int c = i - row * cpr;
    const int bt = row / p.H;                       // b * F*N + tok
    const int h = row - bt * p.H;
    const int b = bt / FN;
    const int tok = bt - b * FN;
    const int fi = tok / p.N;
    const int n = tok - fi * p.N;
    const int slot = cache_slot(p.first_frame + fi, p.n_sink, p.n_local);
    const size_t drow = (static_cast<size_t>(b) * S * p.N + static_cast<size_t>(slot) * p.N + n) * p.H + h;
    float kx[8], vx[8];
    if (active) {
      load_chunk8<Tin>(kin + static_cast<size_t>(row) * p.D + c * 8, kx);
      load_chunk8<Tin>(vin + static_cast<size_t>(row) * p.D + c * 8, vx);
      if (p.rp.enabled) {
        const int r = n / p.rp.grid_w, col = n - r * p.rp.grid_w;
        rotate_chunk8(kx, c * 4, static_cast<float>(p.rp.t_first + fi), static_cast<float>(r),
                      static_cast<float>(col), s_omega + h * P, p.rp.pt, pth);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) kx[e] = vx[e] = 0.f;
    }
    if constexpr (sizeof(C) == 1) {
      float ks, vs;
      const uint2 kq = quantize_chunk8_e4m3(kx, cpr, &ks);
      const uint2 vq = quantize_chunk8_e4m3(vx, cpr, &vs);
      if (active) {
        uint8_t* kc = static_cast<uint8_t*>(p.k_cache);
        uint8_t* vc = static_cast<uint8_t*>(p.v_cache);
        *reinterpret_cast<uint2*>(kc + drow * p.D + c * 8) = kq;
        *reinterpret_cast<uint2*>(vc + drow * p.D + c * 8) = vq;
        if (c == 0) {
          p.k_scale[drow] = ks;
          p.v_scale[drow] = vs;
        }
      }
    } else {
      if (active) {
        store_chunk8<C>(static_cast<C*>(p.k_cache) + drow * p.D + c * 8, kx);
        store_chunk8<C>(static_cast<C*>(p.v_cache) + drow * p.D + c * 8, vx);
      }
    }
  }
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
};

__global__ void __launch_bounds__(256) dequant_e4m3_kernel(const DequantParams p) {
  const int which = blockIdx.y;
  const int cpr = p.D / 16;  // 16-code chunks per (token, head) row
  const int per_batch = p.rows * p.H * cpr;
  const int total = p.B * per_batch;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += gridDim.x * blockDim.x) {
    const int b = idx / per_batch;
    const int r = idx - b * per_batch;         // (token * H + h) * cpr + c within the batch entry
    const int th = r / cpr, c = r - th * cpr;  // token-head row, chunk
    const size_t row = static_cast<size_t>(b) * p.batch_rows * p.H + th;
    const float sc = p.scale[which][row];
    const uint4 u = *reinterpret_cast<const uint4*>(p.src[which] + row * p.D + c * 16);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const __nv_fp8x2_storage_t q = static_cast<__nv_fp8x2_storage_t>((w[i] >> (16 * half)) & 0xFFFFu);
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(q, __NV_E4M3);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        o[2 * i + half] = pack_bf16(f.x * sc, f.y * sc);
      }
    }
    uint4* d = reinterpret_cast<uint4*>(p.dst[which] + row * p.D + c * 16);
    d[0] = make_uint4(o[0], o[1], o[2], o[3]);
    d[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace ll
