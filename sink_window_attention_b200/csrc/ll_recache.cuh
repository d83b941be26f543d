// ll_recache.cuh — KV recache at a prompt switch (LongLive review, "KV Recache":
// the cache is rebuilt from the generated frames with the new prompt).
//
// For every cached token row t (slot order) and both projections:
//   K[t] = RoPE(RMSNorm(X[t] Wk; gamma, eps))  at the slot's frame position,
//   V[t] = X[t] Wv,
// written straight into the cache row t (the rows of X are in slot order, so
// the scatter into slots is the identity on rows).
//
// One GEMM on the tensor cores: C[M, Dout] = X[M, Din] W[Din, Dout], output
// tiles of 128 rows x 256 columns (M=128, N=256, K=16 MMAs run at the full
// tensor rate), X as the K-major and W as the MN-major operand, both brought
// by TMA with 128-byte swizzle through a 2-stage ring, the accumulator in 256
// TMEM columns. The RMSNorm spans the whole Dout-wide row of K, i.e. all
// Dout/256 column tiles of a row block: those CTAs form one thread-block
// cluster and exchange their per-row partial sums of squares through
// distributed shared memory. The epilogue (warps 4-7, one row per thread)
// then normalises, applies gamma and the 3D RoPE pair rotation, converts to
// the cache type (bf16, or E4M3 with a per (token, head) scale) and stores.
// Two CTAs fit on an SM, so one CTA's epilogue overlaps the other's GEMM.
#pragma once

#include "ll_common.cuh"
#include "ll_rope_append.cuh"

namespace ll {

constexpr int kMaxSlots = 64;

struct RecacheParams {
  void* k_cache;       // [B][S*N][H][D] bf16 or E4M3 codes
  void* v_cache;
  float* k_scale;      // [B][S*N][H] (FP8 only)
  float* v_scale;
  const float* gamma;  // [Dout]
  float eps;
  int M;               // rows = n_slots * N
  int Din, Dout, H, D, N, S;  // S: slots of the cache
  int fp8;
  int slot_frame[kMaxSlots];  // absolute frame held by each recomputed slot
  RopeParams rp;              // rp.t_first = t_offset (frames add their own index)
};

struct RecacheTraits {
  static constexpr int BM = 128, BN = 256, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;   // 16 KB: X rows x 64 (one 128-byte swizzle column)
  static constexpr int B_BYTES = BK * BN * 2;   // 32 KB: 64 K rows x 256 columns (4 blocks of 64)
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = 2;
  static constexpr int CTRL_BYTES = 3072;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + CTRL_BYTES + 1024;
  static constexpr int TMEM_COLS = 256;
  static constexpr int THREADS = 256;
  static_assert(SMEM_BYTES * 2 <= 232448, "two CTAs per SM");
};

__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Grid: (Dout/256 column tiles = one cluster, ceil(M/128) row blocks, 2 * B):
// blockIdx.z = 2*b + (0: K, 1: V).
__global__ void __launch_bounds__(256, 2)
    kv_recache_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWk,
                      const __grid_constant__ CUtensorMap tmWv, const RecacheParams p) {
  using TR = RecacheTraits;
  constexpr int BM = TR::BM, BN = TR::BN, BK = TR::BK, ST = TR::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ctrl = smem + ST * TR::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + ST;
  uint64_t* acc_full = empty + ST;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  float* s_ss = reinterpret_cast<float*>(ctrl + 128);       // [128] partial sum of squares per row
  float* s_gamma = reinterpret_cast<float*>(ctrl + 640);    // [256]
  float* s_omega = s_gamma + BN;                            // [BN / D heads][D/2] = 128 floats

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = blockIdx.x;             // column tile == rank in the cluster
  const int m0 = blockIdx.y * BM;
  const int b = blockIdx.z >> 1;
  const bool is_k = (blockIdx.z & 1) == 0;
  const int n0 = nt * BN;
  const int kblocks = p.Din / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, TR::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp >= 2 && warp < 4) {  // stage gamma and this tile's heads' frequencies
    const int tid = threadIdx.x - 64;
    for (int j = tid; j < BN; j += 64) s_gamma[j] = p.gamma[n0 + j];
    const int h0 = n0 / p.D, nh = BN / p.D, P = p.D / 2;
    if (p.rp.enabled)
      for (int j = tid; j < nh * P; j += 64) s_omega[j] = omega_of(p.rp, h0 + j / P, j % P);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      const CUtensorMap* tmW = is_k ? &tmWk : &tmWv;
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(tmW);
      int issued = 0;
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % ST;
        if (!mbar_wait(&empty[s], ((kb / ST) & 1) ^ 1, s_abort)) break;
        uint8_t* sa = smem + s * TR::STAGE_BYTES;
        uint8_t* sb = sa + TR::A_BYTES;
        mbar_expect_tx(&full[s], TR::STAGE_BYTES);
        tma_load_3d(sa, &tmX, &full[s], kb * BK, m0, b);
#pragma unroll
        for (int blk = 0; blk < BN / 64; ++blk) tma_load_2d(sb + blk * (BK * 128), tmW, &full[s], n0 + blk * 64, kb * BK);
        issued = kb + 1;
      }
      if (*s_abort)
        for (int t = issued - ST > 0 ? issued - ST : 0; t < issued; ++t) mbar_wait_teardown(&full[t % ST], (t / ST) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_dense(BM, BN, 1, false, true);
      const uint32_t a0 = smem_addr(smem);
      const DescWords dA = desc_words(a0, 16, 1024, 2);
      const DescWords dB = desc_words(a0 + TR::A_BYTES, BK * 128, 1024, 2);
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % ST;
        if (!mbar_wait(&full[s], (kb / ST) & 1, s_abort)) break;
        tc_fence_after();
        const uint32_t so = s * TR::STAGE_BYTES;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          mma_bf16_ss(tbase, desc_at(dA, so + k * 32), desc_at(dB, so + k * 16 * 128), idesc,
                      (kb > 0 || k > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
      }
      mma_commit(acc_full);
      mbar_wait_teardown(acc_full, 0);  // TMEM stays allocated until every MMA is done
    }
  }

  // ------------------------------------------------ epilogue (warps 4-7), one row per thread
  const int row = threadIdx.x - 128;
  const uint32_t taddr = tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  bool ok = false;
  if (warp >= 4) {
    ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, s_abort));
    if (is_k) {
      float ss = 0.f;
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_load32(taddr + c * 32, r);
          tmem_load_wait(r);
#pragma unroll
          for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(r[e]), __uint_as_float(r[e]), ss);
        }
      }
      s_ss[row] = ss;
    }
  }
  // every CTA of the cluster (all threads) has published its partial sums
  cluster_sync_all();
  if (warp >= 4) {
    float inv_rms = 1.f;
    if (is_k) {
      const uint32_t mine = smem_addr(&s_ss[row]);
      float tot = 0.f;
      for (int r = 0; r < p.Dout / BN; ++r) tot += ld_cluster_f32(cluster_map(mine, r));
      inv_rms = rsqrtf(tot / static_cast<float>(p.Dout) + p.eps);
    }
    const int t = m0 + row;
    const bool live = ok && t < p.M;
    const int slot = live ? t / p.N : 0;
    const int n = live ? t - slot * p.N : 0;
    const int gw = p.rp.grid_w > 0 ? p.rp.grid_w : 1;
    const float pos_t = temporal_pos(p.rp, live ? p.slot_frame[slot] : 0);
    const float pos_r = static_cast<float>(n / gw);
    const float pos_c = static_cast<float>(n % gw);
    const size_t crow = static_cast<size_t>(b) * p.S * p.N + t;  // cache token row
    const int P = p.D / 2;
    const int pth = p.rp.pt + p.rp.ph;
    // accumulator columns [col, col+32) of head hc of this tile -> final values
    auto load_transform = [&](int hc, int c, float (&x)[32]) {
      uint32_t r[32];
      tmem_load32(taddr + (hc * p.D + c * 32), r);
      tmem_load_wait(r);
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(r[e]);
      if (!is_k) return;
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] *= inv_rms * s_gamma[hc * p.D + c * 32 + e];
      if (p.rp.enabled) {
        const float* om = s_omega + hc * P;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int j = c * 16 + q;  // pair index inside the head
          const float pos = j < p.rp.pt ? pos_t : (j < pth ? pos_r : pos_c);
          float sn, cs;
          sincosf(pos * om[j], &sn, &cs);
          const float a = x[2 * q], a2 = x[2 * q + 1];
          x[2 * q] = a * cs - a2 * sn;
          x[2 * q + 1] = a * sn + a2 * cs;
        }
      }
    };
    if (ok) {
      tc_fence_after();
      for (int hc = 0; hc < BN / p.D; ++hc) {
        const int h = (n0 + hc * p.D) / p.D;
        if (!p.fp8) {
          for (int c = 0; c < p.D / 32; ++c) {
            float x[32];
            load_transform(hc, c, x);
            if (!live) continue;
            __nv_bfloat16* dst =
                static_cast<__nv_bfloat16*>(is_k ? p.k_cache : p.v_cache) + (crow * p.H + h) * p.D + c * 32;
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              float y[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) y[e] = x[q8 * 8 + e];
              store_chunk8<__nv_bfloat16>(dst + q8 * 8, y);
            }
          }
        } else {
          // E4M3 per (token, head): the head's max first, then the codes (the
          // accumulator is still in TMEM, so the values are simply recomputed)
          float amax = 0.f;
          for (int c = 0; c < p.D / 32; ++c) {
            float x[32];
            load_transform(hc, c, x);
#pragma unroll
            for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(x[e]));
          }
          const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
          for (int c = 0; c < p.D / 32; ++c) {
            float x[32];
            load_transform(hc, c, x);
            if (!live) continue;
            uint8_t* dst = static_cast<uint8_t*>(is_k ? p.k_cache : p.v_cache) + (crow * p.H + h) * p.D + c * 32;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 v =
                    make_float2(__fdiv_rn(x[q * 8 + 2 * i], scale), __fdiv_rn(x[q * 8 + 2 * i + 1], scale));
                w[i] = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(v, __NV_SATFINITE, __NV_E4M3));
              }
              *reinterpret_cast<uint2*>(dst + q * 8) = make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
            }
          }
          if (live) (is_k ? p.k_scale : p.v_scale)[crow * p.H + h] = scale;
        }
      }
    }
  }
  // peers may still read this CTA's partial sums until everyone is here
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, TR::TMEM_COLS);
  }
}

}  // namespace ll
