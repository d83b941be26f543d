// ll_recache.cuh — KV recache at a prompt switch (LongLive review, "KV Recache":
// the cache is rebuilt from the generated frames with the new prompt).
//
// For every cached token row t (slot order) and both projections:
//   K[t] = RoPE(RMSNorm(X[t] Wk; gamma, eps))  at the slot's frame position,
//   V[t] = X[t] Wv,
// written straight into the cache row t (the rows of X are in slot order, so
// the scatter into slots is the identity on rows).
//
// One GEMM on the tensor cores, C[M, Dout] = X[M, Din] W[Din, Dout] for W = Wk
// and W = Wv, in output tiles of 128 rows x 256 columns (M=128, N=256, K=16
// MMAs run at the full tensor rate), X as the K-major and W as the MN-major
// operand, both brought by TMA with 128-byte swizzle. The kernel is
// persistent: the Dout/256 column tiles of a row block form one
// thread-block cluster, and each cluster walks a list of (row block, K or V)
// tiles through a 4-stage ring, with two accumulators in TMEM (256 columns
// each) so that the epilogue of one tile (warps 4-7, one row per thread)
// runs while the MMAs of the next accumulate into the other. The RMSNorm of
// K spans the whole Dout-wide row, i.e. every column tile of the row block:
// the cluster's CTAs exchange their per-row partial sums of squares through
// distributed shared memory, signalling each other with cluster-scope
// mbarriers (double-buffered, so the exchange of one tile overlaps the
// next). The epilogue then normalises, applies gamma and the 3D RoPE pair
// rotation, converts to the cache type (bf16, or E4M3 with a per (token,
// head) scale) and stores.
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
  int M;               // rows per batch entry = n_slots * N
  int B;               // batch entries
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
  static constexpr int STAGES = 4;
  static constexpr int CTRL_BYTES = 4096;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + CTRL_BYTES + 1024;
  static constexpr int TMEM_COLS = 512;         // accumulators at columns 0 and BN
  static constexpr int THREADS = 384;          // warp 0 TMA, warp 1 MMA, warps 4-11 epilogue
  static constexpr int MAX_CLUSTER = 8;         // Dout / BN <= 8
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
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
// Arrive (release, cluster scope) on the mbarrier at the same shared-memory
// offset in cluster CTA `rank`.
__device__ __forceinline__ void mbar_arrive_cluster(uint64_t* bar, uint32_t rank) {
  const uint32_t a = cluster_map(smem_addr(bar), rank);
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(a) : "memory");
}
// mbar_wait with acquire at cluster scope: writes a peer CTA made before its
// release-arrive are visible afterwards. Bounded like every wait.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const uint32_t a = smem_addr(bar);
  const long long t0 = clock64();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
    if (*abort) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      atomicOr(&g_error_word, kErrWaitTimeout);
      *abort = 1;
      return false;
    }
  }
}

// Grid: (C = Dout/256 column tiles = one cluster, G clusters). Cluster g walks
// the contiguous range [g T / G, (g + 1) T / G) of the T = 2 * MB * B tiles
// (t -> kind t % 2 (0: K, 1: V), row block (t / 2) % MB, batch t / (2 MB)),
// so every cluster alternates K and V tiles.
__global__ void __launch_bounds__(384, 1)
    kv_recache_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWk,
                      const __grid_constant__ CUtensorMap tmWv, const RecacheParams p) {
  using TR = RecacheTraits;
  constexpr int BM = TR::BM, BN = TR::BN, BK = TR::BK, ST = TR::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ctrl = smem + ST * TR::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* empty = full + ST;
  uint64_t* acc_full = empty + ST;     // [2] the MMAs of a tile are complete
  uint64_t* acc_empty = acc_full + 2;  // [2] the epilogue has read the accumulator
  uint64_t* ss_full = acc_empty + 2;   // [2] every CTA of the cluster published its partial sums
  uint64_t* ss_empty = ss_full + 2;    // [2] every CTA of the cluster has read them
  uint64_t* drain = ss_empty + 2;      // every MMA issued has completed
  uint64_t* part_ready = drain + 1;    // the second epilogue group's partial sums are in s_part
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(part_ready + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  float* s_ss = reinterpret_cast<float*>(ctrl + 256);          // [2][128] partial sums of squares per row
  float* s_gamma = reinterpret_cast<float*>(ctrl + 1280);      // [256]
  float* s_omega = s_gamma + BN;                               // [BN / D heads][D/2] = 128 floats
  float* s_part = s_omega + BN / 2;                            // [128] second group's partial sums

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = static_cast<int>(gridDim.x);   // cluster size
  const int nt = blockIdx.x;                   // column tile == rank in the cluster
  const int G = static_cast<int>(gridDim.y);
  const int cl = blockIdx.y;
  const int n0 = nt * BN;
  const int kblocks = p.Din / BK;
  const int MB = (p.M + BM - 1) / BM;
  const int ntiles = 2 * MB * p.B;
  const int t_begin = static_cast<int>(static_cast<long long>(cl) * ntiles / G);
  const int t_end = static_cast<int>(static_cast<long long>(cl + 1) * ntiles / G);

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 8);      // one arrival per epilogue warp
      mbar_init(&ss_full[s], 4 * C);    // the first epilogue group's warps of every CTA of the cluster
      mbar_init(&ss_empty[s], 8 * C);   // every epilogue warp of every CTA of the cluster
    }
    mbar_init(drain, 1);
    mbar_init(part_ready, 4);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, TR::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp >= 2 && warp < 4) {  // stage gamma and this column tile's heads' frequencies
    const int tid = threadIdx.x - 64;
    for (int j = tid; j < BN; j += 64) s_gamma[j] = p.gamma[n0 + j];
    const int h0 = n0 / p.D, nh = BN / p.D, P = p.D / 2;
    if (p.rp.enabled)
      for (int j = tid; j < nh * P; j += 64) s_omega[j] = omega_of(p.rp, h0 + j / P, j % P);
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised in every CTA before any remote arrive
  tc_fence_after();
  const uint32_t tbase = *s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmWk);
      tma_prefetch_desc(&tmWv);
      int issued = 0;  // k-blocks issued so far (ring position)
      bool ok = true;
      for (int t = t_begin; ok && t < t_end; ++t) {
        const bool is_k = (t & 1) == 0;
        const int m0 = ((t >> 1) % MB) * BM, b = (t >> 1) / MB;
        const CUtensorMap* tmW = is_k ? &tmWk : &tmWv;
        for (int kb = 0; kb < kblocks; ++kb, ++issued) {
          const int s = issued % ST;
          if (!mbar_wait(&empty[s], ((issued / ST) & 1) ^ 1, s_abort)) { ok = false; break; }
          uint8_t* sa = smem + s * TR::STAGE_BYTES;
          uint8_t* sb = sa + TR::A_BYTES;
          mbar_expect_tx(&full[s], TR::STAGE_BYTES);
          tma_load_3d(sa, &tmX, &full[s], kb * BK, m0, b);
#pragma unroll
          for (int blk = 0; blk < BN / 64; ++blk)
            tma_load_2d(sb + blk * (BK * 128), tmW, &full[s], n0 + blk * 64, kb * BK);
        }
      }
      if (*s_abort)  // let the copies in flight land before the CTA exits
        for (int q = issued - ST > 0 ? issued - ST : 0; q < issued; ++q) mbar_wait_teardown(&full[q % ST], (q / ST) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_dense(BM, BN, 1, false, true);
      const uint32_t a0 = smem_addr(smem);
      const DescWords dA = desc_words(a0, 16, 1024, 2);
      const DescWords dB = desc_words(a0 + TR::A_BYTES, BK * 128, 1024, 2);
      int consumed = 0, j = 0;
      bool ok = true;
      for (int t = t_begin; ok && t < t_end; ++t, ++j) {
        const int acc = j & 1;
        if (!mbar_wait(&acc_empty[acc], ((j >> 1) & 1) ^ 1, s_abort)) break;
        tc_fence_after();
        const uint32_t d = tbase + acc * BN;
        for (int kb = 0; kb < kblocks; ++kb, ++consumed) {
          const int s = consumed % ST;
          if (!mbar_wait(&full[s], (consumed / ST) & 1, s_abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t so = s * TR::STAGE_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16_ss(d, desc_at(dA, so + k * 32), desc_at(dB, so + k * 16 * 128), idesc,
                        (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&acc_full[acc]);
      }
      mma_commit(drain);  // TMEM stays allocated until every MMA issued above is done
      mbar_wait_teardown(drain, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue, one row per thread: warps 4-7 take the
    // first half of the tile's heads, warps 8-11 the second half (the same rows, other TMEM columns)
    const int grp = (warp - 4) >> 2;
    const int row = (threadIdx.x - 128) & 127;
    const int hpg = BN / p.D / 2;  // heads per group
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int P = p.D / 2;
    const int pth = p.rp.pt + p.rp.ph;
    const int gw = p.rp.grid_w > 0 ? p.rp.grid_w : 1;
    int j = 0, kidx = 0;
    bool ok = true;
    for (int t = t_begin; ok && t < t_end; ++t, ++j) {
      const int acc = j & 1;
      const bool is_k = (t & 1) == 0;
      const int m0 = ((t >> 1) % MB) * BM, b = (t >> 1) / MB;
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], (j >> 1) & 1, s_abort));
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr = tbase + lane_off + acc * BN;
      const int tr = m0 + row;
      const bool live = tr < p.M;
      const int slot = live ? tr / p.N : 0;
      const int n = live ? tr - slot * p.N : 0;
      const float pos_t = temporal_pos(p.rp, live ? p.slot_frame[slot] : 0);
      const float pos_r = static_cast<float>(n / gw);
      const float pos_c = static_cast<float>(n % gw);
      const size_t crow = static_cast<size_t>(b) * p.S * p.N + tr;  // cache token row
      float inv_rms = 1.f;
      if (is_k) {
        // partial sum of squares of this row over the tile's 256 columns (each
        // group its half), exchanged with the other column tiles of the row block
        float ss = 0.f;
#pragma unroll 1
        for (int c = 0; c < BN / 64; ++c) {
          uint32_t r[32];
          tmem_load32(taddr + grp * (BN / 2) + c * 32, r);
          tmem_load_wait(r);
#pragma unroll
          for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(r[e]), __uint_as_float(r[e]), ss);
        }
        const int buf = kidx & 1, use = kidx >> 1;
        if (grp == 1) {
          s_part[row] = ss;  // read by group 0 before it publishes, i.e. before this group passes ss_full
          __syncwarp();
          if (lane == 0) mbar_arrive(part_ready);
        } else {
          ok = __all_sync(0xffffffffu, mbar_wait(part_ready, kidx & 1, s_abort));
          if (!ok) break;
          ss += s_part[row];
          // the slot's previous use (two K tiles ago) has been read by every CTA
          if (use > 0) ok = __all_sync(0xffffffffu, mbar_wait_cluster(&ss_empty[buf], (use - 1) & 1, s_abort));
          if (!ok) break;
          s_ss[buf * 128 + row] = ss;
          asm volatile("fence.acq_rel.cluster;" ::: "memory");  // each lane's sum before the warp's arrive
          __syncwarp();
          if (lane == 0)
            for (int r = 0; r < C; ++r) mbar_arrive_cluster(&ss_full[buf], r);
        }
        ok = __all_sync(0xffffffffu, mbar_wait_cluster(&ss_full[buf], use & 1, s_abort));
        if (!ok) break;
        const uint32_t mine = smem_addr(&s_ss[buf * 128 + row]);
        float tot = 0.f;
        for (int r = 0; r < C; ++r) tot += ld_cluster_f32(cluster_map(mine, r));
        __syncwarp();
        if (lane == 0)
          for (int r = 0; r < C; ++r) mbar_arrive_cluster(&ss_empty[buf], r);
        inv_rms = rsqrtf(tot / static_cast<float>(p.Dout) + p.eps);
        ++kidx;
      }
      // accumulator columns [c*32, c*32+32) of head hc -> final values
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
            const int jj = c * 16 + q;  // pair index inside the head
            const float pos = jj < p.rp.pt ? pos_t : (jj < pth ? pos_r : pos_c);
            float sn, cs;
            sincos_reduced(pos * om[jj], sn, cs);
            const float a = x[2 * q], a2 = x[2 * q + 1];
            x[2 * q] = a * cs - a2 * sn;
            x[2 * q + 1] = a * sn + a2 * cs;
          }
        }
      };
      for (int hc = grp * hpg; hc < (grp + 1) * hpg; ++hc) {
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
      // the accumulator may take the next tile's MMAs
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
  }
  // every CTA of the cluster is done with every other one's partial sums
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, TR::TMEM_COLS);
  }
}

}  // namespace ll
