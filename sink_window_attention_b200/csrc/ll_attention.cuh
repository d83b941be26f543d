// ll_attention.cuh — sink-window attention on sm_100a tensor cores.
//
// What it computes (LoL review, "Multi-head attention"; LongLive review,
// "Short-Window Attention" and "Frame Sink"): for every head,
//   O = softmax(RoPE(Q) K^T * scale) V
// over all tokens of the occupied cache slots [0, S_valid), i.e. the 3 sink
// frames plus the most recent local frames; there is no mask inside that set.
//
// How: a flash-style single pass with an online softmax.
//  * one CTA per (query tile of 128 rows, head, batch);
//  * warp 0 (one lane) streams K and V tiles of 128 keys straight out of the
//    [B][S*N][H][D] cache with 4D TMA loads (128-byte swizzle, rows past the
//    valid keys are zero-filled by the TMA unit), STAGES deep; V is the
//    MN-major operand of P V, which for 32-bit (tf32) data needs the 128-byte
//    swizzle with 32-byte atoms;
//  * warp 1 owns the tensor memory (512 columns: two S buffers and O) and one
//    lane issues tcgen05.mma: S_j = Q K_j^T into the free S buffer while the
//    softmax works on the other one, then O += P_j V_j;
//  * warps 4-7 (one TMEM lane quarter each, one query row per thread) read
//    S_j from TMEM, keep the running max / sum, write P_j = exp2(...) to
//    shared memory in the operand layout, rescale O in TMEM only when the
//    running max grows by more than 2^8 (the final division uses the same
//    stale max, so the result is unchanged), and finally normalise O and
//    store it;
//  * Q is loaded by warps 1-7 with plain 128-bit loads, rotated (3D RoPE with
//    the head's jittered temporal base) in registers and written to shared
//    memory in the swizzled layout, so RoPE costs no extra pass over Q.
#pragma once

#include "ll_common.cuh"
#include "ll_rope_append.cuh"

namespace ll {

template <int D_, typename T_>
struct AttnTraits {
  using T = T_;
  static constexpr int D = D_;
  static constexpr int ES = sizeof(T);
  static constexpr int BM = 128;                    // query rows per tile (TMEM lanes)
  static constexpr int BN = 128;                    // keys per KV tile
  static constexpr int ROWB = D * ES;               // bytes of one Q/K/V row
  static constexpr int NB = ROWB / 128;             // 128-byte column blocks per row
  static constexpr int ELEMS_PER_BLOCK = 128 / ES;  // elements of D per column block
  static constexpr int Q_BYTES = BM * ROWB;
  static constexpr int KV_BYTES = BN * ROWB;
  static constexpr int PROWB = BN * ES;             // bytes of one P row
  static constexpr int P_BYTES = BM * PROWB;
  static constexpr int QK_STEPS = ROWB / 32;        // MMAs per S tile (32 bytes of K each)
  static constexpr int PV_STEPS = PROWB / 32;       // MMAs per P V
  static constexpr int MMA_K = 32 / ES;             // reduction elements per MMA
  static constexpr int FMT = (ES == 2) ? 1 : 2;     // bf16 / tf32
  static constexpr int CTRL_BYTES = 1024;
  static constexpr int FIXED_BYTES = Q_BYTES + P_BYTES + CTRL_BYTES + 1024;  // + alignment slack
  static constexpr int NSTAGE = (FIXED_BYTES + 8 * KV_BYTES <= 232448)   ? 4
                                : (FIXED_BYTES + 6 * KV_BYTES <= 232448) ? 3
                                                                         : 2;
  static constexpr int SMEM_BYTES = FIXED_BYTES + 2 * NSTAGE * KV_BYTES;
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL0 = 0, S_COL1 = BN, O_COL = 2 * BN;
  static constexpr int THREADS = 256;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
  static_assert(NB >= 1 && ROWB % 128 == 0, "rows must be whole 128-byte blocks");
};

struct AttnParams {
  const void* q;     // [B][Tq][H][D]
  void* out;         // [B][Tq][H][D]
  float* lse;        // [B][H][Tq] or nullptr
  int B, H, Tq, Nk;  // Nk: valid keys per batch entry
  float softmax_scale;
  RopeParams rp;     // Q rotation (rp.enabled == 0: q already rotated); rp.t_first = first query frame
  int N;             // tokens per frame
};

template <class TR>
__global__ void __launch_bounds__(256, 1)
    sink_window_attention_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                                 const AttnParams p) {
  using T = typename TR::T;
  constexpr int BM = TR::BM, BN = TR::BN, D = TR::D, ST = TR::NSTAGE;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + TR::Q_BYTES;
  uint8_t* sV = sK + ST * TR::KV_BYTES;
  uint8_t* sP = sV + ST * TR::KV_BYTES;
  uint8_t* ctrl = sP + TR::P_BYTES;
  uint64_t* k_full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* v_full = k_full + ST;
  uint64_t* kv_empty = v_full + ST;
  uint64_t* s_full = kv_empty + ST;  // [2]
  uint64_t* p_ready = s_full + 2;
  uint64_t* o_done = p_ready + 1;
  uint64_t* drain = o_done + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  float* s_omega = reinterpret_cast<float*>(ctrl + 512);  // [D/2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int q0 = qt * BM;
  const int nkv = (p.Nk + BN - 1) / BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_ready, BM);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, TR::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int st = j % ST, n = j / ST;
        if (!mbar_wait(&kv_empty[st], (n & 1) ^ 1, s_abort)) break;
        mbar_expect_tx(&k_full[st], TR::KV_BYTES);
#pragma unroll
        for (int blk = 0; blk < TR::NB; ++blk)
          tma_load_4d(sK + st * TR::KV_BYTES + blk * (BN * 128), &tmK, &k_full[st], blk * TR::ELEMS_PER_BLOCK, h,
                      j * BN, b);
        mbar_expect_tx(&v_full[st], TR::KV_BYTES);
#pragma unroll
        for (int blk = 0; blk < TR::NB; ++blk)
          tma_load_4d(sV + st * TR::KV_BYTES + blk * (BN * 128), &tmV, &v_full[st], blk * TR::ELEMS_PER_BLOCK, h,
                      j * BN, b);
        issued = j + 1;
      }
      if (*s_abort) {  // let the copies already in flight land before the CTA exits
        for (int t = issued - ST > 0 ? issued - ST : 0; t < issued; ++t) {
          mbar_wait_teardown(&k_full[t % ST], (t / ST) & 1);
          mbar_wait_teardown(&v_full[t % ST], (t / ST) & 1);
        }
      }
    }
  } else {
    // ------------------------------------------- Q load with fused 3D RoPE (warps 1-7)
    const int tid = threadIdx.x - 32;  // 0..223
    constexpr int NT = 224;
    if (p.rp.enabled) build_omega_one_head(s_omega, p.rp, h, D / 2, tid, NT);
    asm volatile("bar.sync 1, 224;" ::: "memory");
    const T* q = static_cast<const T*>(p.q);
    constexpr int GPR = D / 8;  // 8-element groups per row
    const int pth = p.rp.pt + p.rp.ph;
    for (int g = tid; g < BM * GPR; g += NT) {
      const int r = g / GPR, e8 = g - r * GPR;
      const int t = q0 + r;
      float x[8];
      if (t < p.Tq) {
        load_chunk8<T>(q + ((static_cast<long long>(b) * p.Tq + t) * p.H + h) * D + e8 * 8, x);
        if (p.rp.enabled) {
          const int fi = t / p.N, n = t - fi * p.N;
          const int rr = n / p.rp.grid_w, cc = n - rr * p.rp.grid_w;
          rotate_chunk8(x, e8 * 4, static_cast<float>(p.rp.t_first + fi), static_cast<float>(rr),
                        static_cast<float>(cc), s_omega, p.rp.pt, pth);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = 0.f;
      }
      // 16-byte chunks of this group inside the row, then their swizzled place
      if constexpr (TR::ES == 2) {
        const int chunk = e8;  // 8 bf16 = 16 bytes
        uint4 u;
        u.x = pack_bf16(x[0], x[1]);
        u.y = pack_bf16(x[2], x[3]);
        u.z = pack_bf16(x[4], x[5]);
        u.w = pack_bf16(x[6], x[7]);
        *reinterpret_cast<uint4*>(sQ + (chunk >> 3) * (BM * 128) + sw128_offset(r, chunk & 7)) = u;
      } else {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int chunk = e8 * 2 + hh;  // 4 floats = 16 bytes
          *reinterpret_cast<float4*>(sQ + (chunk >> 3) * (BM * 128) + sw128_offset(r, chunk & 7)) =
              make_float4(x[4 * hh], x[4 * hh + 1], x[4 * hh + 2], x[4 * hh + 3]);
        }
      }
    }
    fence_proxy_async_smem();
    asm volatile("bar.sync 1, 224;" ::: "memory");

    if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        constexpr uint32_t idS = idesc_dense(BM, BN, TR::FMT, false, false);
        constexpr uint32_t idO = idesc_dense(BM, D, TR::FMT, false, true);
        const uint32_t tS[2] = {tbase + TR::S_COL0, tbase + TR::S_COL1};
        const uint32_t tO = tbase + TR::O_COL;
        const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV), aP = smem_addr(sP);
        auto issue_qk = [&](uint32_t d, int st) {
#pragma unroll
          for (int k = 0; k < TR::QK_STEPS; ++k) {
            const uint32_t off = (k >> 2) * (BM * 128) + (k & 3) * 32;
            const uint32_t offk = (k >> 2) * (BN * 128) + (k & 3) * 32;
            const uint64_t da = desc_sw128(aQ + off, 16, 1024);
            const uint64_t db = desc_sw128(aK + st * TR::KV_BYTES + offk, 16, 1024);
            if constexpr (TR::ES == 2) mma_bf16_ss(d, da, db, idS, k > 0 ? 1u : 0u);
            else mma_tf32_ss(d, da, db, idS, k > 0 ? 1u : 0u);
          }
        };
        auto issue_pv = [&](int st, bool acc) {
#pragma unroll
          for (int k = 0; k < TR::PV_STEPS; ++k) {
            const uint32_t offp = (k >> 2) * (BM * 128) + (k & 3) * 32;
            const uint64_t da = desc_sw128(aP + offp, 16, 1024);
            const uint32_t av = aV + st * TR::KV_BYTES + k * TR::MMA_K * 128;
            if constexpr (TR::ES == 2) {
              mma_bf16_ss(tO, da, desc_sw128(av, BN * 128, 1024), idO, (acc || k > 0) ? 1u : 0u);
            } else {
              mma_tf32_ss(tO, da, desc_mn_sw128_atom32(av, BN * 128, 512), idO, (acc || k > 0) ? 1u : 0u);
            }
          }
        };
        if (mbar_wait(&k_full[0], 0, s_abort)) {
          tc_fence_after();
          issue_qk(tS[0], 0);
          mma_commit(&s_full[0]);
          for (int j = 0; j < nkv; ++j) {
            if (j + 1 < nkv) {
              const int st1 = (j + 1) % ST;
              if (!mbar_wait(&k_full[st1], ((j + 1) / ST) & 1, s_abort)) break;
              tc_fence_after();
              issue_qk(tS[(j + 1) & 1], st1);
              mma_commit(&s_full[(j + 1) & 1]);
            }
            if (!mbar_wait(p_ready, j & 1, s_abort)) break;
            const int st = j % ST;
            if (!mbar_wait(&v_full[st], (j / ST) & 1, s_abort)) break;
            tc_fence_after();
            issue_pv(st, j > 0);
            mma_commit(o_done);
            mma_commit(&kv_empty[st]);
          }
        }
        // every MMA issued above has finished once `drain` completes
        mma_commit(drain);
        mbar_wait_teardown(drain, 0);
      }
    } else if (warp >= 4) {
      // ------------------------------------------------ softmax / correction / epilogue
      const int row = threadIdx.x - 128;           // 0..127 == TMEM lane
      const uint32_t lane_off = static_cast<uint32_t>((warp - 4) * 32) << 16;
      const float scale = p.softmax_scale > 0.f ? p.softmax_scale : rsqrtf(static_cast<float>(D));
      const float sl2 = scale * 1.4426950408889634f;
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int j = 0; j < nkv && ok; ++j) {
        // tcgen05.ld is warp-collective: every lane must agree before using it
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[j & 1], (j >> 1) & 1, s_abort))) { ok = false; break; }
        tc_fence_after();
        const uint32_t tS = tbase + lane_off + ((j & 1) ? TR::S_COL1 : TR::S_COL0);
        uint32_t sr[BN / 32][32];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_load32(tS + c * 32, sr[c]);
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_load_wait(sr[c]);
        const int kv_valid = p.Nk - j * BN;
        float mx = -INFINITY;
        if (kv_valid >= BN) {
#pragma unroll
          for (int c = 0; c < BN / 32; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(sr[c][e]));
        } else {
#pragma unroll
          for (int c = 0; c < BN / 32; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (c * 32 + e >= kv_valid) sr[c][e] = __float_as_uint(-INFINITY);
              mx = fmaxf(mx, __uint_as_float(sr[c][e]));
            }
        }
        const float m_new = mx * sl2;
        float m_use = m_run;
        bool rescale = false;
        if (m_new > m_run + 8.0f) {
          m_use = m_new;
          rescale = (j > 0);
        }
        // P buffer and O are free once the previous P V has completed
        if (j > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, s_abort))) { ok = false; break; }
          tc_fence_after();
        }
        // tcgen05.ld/st are warp-collective: the warp rescales together when any
        // of its rows needs it; rows that do not scale by 1
        if (__any_sync(0xffffffffu, rescale)) {
          const float alpha = rescale ? ex2(m_run - m_use) : 1.0f;
          l_run *= alpha;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_load32(tbase + lane_off + TR::O_COL + c * 32, o);
            tmem_load_wait(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_store32(tbase + lane_off + TR::O_COL + c * 32, o);
          }
          tmem_store_wait();
        }
        m_run = m_use;
        const float neg_m = -m_use;
        float lsum = 0.f;
        if constexpr (TR::ES == 2) {
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {  // 8 probabilities -> one 16-byte chunk
              float pv[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                pv[e] = ex2(fmaf(__uint_as_float(sr[c][g * 8 + e]), sl2, neg_m));
                lsum += pv[e];
              }
              uint4 u;
              u.x = pack_bf16(pv[0], pv[1]);
              u.y = pack_bf16(pv[2], pv[3]);
              u.z = pack_bf16(pv[4], pv[5]);
              u.w = pack_bf16(pv[6], pv[7]);
              const int chunk = c * 4 + g;  // 16-byte chunk index within the P row
              *reinterpret_cast<uint4*>(sP + (chunk >> 3) * (BM * 128) + sw128_offset(row, chunk & 7)) = u;
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
#pragma unroll
            for (int g = 0; g < 8; ++g) {  // 4 probabilities -> one 16-byte chunk
              float pv[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                pv[e] = ex2(fmaf(__uint_as_float(sr[c][g * 4 + e]), sl2, neg_m));
                lsum += pv[e];
              }
              const int chunk = c * 8 + g;
              *reinterpret_cast<float4*>(sP + (chunk >> 3) * (BM * 128) + sw128_offset(row, chunk & 7)) =
                  make_float4(pv[0], pv[1], pv[2], pv[3]);
            }
          }
        }
        l_run += lsum;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_ready);
      }
      if (ok && __all_sync(0xffffffffu, mbar_wait(o_done, (nkv - 1) & 1, s_abort))) {
        tc_fence_after();
        const int t = q0 + row;
        const float inv_l = 1.0f / l_run;
        T* out = static_cast<T*>(p.out);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_load32(tbase + lane_off + TR::O_COL + c * 32, o);
          tmem_load_wait(o);
          if (t < p.Tq) {
            T* dst = out + ((static_cast<long long>(b) * p.Tq + t) * p.H + h) * D + c * 32;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              float x[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(o[g * 8 + e]) * inv_l;
              store_chunk8<T>(dst + g * 8, x);
            }
          }
        }
        if (p.lse != nullptr && t < p.Tq)
          p.lse[(static_cast<long long>(b) * p.H + h) * p.Tq + t] = (m_run + log2f(l_run)) * 0.6931471805599453f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, TR::TMEM_COLS);
  }
}

}  // namespace ll
