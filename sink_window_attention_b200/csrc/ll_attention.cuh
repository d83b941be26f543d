// ll_attention.cuh — sink-window attention on sm_100a tensor cores.
//
// What it computes (LoL review, "Multi-head attention"; LongLive review,
// "Short-Window Attention" and "Frame Sink"): for every head,
//   O = softmax(RoPE(Q) K^T * scale) V
// over all tokens of the occupied cache slots [0, S_valid), i.e. the 3 sink
// frames plus the most recent local frames; there is no mask inside that set.
//
// How (flash-style single pass, online softmax in the exp2 domain):
//  * Work is a list of units = (128-row query tile, head, batch), each with
//    nkv tiles of 128 keys. A persistent grid of G CTAs (G = #SMs) splits the
//    flattened (unit, key tile) range into G equal contiguous ranges, so every
//    SM gets the same number of key tiles; a CTA processes its range as pieces
//    (one piece per unit it touches). A piece that covers a whole unit writes
//    O directly; otherwise it writes its unnormalised (O, m, l) to a workspace
//    slot and the CTA that finishes a unit's last piece merges all of them.
//  * warp 0 (one lane) streams K tiles and V tiles straight out of the
//    [B][S*N][H][D] cache with 4D TMA loads (128-byte swizzle; rows past the
//    valid keys read as zeros). K and V have rings and cursors of their own,
//    each refilled as soon as a stage frees, so K runs ahead of V.
//  * Q tiles come in by TMA (the same swizzled operand layout, rows past the
//    query count zero-filled) into a double buffer; warps 2-3 then apply the
//    3D RoPE in place in shared memory (angles reduced to [-pi, pi], then the
//    hardware sine/cosine), so RoPE costs no extra pass over Q in HBM.
//  * warp 1 owns 512 TMEM columns: S_A, S_B (128 each) and O_A, O_B. One lane
//    issues tcgen05.mma: S_i = Q K_i^T into S_(i mod 2) and O_(i mod 2) +=
//    P_i V_i, where P_i sits in the TMEM columns of S_i (the A operand is read
//    from tensor memory), so P never touches shared memory.
//  * two softmax warpgroups (warps 4-7: even key tiles of a piece, warps 8-11:
//    odd ones; one query row per thread, one TMEM lane quarter per warp) keep
//    independent running (max, sum) and O; O is rescaled in TMEM only when the
//    running max grows by more than 2^8 (the final division uses the same max,
//    so the result is unchanged). At the end of a piece warpgroup A merges
//    the two halves.
//  * Every mbarrier wait is bounded; a wait that gives up records an error,
//    raises an abort flag the other roles see, and all roles still walk the
//    same named-barrier sequence so nothing can hang. TMEM accesses
//    (warp-collective) only run under warp-uniform conditions.
#pragma once

#include <type_traits>

#include "ll_common.cuh"
#include "ll_rope_append.cuh"

namespace ll {

// Marks the attention variant over an E4M3 cache on the FP8 tensor cores:
// the bf16 Q tile is quantised to E4M3 (one scale per tile) in shared memory,
// K and V arrive as E4M3 codes with their per-(token, head) scales, and
// S = Q K^T and O += P' V run as kind::f8f6f4 MMAs.
struct E4M3Kv {};

template <int D_, typename T_>
struct AttnTraits {
  static constexpr bool FP8 = std::is_same<T_, E4M3Kv>::value;
  using T = typename std::conditional<FP8, __nv_bfloat16, T_>::type;  // Q and O
  static constexpr int D = D_;
  static constexpr int ES = FP8 ? 1 : static_cast<int>(sizeof(T));  // bytes per MMA operand element
  static constexpr int BM = 128;                    // query rows per tile (TMEM lanes)
  static constexpr int BN = 128;                    // keys per KV tile
  static constexpr int ROWB = D * ES;               // bytes of one Q/K/V operand row
  static constexpr int NB = ROWB / 128;             // 128-byte column blocks per row
  static constexpr int ELEMS_PER_BLOCK = 128 / ES;  // elements of D per column block
  static constexpr int Q_BYTES = BM * ROWB;         // one Q operand tile
  static constexpr int QSTG_BYTES = FP8 ? BM * D * 2 : 0;  // bf16 tile that the E4M3 Q is quantised from
  static constexpr int KV_BYTES = BN * ROWB;
  static constexpr int SC_BYTES = FP8 ? 2 * BN * 16 : 0;  // K and V scale boxes ([BN][4 heads] fp32) per V stage
  static constexpr int VSTAGE_BYTES = KV_BYTES + SC_BYTES;
  static constexpr int QK_STEPS = ROWB / 32;        // MMAs per S tile (32 bytes of K each)
  static constexpr int PV_STEPS = BN * ES / 32;     // MMAs per P V (8 bf16 / 16 tf32 / 4 e4m3)
  static constexpr int MMA_K = 32 / ES;             // reduction elements per MMA
  static constexpr int FMT = FP8 ? 0 : (ES == 2) ? 1 : 2;  // e4m3 / bf16 / tf32
  static constexpr int QST = 2;                     // Q buffers
  static constexpr int CTRL_BYTES = 2048;
  static constexpr int STAGE_BUDGET = 232448 - CTRL_BYTES - 1024 - QST * Q_BYTES - QSTG_BYTES;
  static constexpr int STAGES = STAGE_BUDGET / KV_BYTES;
  static constexpr int KST = FP8 ? 4 : STAGES >= 8 ? 4 : (STAGES + 1) / 2;
  static constexpr int VST = FP8 ? 4 : STAGES >= 8 ? 4 : STAGES - KST;
  static constexpr int SMEM_BYTES =
      CTRL_BYTES + 1024 + QST * Q_BYTES + QSTG_BYTES + KST * KV_BYTES + VST * VSTAGE_BYTES;
  static constexpr int TMEM_COLS = 512;
  static constexpr int S_COL0 = 0, O_COL0 = 2 * BN;  // S_w at w*BN, O_w at O_COL0 + w*D
  static constexpr int THREADS = 384;
  // register split: launch 168 per thread (384 x 168 = 64512); warpgroup 0
  // (producer, MMA, Q loader) gives up 96 per thread, the two softmax
  // warpgroups take 48 more: 128 x 72 + 256 x 216 = 64512. The build checks
  // that ptxas allocated exactly LAUNCH_REGS.
  static constexpr int LAUNCH_REGS = 168, REGS_LOW = 72, REGS_HIGH = 216;
  static_assert(128 * REGS_LOW + 256 * REGS_HIGH <= THREADS * LAUNCH_REGS, "register split exceeds the launch");
  // One partial: O chunk-major ([D/4][BM] float4, so that the 32 rows of a
  // warp read and write 512 contiguous bytes per chunk), then m, then l.
  static constexpr int SLOT_FLOATS = BM * D + 2 * BM;
  static_assert(KST >= 2 && VST >= 2, "need at least two K and two V stages");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(O_COL0 + 2 * D <= TMEM_COLS, "TMEM budget");
  static_assert(NB >= 1 && ROWB % 128 == 0, "rows must be whole 128-byte blocks");
  static_assert(!FP8 || D == 128, "the E4M3 variant is written for D = 128 (one 128-byte row)");
  static_assert(VSTAGE_BYTES % 1024 == 0 && QSTG_BYTES % 1024 == 0, "1024-byte aligned buffers");
};

struct AttnParams {
  const void* q;     // [B][Tq][H][D]
  void* out;         // [B][Tq][H][D]
  float* lse;        // [B][H][Tq] or nullptr
  int B, H, Tq, Nk;  // Nk: valid keys per batch entry
  int N;             // tokens per frame
  float softmax_scale;
  RopeParams rp;     // Q rotation (rp.enabled == 0: q already rotated); rp.t_first = first query frame
  int q_tiles;       // ceil(Tq / 128)
  int nkv;           // ceil(Nk / 128)
  int units;         // q_tiles * H * B
  int grid;          // G: number of CTAs
  long long total;   // units * nkv
  int* counters;     // [units] arrivals per unit (zeroed by the host before the launch)
  float* partials;   // [(grid + units) * SLOT_FLOATS]
  // Fused append (ll_append_and_attend): every CTA first writes its share of
  // the new frames' K/V into the cache, then all CTAs meet at a grid barrier
  // (cooperative launch: all CTAs are co-resident) before any K/V is read.
  int fuse_append;
  unsigned int gen;                // generation tag of this launch in the barrier word
  unsigned long long* grid_bar;    // [generation:32 | arrivals:32]
  AppendParams ap;                 // the append (input dtype = cache dtype = T)
  // E4M3 variant: the largest V scale of each (batch, head) over the valid
  // keys ([B][H], from a pass before the launch); it fixes the power-of-two
  // shift of the reference max that keeps P' = p * scale_v inside E4M3's range
  const float* v_scale_max;
};

// A piece: key tiles [j0, j0 + n) of unit u.
struct Piece {
  int u, j0, n;
};

// CTA that owns flattened iteration i when `total` iterations are split into
// G contiguous ranges starting at floor(g * total / G).
__device__ __forceinline__ int owner_of(long long i, long long total, int G) {
  return static_cast<int>(((i + 1) * G - 1) / total);
}

// Q tile of unit u, rotated with this head's frequencies `om` [D/2], into
// the 128-byte-swizzled K-major operand layout at sQ.
// Apply the 3D RoPE in place to a Q tile that TMA has put into shared memory
// (128-byte swizzled, K-major: the operand layout the MMA reads). Rows past
// Tq were zero-filled by TMA and stay zero. Each thread takes 8-element
// groups; rotation in fp32, rounded back to the tile's type.
template <class TR>
__device__ __forceinline__ void rope_q_tile_inplace(uint8_t* sQ, const AttnParams& p, const float* om, int u, int tid,
                                                    int nthreads) {
  using T = typename TR::T;
  constexpr int BM = TR::BM, D = TR::D;
  constexpr int GPR = D / 8;  // 8-element groups per row
  const int q0 = (u % p.q_tiles) * BM;
  const int pth = p.rp.pt + p.rp.ph;
  for (int g = tid; g < BM * GPR; g += nthreads) {
    const int r = g / GPR, e8 = g - r * GPR;
    const int t = q0 + r;
    if (t >= p.Tq) continue;
    const int fi = t / p.N, n = t - fi * p.N;
    const int rr = n / p.rp.grid_w, cc = n - rr * p.rp.grid_w;
    float x[8];
    if constexpr (TR::ES == 2) {
      uint4* ptr = reinterpret_cast<uint4*>(sQ + (e8 >> 3) * (BM * 128) + sw128_offset(r, e8 & 7));
      const uint4 v = *ptr;
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
      }
      rotate_chunk8(x, e8 * 4, temporal_pos(p.rp, fi), static_cast<float>(rr),
                    static_cast<float>(cc), om, p.rp.pt, pth);
      *ptr = make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
    } else {
      float4* p0 = reinterpret_cast<float4*>(sQ + ((2 * e8) >> 3) * (BM * 128) + sw128_offset(r, (2 * e8) & 7));
      float4* p1 = reinterpret_cast<float4*>(sQ + ((2 * e8 + 1) >> 3) * (BM * 128) + sw128_offset(r, (2 * e8 + 1) & 7));
      const float4 a = *p0, b = *p1;
      x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
      x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
      rotate_chunk8(x, e8 * 4, temporal_pos(p.rp, fi), static_cast<float>(rr),
                    static_cast<float>(cc), om, p.rp.pt, pth);
      *p0 = make_float4(x[0], x[1], x[2], x[3]);
      *p1 = make_float4(x[4], x[5], x[6], x[7]);
    }
  }
  fence_proxy_async_smem();  // the generic-proxy writes are read by the tensor core
}

// E4M3 variant: quantise the bf16 Q tile in `stage` (RoPE already applied;
// 128-byte swizzled K-major, D/64 column blocks) into the E4M3 operand tile
// `q8` (one 128-byte block per row, same swizzle) with one scale per tile:
// scale = max|q| / 448 (1 for a zero tile), codes = RNE(q / scale) saturated.
// Threads tid 0..nthreads-1 synchronise on named barrier `bar`; every thread
// passes both barriers whatever `active` says (a thread whose wait gave up
// passes inactive), so the barrier counts always match. `amax_word` is a
// shared word this call may overwrite.
template <class TR>
__device__ __forceinline__ void quantize_q_tile(const uint8_t* stage, uint8_t* q8, float* scale_out,
                                                unsigned int* amax_word, int tid, int nthreads, int bar, bool active) {
  constexpr int BM = TR::BM, D = TR::D;
  if (tid == 0) *amax_word = 0u;
  asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(nthreads) : "memory");
  float amax = 0.f;
  for (int g = active ? tid : BM * (D / 8); g < BM * (D / 8); g += nthreads) {
    const int r = g / (D / 8), e8 = g - r * (D / 8);
    const uint4 v = *reinterpret_cast<const uint4*>(stage + (e8 >> 3) * (BM * 128) + sw128_offset(r, e8 & 7));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      amax = fmax3(amax, fabsf(f.x), fabsf(f.y));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((tid & 31) == 0) atomicMax(amax_word, __float_as_uint(amax));  // non-negative floats order as integers
  asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(nthreads) : "memory");
  const float tmax = __uint_as_float(*amax_word);
  const float sc = tmax > 0.f ? tmax / 448.0f : 1.0f;
  const float inv = 1.0f / sc;
  for (int g = active ? tid : BM * (D / 16); g < BM * (D / 16); g += nthreads) {
    const int r = g / (D / 16), c = g - r * (D / 16);  // output chunk c: elements 16c .. 16c + 15
    uint32_t out[4];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int e8 = 2 * c + half;
      const uint4 v = *reinterpret_cast<const uint4*>(stage + (e8 >> 3) * (BM * 128) + sw128_offset(r, e8 & 7));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[2 * i]));
        const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[2 * i + 1]));
        const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(f0.x * inv, f0.y * inv), __NV_SATFINITE, __NV_E4M3);
        const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(f1.x * inv, f1.y * inv), __NV_SATFINITE, __NV_E4M3);
        out[2 * half + i] = lo | (hi << 16);
      }
    }
    *reinterpret_cast<uint4*>(q8 + sw128_offset(r, c)) = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (tid == 0) *scale_out = sc;
  fence_proxy_async_smem();  // the generic-proxy writes are read by the tensor core
}

// TMA copy of the Q tile of unit u into a Q buffer (NB column blocks of 128
// bytes x BM rows; rows past Tq read as zeros). One thread.
template <class TR>
__device__ __forceinline__ void tma_q_tile(uint8_t* dst, const CUtensorMap* tmQ, uint64_t* bar, const AttnParams& p,
                                           int u) {
  const int qt = u % p.q_tiles, h = (u / p.q_tiles) % p.H, b = u / (p.q_tiles * p.H);
  mbar_expect_tx(bar, TR::Q_BYTES);
#pragma unroll
  for (int blk = 0; blk < TR::NB; ++blk)
    tma_load_4d(dst + blk * (TR::BM * 128), tmQ, bar, blk * TR::ELEMS_PER_BLOCK, h, qt * TR::BM, b);
}

template <class TR>
__global__ void __launch_bounds__(384, 1)
    sink_window_attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKS,
                                 const __grid_constant__ CUtensorMap tmVS, const AttnParams p) {
  using T = typename TR::T;
  // the Q tile as loaded: bf16 staging for the E4M3 variant, else the operand itself
  using QTR = typename std::conditional<TR::FP8, AttnTraits<TR::D, __nv_bfloat16>, TR>::type;
  constexpr int BM = TR::BM, BN = TR::BN, D = TR::D, KST = TR::KST, VST = TR::VST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                              // [QST][Q_BYTES]
  uint8_t* sQs = sQ + TR::QST * TR::Q_BYTES;       // [QSTG_BYTES] bf16 Q tile (E4M3 variant)
  uint8_t* sK = sQs + TR::QSTG_BYTES;              // [KST][KV_BYTES]
  uint8_t* sV = sK + KST * TR::KV_BYTES;           // [VST][VSTAGE_BYTES]: V tile (+ K and V scale boxes)
  uint8_t* ctrl = sV + VST * TR::VSTAGE_BYTES;
  uint64_t* k_full = reinterpret_cast<uint64_t*>(ctrl);
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + VST;
  uint64_t* q_full = v_empty + VST;   // [2]
  uint64_t* q_empty = q_full + 2;     // [2]
  uint64_t* s_full = q_empty + 2;     // [2] per softmax warpgroup
  uint64_t* p_ready = s_full + 2;     // [2]
  uint64_t* o_done = p_ready + 2;     // [2]
  uint64_t* b_ready = o_done + 2;     // warpgroup B's piece state is in smem
  uint64_t* merged = b_ready + 1;     // warpgroup A has read O_A, O_B of the piece
  uint64_t* drain = merged + 1;
  uint64_t* q_tma = drain + 1;        // [2] TMA copy of a Q tile landed
  uint64_t* ap_bar = q_tma + 2;       // fused append: this CTA's K/V rows landed in shared memory
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(ap_bar + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  volatile int* s_last = reinterpret_cast<volatile int*>(s_tmem + 2);
  float* s_mB = reinterpret_cast<float*>(ctrl + 384);      // [128]
  float* s_lB = s_mB + BM;                                 // [128]
  float* s_omega = reinterpret_cast<float*>(ctrl + 1408);  // [2][D/2]: one head per Q buffer
  float* s_qscale = reinterpret_cast<float*>(ctrl + 1920);  // [2] E4M3 variant: scale of each Q buffer
  unsigned int* s_qamax = reinterpret_cast<unsigned int*>(ctrl + 1928);
  static_assert(1408 + 2 * (D / 2) * 4 <= 1920 && 1932 <= TR::CTRL_BYTES, "control block layout");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x;
  const long long it_begin = g * p.total / p.grid;
  const long long it_end = (g + 1) * p.total / p.grid;

  if (threadIdx.x == 0) {
    for (int s = 0; s < KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_ready[s], BM);
      mbar_init(&o_done[s], 1);
    }
    mbar_init(b_ready, BM);
    mbar_init(merged, BM);
    mbar_init(drain, 1);
    mbar_init(&q_tma[0], 1);
    mbar_init(&q_tma[1], 1);
    mbar_init(ap_bar, 1);
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

  // The piece sequence of this CTA, walked identically by every role.
  auto next_piece = [&](long long& it, Piece& pc) -> bool {
    if (it >= it_end) return false;
    pc.u = static_cast<int>(it / p.nkv);
    pc.j0 = static_cast<int>(it - static_cast<long long>(pc.u) * p.nkv);
    const long long left = it_end - it;
    pc.n = static_cast<int>(left < p.nkv - pc.j0 ? left : p.nkv - pc.j0);
    it += pc.n;
    return true;
  };

  // The first piece's Q tile comes in by TMA; warps 2-11 rotate it together
  // (the softmax warpgroups have nothing to do before it). Later pieces:
  // warps 2-3. With a fused append, the whole CTA first writes its share of
  // the new frames into the cache while that Q copy is in flight.
  {
    long long it0 = it_begin;
    Piece pc0;
    next_piece(it0, pc0);
    if (threadIdx.x == 64) tma_q_tile<QTR>(TR::FP8 ? sQs : sQ, &tmQ, &q_tma[0], p, pc0.u);
    if (!TR::FP8 && p.fuse_append) {
      // This CTA's contiguous share of the new frames' tokens (all batch
      // entries): their K and V rows come into the K/V stage buffers (which
      // TMA fills only after the barrier) by bulk copies, K is rotated in
      // shared memory, and bulk stores write both into the frames' cache
      // slots. The frequency tables live in the second Q buffer, which the Q
      // loader fills only after this prologue.
      const AppendParams& ap = p.ap;
      float* s_aom = reinterpret_cast<float*>(sQ + TR::Q_BYTES);
      float* s_atc = s_aom + ap.H * (ap.D / 2);
      const int RB = ap.H * ap.D * static_cast<int>(sizeof(T));  // bytes of one token row
      const int FN = ap.F * ap.N, S = ap.n_sink + ap.n_local;
      const int ttot = ap.B * FN;
      const int t0 = static_cast<int>(static_cast<long long>(g) * ttot / p.grid);
      const int t1 = static_cast<int>(static_cast<long long>(g + 1) * ttot / p.grid);
      const int R = (KST + VST) * TR::KV_BYTES / (2 * RB);  // tokens per round (K half, then V half)
      uint8_t* sKr = sK;                                     // [R][H][D] K rows
      uint8_t* sVr = sK + static_cast<size_t>(R) * RB;      // [R][H][D] V rows
      const T* kin = static_cast<const T*>(ap.k_in);
      const T* vin = static_cast<const T*>(ap.v_in);
      T* kc = static_cast<T*>(ap.k_cache);
      T* vc = static_cast<T*>(ap.v_cache);
      // the pieces of [r0, r0 + n) that are contiguous in the cache: one (batch, frame) each
      auto for_segments = [&](int r0, int n, auto&& fn) {
        for (int r = r0; r < r0 + n;) {
          const int b = r / FN, rem = r - b * FN, fi = rem / ap.N, nn = rem - fi * ap.N;
          const int len = min(ap.N - nn, r0 + n - r);
          const long long crow = (static_cast<long long>(b) * S + cache_slot(ap.first_frame + fi, ap.n_sink,
                                                                             ap.n_local)) * ap.N + nn;
          fn(r - r0, static_cast<long long>(r), crow, len);
          r += len;
        }
      };
      int round = 0;
      for (int r0 = t0; r0 < t1; r0 += R, ++round) {
        const int n = min(R, t1 - r0);
        if (threadIdx.x == 0) {
          mbar_expect_tx(ap_bar, 2u * static_cast<uint32_t>(n) * RB);
          bulk_load(sKr, kin + static_cast<size_t>(r0) * ap.H * ap.D, static_cast<uint32_t>(n) * RB, ap_bar);
          bulk_load(sVr, vin + static_cast<size_t>(r0) * ap.H * ap.D, static_cast<uint32_t>(n) * RB, ap_bar);
        }
        if (round == 0 && ap.rp.enabled) build_append_tables(s_aom, s_atc, ap);  // while the rows are in flight
        const bool landed = mbar_wait(ap_bar, round & 1, s_abort);
        if (landed && ap.rp.enabled) {
          const int hg = append_heads_per_thread(ap.H), cpr = ap.D / 8, per_tok = (ap.H / hg) * cpr;
          for (int i = threadIdx.x; i < n * per_tok; i += blockDim.x) {
            const int tl = i / per_tok, rem = i - tl * per_tok;
            const int grp = rem / cpr;
            const int tg = (r0 + tl) % FN;  // token within the batch entry's new frames
            AppendItem ai;
            ai.c = rem - grp * cpr;
            ai.h0 = grp * hg;
            ai.fi = tg / ap.N;
            ai.n = tg - ai.fi * ap.N;
            T* row = reinterpret_cast<T*>(sKr + static_cast<size_t>(tl) * RB);
            float kx[kAppendMaxHg][8];
#pragma unroll
            for (int k = 0; k < kAppendMaxHg; ++k)
              if (k < hg) load_chunk8<T>(row + (ai.h0 + k) * ap.D + ai.c * 8, kx[k]);
            append_rotate(ap, ai, s_aom, s_atc, kx);
#pragma unroll
            for (int k = 0; k < kAppendMaxHg; ++k)
              if (k < hg) store_chunk8<T>(row + (ai.h0 + k) * ap.D + ai.c * 8, kx[k]);
          }
        }
        if (!landed && threadIdx.x == 0) mbar_wait_teardown(ap_bar, round & 1);  // the copies must land
        fence_proxy_async_smem();  // the rotated rows are read by the bulk stores (async proxy)
        __syncthreads();
        if (threadIdx.x == 0) {
          if (landed)
            for_segments(r0, n, [&](int off, long long, long long crow, int len) {
              bulk_store(kc + crow * ap.H * ap.D, sKr + static_cast<size_t>(off) * RB, static_cast<uint32_t>(len) * RB);
              bulk_store(vc + crow * ap.H * ap.D, sVr + static_cast<size_t>(off) * RB, static_cast<uint32_t>(len) * RB);
            });
          bulk_store_commit_wait();  // complete before the rows are reused or the barrier is passed
        }
        if (r0 + R < t1) __syncthreads();  // the next round reuses the buffers
      }
      // Every thread's shared-memory writes (rows, tables) were fenced for the
      // async proxy before the last round's bulk stores, and thread 0 alone
      // wrote global memory (those stores, complete). Thread 0 fences them for
      // the other CTAs' TMA reads and meets those CTAs at the grid barrier; it
      // then issues every K/V load into the stage buffers that held the rows.
      // The Q loader, which refills the buffer that held the tables, passed
      // the last round's block barrier after every access to them. The other
      // warps go on meanwhile: the first Q tile's RoPE needs nothing from the
      // append.
      if (threadIdx.x == 0) {
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
        grid_barrier(p.grid_bar, p.gen, static_cast<unsigned int>(p.grid), s_abort);
      }
      __syncwarp();  // warp 0 reconverges before its setmaxnreg
    }
    if (warp >= 2) {
      const int tid = threadIdx.x - 64;  // 0..319
      if (p.rp.enabled)
        for (int j = tid; j < D / 2; j += 320) s_omega[j] = omega_of(p.rp, (pc0.u / p.q_tiles) % p.H, j);
      asm volatile("bar.sync 4, 320;" ::: "memory");
      const bool landed = mbar_wait(&q_tma[0], 0, s_abort);
      if (landed && p.rp.enabled) rope_q_tile_inplace<QTR>(TR::FP8 ? sQs : sQ, p, s_omega, pc0.u, tid, 320);
      if (!landed && tid == 0) mbar_wait_teardown(&q_tma[0], 0);  // the copy must land before the CTA exits
      asm volatile("bar.sync 4, 320;" ::: "memory");
      if constexpr (TR::FP8) {
        quantize_q_tile<TR>(sQs, sQ, &s_qscale[0], s_qamax, tid, 320, 4, landed);
        asm volatile("bar.sync 4, 320;" ::: "memory");
      }
      if (tid == 0) mbar_arrive(&q_full[0]);
    }
  }

  if (warp < 4) {
  // warpgroup 0: producer, MMA issuer, Q loader (same setmaxnreg for its four warps)
  regs_dec<TR::REGS_LOW>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      if constexpr (TR::FP8) {
        tma_prefetch_desc(&tmKS);
        tma_prefetch_desc(&tmVS);
      }
      if (p.fuse_append) asm volatile("fence.proxy.async.global;" ::: "memory");  // see the append above
      // K and V walk the same tile sequence with cursors of their own; each
      // is loaded as soon as its ring has a free stage, so K runs ahead of V
      // by as many tiles as its ring holds
      long long itK = it_begin, itV = it_begin;
      Piece pk, pv;
      int ik = 0, iv = 0;            // tile within the current piece
      bool hk = next_piece(itK, pk), hv = next_piece(itV, pv);
      int kc = 0, vc = 0;            // K / V tiles issued so far
      long long idle_since = 0;
      int polls = 0;
      while (hk || hv) {
        bool progressed = false;
        if (hk && mbar_test(smem_addr(&k_empty[kc % KST]), ((kc / KST) & 1) ^ 1)) {
          const int st = kc % KST;
          const int h = (pk.u / p.q_tiles) % p.H, b = pk.u / (p.q_tiles * p.H);
          mbar_expect_tx(&k_full[st], TR::KV_BYTES);
#pragma unroll
          for (int blk = 0; blk < TR::NB; ++blk)
            tma_load_4d(sK + st * TR::KV_BYTES + blk * (BN * 128), &tmK, &k_full[st], blk * TR::ELEMS_PER_BLOCK, h,
                        (pk.j0 + ik) * BN, b);
          ++kc;
          if (++ik == pk.n) {
            ik = 0;
            hk = next_piece(itK, pk);
          }
          progressed = true;
        }
        if (hv && mbar_test(smem_addr(&v_empty[vc % VST]), ((vc / VST) & 1) ^ 1)) {
          const int st = vc % VST;
          const int h = (pv.u / p.q_tiles) % p.H, b = pv.u / (p.q_tiles * p.H);
          mbar_expect_tx(&v_full[st], TR::VSTAGE_BYTES);
#pragma unroll
          for (int blk = 0; blk < TR::NB; ++blk)
            tma_load_4d(sV + st * TR::VSTAGE_BYTES + blk * (BN * 128), &tmV, &v_full[st], blk * TR::ELEMS_PER_BLOCK,
                        h, (pv.j0 + iv) * BN, b);
          if constexpr (TR::FP8) {
            // the tile's K and V scales ride with the V tile: [BN keys][4 heads]
            // fp32 boxes from head h rounded down to a multiple of 4 (so that
            // the box's x coordinate is 16-byte aligned)
            uint8_t* sc = sV + st * TR::VSTAGE_BYTES + TR::KV_BYTES;
            tma_load_3d(sc, &tmKS, &v_full[st], h & ~3, (pv.j0 + iv) * BN, b);
            tma_load_3d(sc + BN * 16, &tmVS, &v_full[st], h & ~3, (pv.j0 + iv) * BN, b);
          }
          ++vc;
          if (++iv == pv.n) {
            iv = 0;
            hv = next_piece(itV, pv);
          }
          progressed = true;
        }
        if (progressed) {
          idle_since = 0;
          polls = 0;
        } else {
          __nanosleep(32);
          if (++polls >= 16) {  // bounded: give up if no stage frees for ~1 s
            polls = 0;
            if (*s_abort) break;
            const long long now = clock64();
            if (idle_since == 0) idle_since = now;
            else if (now - idle_since > kWaitLimitCycles) {
              atomicOr(&g_error_word, kErrWaitTimeout);
              *s_abort = 1;
              break;
            }
          }
        }
      }
      if (*s_abort) {  // let the copies already in flight land before the CTA exits
        for (int t = kc - KST > 0 ? kc - KST : 0; t < kc; ++t) mbar_wait_teardown(&k_full[t % KST], (t / KST) & 1);
        for (int t = vc - VST > 0 ? vc - VST : 0; t < vc; ++t) mbar_wait_teardown(&v_full[t % VST], (t / VST) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_dense(BM, BN, TR::FMT, false, false);
      constexpr uint32_t idO = idesc_dense(BM, D, TR::FMT, false, true);
      const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV);
      long long it = it_begin;
      Piece pc;
      int kc = 0, vc = 0, pidx = 0;
      bool ok = true;
      // descriptor words of every buffer, computed once; an MMA then only adds
      // a constant to the low word
      const DescWords dQ = desc_words(aQ, 16, 1024, 2), dK = desc_words(aK, 16, 1024, 2);
      const DescWords dV = TR::ES <= 2 ? desc_words(aV, BN * 128, 1024, 2) : desc_words(aV, BN * 128, 512, 1);
      auto issue_s = [&](int w, int qb) -> bool {
        const int st = kc % KST;
        if (!mbar_wait(&k_full[st], (kc / KST) & 1, s_abort)) return false;
        tc_fence_after();
        const uint32_t d = tbase + TR::S_COL0 + w * BN;
        const uint32_t qoff = qb * TR::Q_BYTES, koff = st * TR::KV_BYTES;
#pragma unroll
        for (int k = 0; k < TR::QK_STEPS; ++k) {
          const uint32_t off = (k >> 2) * (BM * 128) + (k & 3) * 32;
          const uint32_t offk = (k >> 2) * (BN * 128) + (k & 3) * 32;
          const uint64_t da = desc_at(dQ, qoff + off);
          const uint64_t db = desc_at(dK, koff + offk);
          if constexpr (TR::FP8) mma_f8_ss(d, da, db, idS, k > 0 ? 1u : 0u);
          else if constexpr (TR::ES == 2) mma_bf16_ss(d, da, db, idS, k > 0 ? 1u : 0u);
          else mma_tf32_ss(d, da, db, idS, k > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[w]);
        mma_commit(&k_empty[st]);
        ++kc;
        return true;
      };
      auto issue_pv = [&](int w, bool acc) {
        const int st = vc % VST;
        const uint32_t d = tbase + TR::O_COL0 + w * D;
        const uint32_t pa = tbase + TR::S_COL0 + w * BN;  // P_w aliases S_w
        const uint32_t voff = st * TR::VSTAGE_BYTES;
#pragma unroll
        for (int k = 0; k < TR::PV_STEPS; ++k) {
          const uint64_t db = desc_at(dV, voff + k * TR::MMA_K * 128);
          if constexpr (TR::FP8) {  // P' = hi + lo: two MMAs per K step
            mma_f8_ts(d, pa + k * 8, db, idO, (acc || k > 0) ? 1u : 0u);
            mma_f8_ts(d, pa + TR::BN / 4 + k * 8, db, idO, 1u);
          }
          else if constexpr (TR::ES == 2) mma_bf16_ts(d, pa + k * 8, db, idO, (acc || k > 0) ? 1u : 0u);
          else mma_tf32_ts(d, pa + k * 8, db, idO, (acc || k > 0) ? 1u : 0u);
        }
        mma_commit(&o_done[w]);
        mma_commit(&v_empty[st]);
        ++vc;
      };
      int pcnt[2] = {0, 0};  // P tiles consumed per softmax warpgroup
      while (ok && next_piece(it, pc)) {
        const int qb = pidx & 1;
        ok = mbar_wait(&q_full[qb], (pidx >> 1) & 1, s_abort);
        for (int i = 0; ok && i < 2 && i < pc.n; ++i) ok = issue_s(i, qb);
        for (int i = 0; ok && i < pc.n; ++i) {
          const int w = i & 1;
          if (!mbar_wait(&p_ready[w], pcnt[w] & 1, s_abort)) { ok = false; break; }
          ++pcnt[w];
          // the previous piece's O_A / O_B must have been read before the first P V overwrites them
          if (i == 0 && pidx > 0 && !mbar_wait(merged, (pidx - 1) & 1, s_abort)) { ok = false; break; }
          if (!mbar_wait(&v_full[vc % VST], (vc / VST) & 1, s_abort)) { ok = false; break; }
          tc_fence_after();
          issue_pv(w, i >= 2);
          if (i + 2 < pc.n && !issue_s(w, qb)) { ok = false; break; }
        }
        mma_commit(&q_empty[qb]);  // Q buffer free once every MMA issued so far has completed
        ++pidx;
      }
      mma_commit(drain);  // every MMA issued above has finished once `drain` completes
      mbar_wait_teardown(drain, 0);
    }
  } else {
    // ------------------------------------------------ Q loader (warps 2-3): TMA, then RoPE in place
    const int tid = threadIdx.x - 64;  // 0..63
    long long it = it_begin;
    Piece pc;
    next_piece(it, pc);  // the first piece was loaded above
    int pidx = 1;
    while (next_piece(it, pc)) {
      const int qb = pidx & 1;
      const int h = (pc.u / p.q_tiles) % p.H;
      bool ok = mbar_wait(&q_empty[qb], ((pidx >> 1) & 1) ^ 1, s_abort);
      if (ok && tid == 0) tma_q_tile<QTR>(TR::FP8 ? sQs : sQ + qb * TR::Q_BYTES, &tmQ, &q_tma[qb], p, pc.u);
      float* om = s_omega + qb * (D / 2);
      if (ok && p.rp.enabled)
        for (int j = tid; j < D / 2; j += 64) om[j] = omega_of(p.rp, h, j);
      asm volatile("bar.sync 2, 64;" ::: "memory");
      bool q_ok = false;
      if (ok) {
        const bool landed = mbar_wait(&q_tma[qb], (pidx >> 1) & 1, s_abort);
        if (landed && p.rp.enabled)
          rope_q_tile_inplace<QTR>(TR::FP8 ? sQs : sQ + qb * TR::Q_BYTES, p, om, pc.u, tid, 64);
        if (!landed && tid == 0) mbar_wait_teardown(&q_tma[qb], (pidx >> 1) & 1);  // let the copy land
        q_ok = landed;
      }
      if constexpr (TR::FP8) {
        asm volatile("bar.sync 2, 64;" ::: "memory");  // the RoPE writes are visible
        quantize_q_tile<TR>(sQs, sQ + qb * TR::Q_BYTES, &s_qscale[qb], s_qamax, tid, 64, 2, q_ok);
      }
      asm volatile("bar.sync 2, 64;" ::: "memory");
      if (tid == 0) mbar_arrive(&q_full[qb]);
      ++pidx;
    }
  }
  } else {
    // ------------------------------------------------ softmax warpgroups A (warps 4-7) and B (8-11)
    regs_inc<TR::REGS_HIGH>();
    const int wg = (warp - 4) >> 2;                // 0 = A, 1 = B
    const int row = (threadIdx.x - 128) & 127;     // TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tbase + lane_off + TR::S_COL0 + wg * BN;
    const uint32_t tOA = tbase + lane_off + TR::O_COL0;
    const uint32_t tOB = tOA + D;
    const uint32_t tO = wg ? tOB : tOA;
    const float scale = p.softmax_scale > 0.f ? p.softmax_scale : rsqrtf(static_cast<float>(D));
    const float sl2 = scale * 1.4426950408889634f;
    long long it = it_begin;
    Piece pc;
    int cnt = 0, pidx = 0;
    int vbase = 0;  // V tiles of the earlier pieces (E4M3 variant: the stage that holds a tile's scales)
    bool ok = true;
    while (next_piece(it, pc)) {
      float m_run = -INFINITY, l_run = 0.f;
      int mine = 0;
      // E4M3 variant: S = scale_q * scale_k * (Q8 K8^T); the tile's Q scale
      // folds into the exponent factor, the per-key K scale multiplies S.
      // P' = p * scale_v (per key) is what the tensor core multiplies with
      // V8; the reference max is lowered by kshift so that P' stays below 448.
      float sqsl2 = sl2, kshift = 0.f;
      int hq = 0;
      if constexpr (TR::FP8) {
        const int qb = pidx & 1;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&q_full[qb], (pidx >> 1) & 1, s_abort));  // Q scale written
        sqsl2 = s_qscale[qb] * sl2;
        const int hh = (pc.u / p.q_tiles) % p.H, bb = pc.u / (p.q_tiles * p.H);
        const float svm = p.v_scale_max[bb * p.H + hh];
        kshift = svm > 0.f ? fminf(fmaxf(floorf(log2f(1.75f / svm)), -64.f), 64.f) : 0.f;
        hq = hh & 3;
      }
      for (int i = wg; i < pc.n; i += 2, ++mine) {
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&s_full[wg], cnt & 1, s_abort));
        if (!ok) continue;
        tc_fence_after();
        const float* skb = nullptr;  // [BN][4] K scales of this tile (E4M3 variant)
        const float* svb = nullptr;  // [BN][4] V scales
        if constexpr (TR::FP8) {
          const int vidx = vbase + i, vs = vidx % VST;
          ok = __all_sync(0xffffffffu, mbar_wait(&v_full[vs], (vidx / VST) & 1, s_abort));
          if (!ok) continue;
          skb = reinterpret_cast<const float*>(sV + vs * TR::VSTAGE_BYTES + TR::KV_BYTES) + hq;
          svb = skb + BN * 4;
        }
        uint32_t sr[BN / 32][32];
        constexpr int HC = BN / 64;  // chunks of 32 columns per half
        const int kv_valid = p.Nk - (pc.j0 + i) * BN;
        // row max: 3-input max over 8 independent chains (exact in any order);
        // the second half of S is loaded while the first half is reduced
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = -INFINITY;
#pragma unroll
        for (int c = 0; c < HC; ++c) tmem_load32(tS + c * 32, sr[c]);
#pragma unroll
        for (int c = 0; c < HC; ++c) tmem_load_wait(sr[c]);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if (hf == 0) {
#pragma unroll
            for (int c = HC; c < 2 * HC; ++c) tmem_load32(tS + c * 32, sr[c]);
          } else {
#pragma unroll
            for (int c = HC; c < 2 * HC; ++c) tmem_load_wait(sr[c]);
          }
          if constexpr (TR::FP8) {
#pragma unroll
            for (int c = hf * HC; c < (hf + 1) * HC; ++c)
#pragma unroll
              for (int e = 0; e < 32; ++e) sr[c][e] = __float_as_uint(__uint_as_float(sr[c][e]) * skb[(c * 32 + e) * 4]);
          }
          if (kv_valid < BN) {
#pragma unroll
            for (int c = hf * HC; c < (hf + 1) * HC; ++c)
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c * 32 + e >= kv_valid) sr[c][e] = __float_as_uint(-INFINITY);
          }
#pragma unroll
          for (int c = hf * HC; c < (hf + 1) * HC; ++c)
#pragma unroll
            for (int e = 0; e < 16; ++e)
              mx8[e & 7] = fmax3(mx8[e & 7], __uint_as_float(sr[c][2 * e]), __uint_as_float(sr[c][2 * e + 1]));
        }
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        const float m_new = mx * sqsl2;
        float m_use = m_run;
        bool rescale = false;
        if (m_new > m_run + kshift + 8.0f) {  // m_run is the reference: the row max minus kshift
          m_use = m_new - kshift;
          rescale = (mine > 0);
        }
        // S_i complete implies this warpgroup's previous P V (issued before it) is complete
        if (__any_sync(0xffffffffu, rescale)) {
          const float alpha = rescale ? ex2(m_run - m_use) : 1.0f;
          l_run *= alpha;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_load32(tO + c * 32, o);
            tmem_load_wait(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_store32(tO + c * 32, o);
          }
        }
        m_run = m_use;
        // p = 2^(s * scale * log2(e) - m) on pairs: the argument with one packed
        // FMA, the exponential on the MUFU unit, the running sum in 4 packed
        // partial sums
        const uint64_t sl2x2 = f2_pack(sqsl2, sqsl2), negm2 = f2_pack(-m_use, -m_use);
        uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t plo[8];  // E4M3 variant: the lo terms of this chunk's P'
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t x2 =
                f2_fma(f2_pack(__uint_as_float(sr[c][2 * e]), __uint_as_float(sr[c][2 * e + 1])), sl2x2, negm2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            const float a = ex2(x0), a2 = ex2(x1);
            ls2[e & 3] = f2_add(ls2[e & 3], f2_pack(a, a2));
            if constexpr (TR::FP8) {
              // P' = p * scale_v as two E4M3 terms, hi + lo (lo: the fp16
              // residual), ~8 significant bits in all; four keys per 32-bit
              // word, key 4w in the low byte
              const __half2 ph = __floats2half2_rn(a * svb[(c * 32 + 2 * e) * 4], a2 * svb[(c * 32 + 2 * e + 1) * 4]);
              const uint32_t hi = __nv_cvt_halfraw2_to_fp8x2(ph, __NV_SATFINITE, __NV_E4M3);
              const __half2 hih = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(hi), __NV_E4M3);
              const uint32_t lo = __nv_cvt_halfraw2_to_fp8x2(__hsub2(ph, hih), __NV_SATFINITE, __NV_E4M3);
              if (e & 1) {
                sr[c][e >> 1] |= hi << 16;
                plo[e >> 1] |= lo << 16;
              } else {
                sr[c][e >> 1] = hi;
                plo[e >> 1] = lo;
              }
            } else if constexpr (TR::ES == 2) {
              sr[c][e] = pack_bf16(a, a2);  // packed in place: slot e is free once 2e, 2e+1 were read
            } else {
              sr[c][2 * e] = __float_as_uint(a);
              sr[c][2 * e + 1] = __float_as_uint(a2);
            }
          }
          if constexpr (TR::FP8) {  // hi terms in columns [0, 32), lo terms in [32, 64)
            tmem_store8(tS + c * 8, *reinterpret_cast<uint32_t(*)[8]>(&sr[c][0]));
            tmem_store8(tS + BN / 4 + c * 8, plo);
          }
          else if constexpr (TR::ES == 2) tmem_store16(tS + c * 16, *reinterpret_cast<uint32_t(*)[16]>(&sr[c][0]));
          else tmem_store32(tS + c * 32, sr[c]);
        }
        {
          const uint64_t s01 = f2_add(f2_add(ls2[0], ls2[1]), f2_add(ls2[2], ls2[3]));
          float u0, u1;
          f2_unpack(s01, u0, u1);
          l_run += u0 + u1;
        }
        tmem_store_wait();
        tc_fence_before();
        mbar_arrive(&p_ready[wg]);
        ++cnt;
      }
      // ---- end of the piece: the last P V of this warpgroup must be complete
      if (mine > 0 && ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_done[wg], (cnt - 1) & 1, s_abort));
      if (wg == 1) {
        // B: hand (m, l) over to A once A is done with the previous piece
        if (pidx > 0 && ok) ok = __all_sync(0xffffffffu, mbar_wait(merged, (pidx - 1) & 1, s_abort));
        s_mB[row] = mine > 0 ? m_run : -INFINITY;
        s_lB[row] = mine > 0 ? l_run : 0.f;
        tc_fence_before();
        mbar_arrive(b_ready);
      } else {
        // A: merge the two halves, then write O (whole unit) or a partial
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(b_ready, pidx & 1, s_abort));
        tc_fence_after();
        const bool hasB = pc.n >= 2;
        const float mB = s_mB[row], lB = s_lB[row];
        const float mm = fmaxf(m_run, mB);
        const float aA = ex2(m_run - mm);
        const float aB = hasB ? ex2(mB - mm) : 0.f;
        const float L = l_run * aA + lB * aB;
        const int qt = pc.u % p.q_tiles;
        const int h = (pc.u / p.q_tiles) % p.H;
        const int b = pc.u / (p.q_tiles * p.H);
        const int t = qt * BM + row;
        const bool whole = (pc.j0 == 0 && pc.n == p.nkv);
        const long long first_it = static_cast<long long>(pc.u) * p.nkv;
        const int g_first = owner_of(first_it, p.total, p.grid);
        const int g_last = owner_of(first_it + p.nkv - 1, p.total, p.grid);
        float* slot = p.partials + static_cast<size_t>(g + pc.u) * TR::SLOT_FLOATS;
        const float inv_L = 1.0f / L;
        if (ok) {
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            uint32_t oa[16], ob[16];
            tmem_load16(tOA + c * 16, oa);
            if (hasB) tmem_load16(tOB + c * 16, ob);
            tmem_load_wait16(oa);  // waits for both loads
            if (hasB) tmem_load_wait16(ob);
            float* x = reinterpret_cast<float*>(oa);  // merged in place
#pragma unroll
            for (int e = 0; e < 16; ++e)
              x[e] = __uint_as_float(oa[e]) * aA + (hasB ? __uint_as_float(ob[e]) * aB : 0.f);
            if (whole) {
              if (t < p.Tq) {
                T* dst = static_cast<T*>(p.out) + ((static_cast<size_t>(b) * p.Tq + t) * p.H + h) * D + c * 16;
#pragma unroll
                for (int q8 = 0; q8 < 2; ++q8) {
                  float y[8];
#pragma unroll
                  for (int e = 0; e < 8; ++e) y[e] = x[q8 * 8 + e] * inv_L;
                  store_chunk8<T>(dst + q8 * 8, y);
                }
              }
            } else {
              float4* dst = reinterpret_cast<float4*>(slot) + static_cast<size_t>(4 * c) * BM + row;
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4)
                __stcg(dst + q4 * BM, make_float4(x[4 * q4], x[4 * q4 + 1], x[4 * q4 + 2], x[4 * q4 + 3]));
            }
          }
        }
        tc_fence_before();
        mbar_arrive(merged);  // O_A, O_B and s_mB / s_lB may be reused
        if (whole) {
          if (ok && p.lse != nullptr && t < p.Tq)
            p.lse[(static_cast<size_t>(b) * p.H + h) * p.Tq + t] = (mm + log2f(L)) * 0.6931471805599453f;
        } else {
          if (ok) {
            slot[BM * D + row] = mm;
            slot[BM * D + BM + row] = L;
          }
          __threadfence();
          asm volatile("bar.sync 3, 128;" ::: "memory");
          if (row == 0) {
            const int old = ok ? atomicAdd(&p.counters[pc.u], 1) : -1;
            *s_last = (old == g_last - g_first) ? 1 : 0;
          }
          asm volatile("bar.sync 3, 128;" ::: "memory");
          if (*s_last && ok) {
            // the last piece of this unit to finish: merge every piece of it.
            // The loads of several slots are issued before any is used, so
            // the merge costs a few L2 round trips, not one per chunk.
            __threadfence();
            const int ns = g_last - g_first + 1;
            const float* base = p.partials + static_cast<size_t>(g_first + pc.u) * TR::SLOT_FLOATS;
            float mx = -INFINITY, Lt = 0.f;
            for (int s0 = 0; s0 < ns; s0 += 4) {
              float mv[4], lv[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float* sl = base + static_cast<size_t>(s0 + k < ns ? s0 + k : s0) * TR::SLOT_FLOATS;
                mv[k] = s0 + k < ns ? __ldcg(sl + BM * D + row) : -INFINITY;
                lv[k] = s0 + k < ns ? __ldcg(sl + BM * D + BM + row) : 0.f;
              }
              // every piece holds at least one valid key, so its m is finite
              const float nm = fmaxf(mx, fmaxf(fmaxf(mv[0], mv[1]), fmaxf(mv[2], mv[3])));
              Lt *= ex2(mx - nm);
#pragma unroll
              for (int k = 0; k < 4; ++k) Lt += lv[k] * ex2(mv[k] - nm);
              mx = nm;
            }
            const float inv = 1.0f / Lt;
#pragma unroll 1
            for (int cb = 0; cb < D / 32; ++cb) {
              float4 y[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) y[e] = make_float4(0.f, 0.f, 0.f, 0.f);
              for (int s0 = 0; s0 < ns; s0 += 2) {
                float4 v[2][8];
                float a[2];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                  const bool valid = s0 + k < ns;
                  const float* sl = base + static_cast<size_t>(valid ? s0 + k : s0) * TR::SLOT_FLOATS;
                  a[k] = valid ? ex2(__ldcg(sl + BM * D + row) - mx) * inv : 0.f;
                  const float4* src = reinterpret_cast<const float4*>(sl) + static_cast<size_t>(cb * 8) * BM + row;
#pragma unroll
                  for (int e = 0; e < 8; ++e) v[k][e] = __ldcg(src + e * BM);
                }
#pragma unroll
                for (int k = 0; k < 2; ++k)
#pragma unroll
                  for (int e = 0; e < 8; ++e) {
                    y[e].x += v[k][e].x * a[k];
                    y[e].y += v[k][e].y * a[k];
                    y[e].z += v[k][e].z * a[k];
                    y[e].w += v[k][e].w * a[k];
                  }
              }
              if (t < p.Tq) {
                T* dst = static_cast<T*>(p.out) + ((static_cast<size_t>(b) * p.Tq + t) * p.H + h) * D + cb * 32;
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8) {
                  const float z[8] = {y[2 * q8].x, y[2 * q8].y, y[2 * q8].z, y[2 * q8].w,
                                      y[2 * q8 + 1].x, y[2 * q8 + 1].y, y[2 * q8 + 1].z, y[2 * q8 + 1].w};
                  store_chunk8<T>(dst + q8 * 8, z);
                }
              }
            }
            if (p.lse != nullptr && t < p.Tq)
              p.lse[(static_cast<size_t>(b) * p.H + h) * p.Tq + t] = (mx + log2f(Lt)) * 0.6931471805599453f;
          }
        }
      }
      vbase += pc.n;
      ++pidx;
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
