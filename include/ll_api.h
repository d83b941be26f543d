/*
 * ll_api.h — C ABI of the B200 sink-window attention library (libll_swa.so).
 *
 * The method (LongLive: Real-time Interactive Long Video Generation, paper
 * review; LoL: Longer than Longer, paper review) generates video latent frame
 * by latent frame. Every new frame (or 3-frame chunk) attends, per head, to
 * the KV of 3 pinned "frame sink" frames plus a short window of the most
 * recent frames (LongLive review, sections "Short-Window Attention" and
 * "Frame Sink": 9 local + 3 sink = 12 effective frames). Q and K carry a
 * factorised 3D rotary embedding whose temporal base frequency is jittered per
 * head (LoL review, "Method steps"). At a prompt switch the cached frames' K/V
 * are recomputed (LongLive review, "KV Recache").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers into caller-owned memory unless a
 *   parameter says "host". No call allocates device memory and no call keeps
 *   state for the next one (the one device buffer the library owns is the
 *   static scratch array of ll_sink_window_attention_noalloc); every call is
 *   asynchronous on `stream` (a cudaStream_t passed as void*, NULL = legacy
 *   default stream).
 * - Token tensors use the layout [B][T][H][D] (row-major, D fastest), with
 *   T = frames * N, N = grid_h * grid_w tokens per latent frame in row-major
 *   (grid row, grid column) order.
 * - The KV cache of one layer is [B][S*N][H][D], S = n_sink + n_local slots of
 *   N tokens each (slot s holds tokens [s*N, (s+1)*N)). Frame f is stored in
 *   slot f when f < n_sink and in slot n_sink + (f - n_sink) mod n_local
 *   otherwise. After frames 0..f have been written, the occupied slots are the
 *   prefix [0, min(f+1, S)) and they hold exactly the frames a query at frame f
 *   attends to.
 * - Arguments are validated on the host before anything is launched; a bad
 *   argument returns LL_ERR_INVALID_ARG and ll_last_error() says why.
 *   LL_ERR_UNSUPPORTED marks a well-formed request this build does not
 *   implement. LL_ERR_CUDA reports a failed launch or runtime call.
 * - Device-side waits are bounded. A wait that gives up records a code in the
 *   library's device error word and the kernel returns early (its outputs are
 *   then undefined); ll_device_error() reads and clears that word.
 */
#ifndef LL_API_H
#define LL_API_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LL_ABI_VERSION 2
#define LL_MAX_HEADS 64

typedef enum ll_status {
  LL_OK = 0,
  LL_ERR_INVALID_ARG = 1,
  LL_ERR_UNSUPPORTED = 2,
  LL_ERR_CUDA = 3,
  LL_ERR_TIMEOUT = 4
} ll_status;

typedef enum ll_dtype {
  LL_F32 = 0,       /* IEEE float32 */
  LL_BF16 = 1,      /* bfloat16 */
  LL_FP8_E4M3 = 2   /* OCP E4M3 with one fp32 scale per (token, head); cache storage only */
} ll_dtype;

/*
 * Factorised 3D rotary embedding with LoL per-head jitter.
 * LoL review, "Prerequisites: RoPE": a channel pair (x_{2j}, x_{2j+1}) at
 * position p is rotated by [[cos p*w, -sin p*w], [sin p*w, cos p*w]] with
 * w_i = base^(-2i/d). LoL review, "Method steps": theta_hat_h =
 * theta0 * (1 + sigma * eps_h) is the base of head h.
 * Layout: the D/2 pairs of a head are a temporal band of pairs_t pairs, then
 * pairs_h pairs for the grid row and pairs_w for the grid column; inside a
 * band of P pairs, i = 0..P-1 and d = 2P. The temporal band of head h uses
 * base theta0 * (1 + sigma_t * eps_h[h]); the two spatial bands use theta0.
 * Token (frame f, row r, column c) sits at position ((t_offset + f) * s, r, c)
 * with s = t_scale: position interpolation, the baseline that the LoL review
 * compares against ("Motivation" and results table: PI compresses positions),
 * for s in (0, 1); s = 0 or 1 gives plain RoPE, so a zero-initialised field
 * keeps the ABI-1 behaviour. Validation: LL_ERR_INVALID_ARG for s outside
 * [0, 1].
 */
typedef struct ll_rope_desc {
  int pairs_t, pairs_h, pairs_w;  /* pairs per axis; pairs_t + pairs_h + pairs_w = D/2 */
  double theta0;                  /* base frequency, > 1 */
  double sigma_t;                 /* jitter scale on the temporal band, 0 <= sigma_t < 1 */
  const float* eps_h;             /* HOST pointer to H draws in [-1, 1], or NULL for no jitter */
  int grid_h, grid_w;             /* token grid of one latent frame */
  long long t_offset;             /* temporal position of frame 0 */
  double t_scale;                 /* temporal position factor in [0, 1]; 0 or 1 = no interpolation */
} ll_rope_desc;

/*
 * One layer's sink + ring KV cache (caller-owned device memory).
 * k, v: [B][S*N][H][D] of `dtype` (F32, BF16 or FP8_E4M3).
 * k_scale, v_scale: [B][S*N][H] fp32 dequantisation scales, FP8 only
 * (value = decode(code) * scale; 4-byte aligned); NULL for the other dtypes.
 * D: a multiple of 16; an FP8 cache needs D = 16 * 2^k <= 256
 * (LL_ERR_UNSUPPORTED otherwise). k and v must be 16-byte aligned.
 * S*N (rows per batch entry) must not exceed 2^31 - 1 (LL_ERR_INVALID_ARG).
 */
typedef struct ll_kvcache {
  void* k;
  void* v;
  float* k_scale;
  float* v_scale;
  ll_dtype dtype;
  int B, H, D;
  int tokens_per_frame;   /* N; must equal rope grid_h * grid_w when a rope desc is given */
  int n_sink, n_local;    /* 3 and 9 in the pages' setting */
} ll_kvcache;

/* ABI version of the loaded library (LL_ABI_VERSION at build time). */
int ll_abi_version(void);

/* Message describing the last failure on the calling thread ("" if none). */
const char* ll_last_error(void);

/*
 * Slot of frame `frame` in a cache with n_sink pinned and n_local ring slots.
 * Host only (no GPU needed). LongLive review, "Frame Sink": the sink frames
 * are pinned; the short window keeps the most recent local frames.
 * Errors: LL_ERR_INVALID_ARG for frame < 0, n_sink < 0, n_local < 1 or slot NULL.
 */
ll_status ll_slot_of_frame(long long frame, int n_sink, int n_local, int* slot);

/*
 * Synchronises `stream`, then copies the device error word into *code
 * (0 = no error; bit 0 = a bounded wait gave up) and clears it.
 * Returns LL_ERR_TIMEOUT when the word was non-zero.
 */
ll_status ll_device_error(int* code, void* stream);

/*
 * In-place 3D RoPE of x [B][n_frames*N][H][D] (dtype F32 or BF16) holding the
 * consecutive frames first_frame .. first_frame + n_frames - 1.
 * LoL review, "Method steps" (6): (Q'_h, K'_h) = RoPERotate(Q_h, K_h, omega_h).
 * Errors: LL_ERR_INVALID_ARG for NULL x or rope, x not 16-byte aligned,
 * non-positive sizes, first_frame < 0, D not a multiple of 8, a dtype other
 * than F32 / BF16, or an invalid rope descriptor (pairs not summing to D/2,
 * H > LL_MAX_HEADS, ...); LL_ERR_UNSUPPORTED for 2^31 or more 8-element
 * chunks in one call.
 */
ll_status ll_rope_apply(void* x, ll_dtype dtype, int B, int n_frames, int H, int D,
                        long long first_frame, const ll_rope_desc* rope, void* stream);

/*
 * Append frames first_frame .. first_frame + n_frames - 1 to the cache.
 * k, v: [B][n_frames*N][H][D] of in_dtype (F32 or BF16; BF16 for an FP8 cache).
 * K is rotated with `rope` at each frame's own position before it is stored
 * (rope NULL: k is stored as given). Frame f overwrites slot(f), which evicts
 * the oldest local frame once the ring is full (LongLive review, "Frame Sink"
 * and "Short-Window Attention"). For an FP8 cache each (token, head) row is
 * stored as E4M3 codes of x / scale with scale = max|x| / 448 (1 for a zero
 * row), round-to-nearest-even with saturation.
 * The library keeps no state: calling again with the same first_frame writes
 * the same slots again (one call per denoising pass of the current frame, the
 * last pass's K/V staying in the cache).
 * slots_out: optional HOST array of n_frames ints receiving the slots written.
 * Errors: LL_ERR_INVALID_ARG for NULL or misaligned tensors (k, v 16-byte
 * aligned), first_frame < 0, n_frames < 1 or > n_local (a call may not
 * overwrite its own frames), dtype mismatch with the cache, a rope grid
 * inconsistent with N or an otherwise invalid rope descriptor, an invalid
 * cache descriptor.
 */
ll_status ll_kvcache_append(const ll_kvcache* cache, const void* k, const void* v,
                            ll_dtype in_dtype, long long first_frame, int n_frames,
                            const ll_rope_desc* rope, int* slots_out, void* stream);

/*
 * Attention of the query frames first_frame .. first_frame + n_query_frames - 1
 * over every cached token of the frames they may see: with f the last query
 * frame, the key set is all tokens of slots [0, min(f+1, S)), i.e. the 3 sink
 * frames plus the most recent frames up to f (LongLive review,
 * "Short-Window Attention", "Frame Sink"). The query frames must already be
 * in the cache (append first). Inside the key set there is no mask, so the
 * tokens of a query frame or chunk see each other (frame-level causality).
 * Per head h: out = softmax(Q'_h K_h^T * softmax_scale) V_h
 * (LoL review, "Multi-head attention"), with Q' = RoPE(Q) when rope != NULL
 * (rope NULL: q is already rotated).
 * q, out: [B][n_query_frames*N][H][D]; BF16 for BF16 and FP8 caches, F32 for an
 * F32 cache. softmax_scale 0 means 1/sqrt(D). lse (optional, NULL to skip):
 * [B][H][n_query_frames*N] fp32 natural-log sum of exp of the scaled scores,
 * 4-byte aligned.
 * workspace: device scratch of at least
 * ll_sink_window_attention_workspace_bytes(...) bytes (NULL allowed when that
 * is 0); its contents need not be initialised and are clobbered.
 * Errors: LL_ERR_INVALID_ARG for NULL or misaligned tensors (q, out and
 * workspace 16-byte aligned, lse 4-byte aligned), first_frame < 0,
 * n_query_frames < 1 or > n_local, softmax_scale negative or not finite, a q
 * dtype that does not fit the cache, an invalid rope or cache descriptor, a
 * workspace that is too small; LL_ERR_UNSUPPORTED for D other than 64 or
 * 128 (BF16 and FP8 caches) or 64 (F32). All are reported before anything
 * is launched.
 */
size_t ll_sink_window_attention_workspace_bytes(const ll_kvcache* cache, int n_query_frames);

ll_status ll_sink_window_attention(const void* q, ll_dtype q_dtype, const ll_kvcache* cache,
                                   long long first_frame, int n_query_frames,
                                   const ll_rope_desc* rope, float softmax_scale,
                                   void* out, float* lse, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * The same attention over an FP8_E4M3 cache on the FP8 tensor cores (LongLive
 * model card, abstract: FP8 inference; here it is the KV cache, not the
 * weights, that is 8-bit). Per 128-row query tile, RoPE(Q) is quantised to
 * E4M3 with one scale (max|q| / 448); S = Q8 K8^T runs as a kind::f8f6f4
 * MMA over the cache's codes and is multiplied by the tile's Q scale and each
 * key's K scale; the softmax weights p are multiplied by each key's V scale
 * and stored as two E4M3 terms (hi + lo, ~8 significant bits), and
 * O += P' V8 runs as two kind::f8f6f4 MMAs per key block. The reference
 * max of each row is lowered by a power of two from the largest V scale of
 * the head (a pass over the scales before the attention launch) so that P'
 * stays inside E4M3's range. Results agree with the unquantised attention
 * to the FP8 tolerance (max error <= 5e-2 max|ref|), not bit for bit with
 * ll_sink_window_attention over the same cache (which dequantises the cache
 * into bf16 and computes in bf16).
 * Arguments, layouts and the other errors as for ll_sink_window_attention;
 * workspace: at least ll_sink_window_attention_fp8_mma_workspace_bytes(...)
 * bytes (0 for a cache this entry point does not take).
 * Errors: LL_ERR_INVALID_ARG for a cache that is not FP8_E4M3 or a q that is
 * not BF16; LL_ERR_UNSUPPORTED for D != 128 or H not a multiple of 4 (the
 * scale boxes are 4 heads wide). Two launches: the scale pass, then the
 * attention.
 */
size_t ll_sink_window_attention_fp8_mma_workspace_bytes(const ll_kvcache* cache, int n_query_frames);

ll_status ll_sink_window_attention_fp8_mma(const void* q, ll_dtype q_dtype, const ll_kvcache* cache,
                                           long long first_frame, int n_query_frames,
                                           const ll_rope_desc* rope, float softmax_scale,
                                           void* out, float* lse, void* workspace,
                                           size_t workspace_bytes, void* stream);

/*
 * ll_kvcache_append of frames first_frame .. first_frame + n_frames - 1
 * followed by ll_sink_window_attention of the same frames as queries, in one
 * kernel: each CTA writes its share of the new frames' K/V into their slots
 * while its first query tile loads, all CTAs meet at a grid-wide barrier, and
 * only then is the cache read (LongLive review, "Frame Sink" and
 * "Short-Window Attention": a new frame enters the window and attends to it).
 * The results equal those of the two calls made one after the other.
 * k, v, q, out: [B][n_frames*N][H][D] of `dtype`, which must be the cache's
 * dtype (BF16 or F32), or BF16 for an FP8 cache. The other arguments are those
 * of the two calls. workspace: device scratch of at least
 * ll_append_and_attend_workspace_bytes(...) bytes, its contents need not be
 * initialised (the grid barrier word is tagged with a per-launch generation,
 * so it never needs resetting), and calls sharing it must be ordered.
 * BF16 / F32 cache: one cooperative launch; every CTA must be resident at
 * once, otherwise the launch fails with LL_ERR_CUDA instead of running.
 * FP8 cache: two launches; the first appends the new frames (codes and scales
 * into their slots) and writes the bf16 staging copy of every occupied row
 * that attention over an FP8 cache reads (the new frames' rows from the
 * codes just written), the second is the bf16 attention over that copy.
 * Errors: those of the two calls; LL_ERR_UNSUPPORTED for D other than 64 /
 * 128 (bf16, FP8) and 64 (f32) and for an FP8 cache of more than 64 slots;
 * LL_ERR_TIMEOUT (from ll_device_error) when the barrier wait gives up.
 */
size_t ll_append_and_attend_workspace_bytes(const ll_kvcache* cache, int n_frames);

ll_status ll_append_and_attend(const ll_kvcache* cache, const void* k, const void* v, const void* q,
                               ll_dtype dtype, long long first_frame, int n_frames,
                               const ll_rope_desc* rope, float softmax_scale, void* out, float* lse,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * Phase-coherence kernel of the temporal RoPE band (LoL review, "Core
 * innovation": the phase concentration C(D) = (1/K) sum_{i=1..K}
 * exp(j w_i D) peaks at the offsets where the sink frames collapse, and the
 * per-head jitter of "Method steps" spreads those peaks across heads).
 * For every head h and frame offset D = delta0 .. delta0 + n_delta - 1:
 *   out[h][k] = (re, im) of (1/K) sum_{i<K} exp(j * w_{h,i} * s * D)
 * with K = rope->pairs_t, w_{h,i} = base_h^(-i/K) the temporal-band
 * frequencies of head h (base_h = theta0 (1 + sigma_t eps_h[h])) and
 * s = t_scale (1 when 0). The spatial bands do not enter (reading: D is an
 * offset between frames). Evaluated in fp64, stored as fp32.
 * out: DEVICE [H][n_delta][2] floats, caller-owned, 8-byte aligned.
 * Errors: LL_ERR_INVALID_ARG for a NULL pointer, H outside [1, LL_MAX_HEADS],
 * n_delta < 1, pairs_t < 1, offsets beyond +-2^40 or an invalid rope
 * descriptor; LL_ERR_UNSUPPORTED when H * n_delta >= 2^31.
 */
ll_status ll_phase_coherence(const ll_rope_desc* rope, int H, long long delta0, int n_delta, float* out,
                             void* stream);

/*
 * Self-test of the library's failure detection (not a step of the method):
 * every device-side wait in the kernels is bounded, and one that gives up
 * records LL_ERR_TIMEOUT in the device error word instead of hanging the
 * context. This launches one CTA that waits on a barrier nothing completes
 * and on a two-CTA grid barrier that only it reaches; each wait gives up
 * after the library's bound (about one second of SM clocks) and the kernel
 * returns. Afterwards ll_device_error() reports LL_ERR_TIMEOUT (and clears
 * the word) and the context stays usable. Asynchronous on `stream`; the
 * error word is shared by all calls of the process, so run it alone.
 */
ll_status ll_selftest_bounded_waits(void* stream);

/*
 * Allocation-free variant of ll_sink_window_attention (the pages have no
 * counterpart; this is a library convenience).
 * Some callers cannot call cudaMalloc or any allocating routine: cudaMalloc
 * may synchronise the whole device, which a frame-rate loop cannot afford,
 * and plugin hosts that own all device memory through their own pools forbid
 * allocation outside them. This entry point takes the same arguments minus
 * the workspace and uses instead a scratch array of
 * LL_NOALLOC_SCRATCH_BYTES bytes that the library holds in static device
 * memory: every GPU that loads the library keeps it until the process exits.
 * - `stream` must belong to the current device (LL_ERR_INVALID_ARG
 *   otherwise): the array used is the current device's copy.
 * - The first call on a device looks up that device's copy of the array (with
 *   the device current); make that first call before any stream capture. The
 *   address is kept for the life of the process: a cudaDeviceReset() (or any
 *   teardown of the device's primary context) invalidates it, so do not call
 *   this entry point again after one.
 * - Requests whose scratch need, ll_sink_window_attention_workspace_bytes(),
 *   exceeds LL_NOALLOC_SCRATCH_BYTES are rejected with LL_ERR_INVALID_ARG
 *   before anything is launched.
 * - All calls on a device share the one array and it keeps the contents of
 *   the last call (the parts that must start at zero are cleared by each
 *   call); calls that overlap on the GPU (e.g. on two streams without
 *   ordering between them) race and give undefined results.
 * - It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * Other arguments, layouts and errors as for ll_sink_window_attention.
 */
#define LL_NOALLOC_SCRATCH_BYTES (48u * 1024u * 1024u)

ll_status ll_sink_window_attention_noalloc(const void* q, ll_dtype q_dtype, const ll_kvcache* cache,
                                           long long first_frame, int n_query_frames,
                                           const ll_rope_desc* rope, float softmax_scale, void* out,
                                           float* lse, void* stream);

/*
 * KV recache at a prompt switch (LongLive review, "KV Recache": the cache is
 * rebuilt from the generated frames together with the new prompt).
 * Slots 0..n_slots-1 are recomputed from hidden states x [B][n_slots*N][d_model]
 * (BF16; rows of slot s belong to the frame held in slot s):
 *   K = RoPE(RMSNorm(x Wk; gamma, rms_eps)),  V = x Wv,
 * RMSNorm over the whole H*D-wide row, RoPE at each slot's frame position.
 * wk, wv: [d_model][H*D] BF16 row-major; gamma: [H*D] fp32, 4-byte aligned.
 * slot_frames: HOST array of n_slots absolute frame indices (frame in slot s),
 * each in [0, 2^31 - 1].
 * workspace: device scratch of at least ll_kv_recache_workspace_bytes(...)
 * bytes (0 in this build, where the row sums of the RMSNorm are exchanged on
 * chip between the CTAs of a cluster; NULL is then allowed). The cache may be
 * BF16 or FP8.
 * Errors: LL_ERR_INVALID_ARG for NULL or misaligned pointers, n_slots outside
 * [1, S], frames outside [0, 2^31 - 1]; LL_ERR_UNSUPPORTED for a d_model that
 * is not a positive multiple of 64, for H*D that is not a multiple of 256 up
 * to 2048 or D other than 64 or 128, and for an F32 cache.
 */
size_t ll_kv_recache_workspace_bytes(const ll_kvcache* cache, int d_model, int n_slots);

ll_status ll_kv_recache(const ll_kvcache* cache, const void* x, int d_model,
                        const void* wk, const void* wv, const float* gamma, float rms_eps,
                        const long long* slot_frames, int n_slots, const ll_rope_desc* rope,
                        void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LL_API_H */
