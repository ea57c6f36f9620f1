/*
 * lh.h — C ABI of liblh.so, the B200 (sm_100a) Lighthouse selection-and-attend layer.
 *
 * The layer (Nous Research's "Lighthouse Attention", as described by the pages cited below) runs, per head:
 *   1. pool    — symmetric L-level average-pool pyramid over Q, K and V with pool factor p;
 *   2. score   — parameter-free per-head l2 norm of the pooled keys;
 *   3. top-K   — chunked (stratified) top-K per level, the coarsest level always kept whole;
 *   4. gather  — the selected entries as one dense, position-ordered sequence of length S, then causal
 *                attention over it;
 *   5. scatter — the outputs written back to token positions with a causality-preserving offset;
 * and the backward of all five (no gradient through scores or indices).
 *
 * Page short names used in the citations:
 *   [W] wispaper.ai, "Lighthouse Attention：预训练长文本的高速公路，训练提速 21 倍且无损恢复"
 *   [E] encorp.ai, "Услуги по внедряване на AI задават правилния въпрос за Lighthouse Attention"
 *   [C] clawdbytes.com, "Lighthouse Attention: the training-time hierarchy that makes quadratic attention …"
 *   [H] news.hamidun.com, "Nous Research introduced Lighthouse Attention to accelerate LLM training"
 *
 * Conventions (every entry point):
 *   - Tensors are DEVICE pointers owned by the caller, contiguous, row-major, last index fastest, 16-byte aligned.
 *     bf16 tensors are passed as void* (IEEE bfloat16 bit patterns).
 *   - Sizes: B batch, H heads, N tokens, d head dim, L levels, p pool factor, k picks per level, C chunks per
 *     level.  w_l = p^l, N_l = N / w_l.  S = sum_{l<=L-2} min(k, N_l) + N_{L-1}.
 *   - Global pyramid id of entry (l, j): off_l + j with off_l = sum_{l'<l} N_l' (level 0 = raw tokens first).
 *   - The library never allocates device memory, never synchronises (except lh_get_status and
 *     lh_set_wait_limit_ns) and never throws.
 *     Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = legacy default stream).
 *   - Scratch memory is the caller's `ws` of at least lh_workspace_bytes(P) bytes.
 *   - Return value: LH_OK, or an error code.  Argument errors are detected on the host before any launch.
 *     A device-side wait that exceeds its bound records LH_ERR_TIMEOUT in a device status word that
 *     lh_get_status reads; no kernel traps.
 *   - Supported: d in {64, 128}; p in {2, 4, 8}; 1 <= L <= 5 with p^(L-1) <= 512; k / C <= 512.
 *     Other valid shapes return LH_ERR_UNSUPPORTED.
 */
#ifndef LH_H_
#define LH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LH_OK 0
#define LH_ERR_INVALID_ARG 1  /* bad sizes, NULL or misaligned pointer, indivisible shapes */
#define LH_ERR_UNSUPPORTED 2  /* valid layer, but outside what the kernels are built for */
#define LH_ERR_CUDA 3         /* a CUDA runtime call or launch failed */
#define LH_ERR_TIMEOUT 4      /* a device wait hit its bound (reported by lh_get_status) */
#define LH_ERR_WORKSPACE 5    /* ws_bytes smaller than lh_workspace_bytes */
#define LH_ERR_RANGE 6        /* a value left the fp16 range of the attention operands (reported by lh_get_status) */

#define LH_MAX_LEVELS 8

/* lh_params.flags: LH_EXPAND_CHILDREN selects the children-expansion reading of the selection, the one under which
 * the size example of [E] "Какво точно промени Nous Research в attention пътя?" (N = 1,000,000, L = 4, p = 4,
 * k = 4,096 -> a gathered sequence of about 65,000 tokens) comes out: the keys of levels 1..L-1 are scored, the
 * chunked top-K ranks level l+1 (C chunks, k/C picks each, ties to the lower index), and level l <= L-2 keeps the
 * p children p*J .. p*J + p-1 of every pick J; the coarsest level is still kept whole.  Then
 * S = sum_{l=1}^{L-1} p*min(k, N_l) + N_{L-1} (64,777 at that example; 65,536 at N = 2^20).  Validity: C | N_l and
 * C | k for every ranked level l with k < N_l.  Everything after the selection (order, gather, attention,
 * scatter, backward) is unchanged.  flags = 0 is the per-level reading of the conventions above. */
#define LH_EXPAND_CHILDREN 1

/* Layer sizes.  flags: 0 or LH_EXPAND_CHILDREN (any other bit is LH_ERR_INVALID_ARG). */
typedef struct lh_params {
  int32_t B, H, N, d, L, p, k, C;
  int32_t flags;
} lh_params;

/* Byte offsets of the saved-context tensors inside the caller's ctx buffer (see lh_forward). */
typedef struct lh_ctx_layout_t {
  uint64_t qg, kg, vg;     /* fp16 [B,H,S,d]: gathered Q, K, V (see lh_gather) */
  uint64_t og;             /* fp32 [B,H,S,d]: attention output over the gathered sequence */
  uint64_t lse;            /* fp32 [B,H,S]: natural-log row log-sum-exp of the attention */
  uint64_t idx_g;          /* int32 [B,H,S]: global pyramid id of gathered row s */
  uint64_t slot;           /* int32 [B,H,R], R = sum_l N_l: gathered position of entry off_l + j, or -1 */
  uint64_t total;          /* bytes needed (= lh_ctx_bytes) */
} lh_ctx_layout_t;

/* ---- host-only queries (no device work) -------------------------------------------------------------- */

/* Static string for a status code. */
const char* lh_error_string(int status);

/* LH_OK if P describes a valid layer the kernels support, else LH_ERR_INVALID_ARG / LH_ERR_UNSUPPORTED.
 * Validity: sizes >= 1, p >= 2, p^(L-1) | N, and C | N_l, C | min(k, N_l) for every level l <= L-2 whose
 * picks are fewer than its entries ([C] "Four-Stage Pipeline…": equal chunks per level). */
int lh_validate(const lh_params* P);

/* Gathered length S (see conventions), or -1 if P is invalid. */
int64_t lh_S(const lh_params* P);

/* N_l, or -1 for an invalid P or level. */
int64_t lh_level_size(const lh_params* P, int level);

/* off_l (global pyramid id of entry (l, 0)), or -1. */
int64_t lh_level_offset(const lh_params* P, int level);

/* Rows per head of the pyramid written by lh_pool: sum_{l=1}^{L-1} N_l (level l starts at row
 * sum_{1<=l'<l} N_l'); -1 if invalid. */
int64_t lh_pyramid_rows(const lh_params* P);

/* Rows per head of the score array: sum_{l=0}^{L-2} N_l (level l starts at row off_l); with LH_EXPAND_CHILDREN
 * sum_{l=1}^{L-1} N_l (level l starts at row off_l - N_0); -1 if invalid. */
int64_t lh_score_rows(const lh_params* P);

/* Rows per head of the slot map: sum_{l=0}^{L-1} N_l; -1 if invalid. */
int64_t lh_slot_rows(const lh_params* P);

/* Bytes of the saved context written by lh_forward and read by lh_backward (0 if invalid). */
size_t lh_ctx_bytes(const lh_params* P);

/* Fills *out with the ctx layout; LH_OK or an error code. */
int lh_ctx_layout(const lh_params* P, lh_ctx_layout_t* out);

/* Scratch bytes every device entry point of this header needs at most (0 if invalid). */
size_t lh_workspace_bytes(const lh_params* P);

/* ---- step-wise API ----------------------------------------------------------------------------------- */

/* Step 1, pool ([W] 核心方法 §1 对称金字塔池化; [E] "Какво точно промени Nous Research в attention пътя?").
 * x: bf16 [B,H,N,d].  pyr: bf16 [B,H,lh_pyramid_rows,d], levels 1..L-1 stacked (finest first).
 * Pooled value = bf16_RN(block sum / p^l), the sum taken in fp64 recursively over the p children, left to right
 * (exact mean rounded once whenever the fp64 sum is exact). */
int lh_pool(const lh_params* P, const void* x, void* pyr, void* stream);

/* Steps 2-3 and the gathered order ([W] 核心方法 §2 层次化选择器; [C] "Four-Stage Pipeline Wraps Standard
 * FlashAttention").
 * k: bf16 [B,H,N,d] raw keys.  Scores: squared l2 norm of the pooled key (raw key at level 0), fp64 sum of
 * squares (eight left to right per group of eight features, then a pairwise tree over the groups), rounded
 * to fp32, for levels 0..L-2 (levels 1..L-1 with LH_EXPAND_CHILDREN).
 * scores_in: optional fp32 [B,H,lh_score_rows]; when non-NULL it replaces the computed scores.  Any finite values
 * are ordered correctly (negative ones included; -0 and +0 are equal and tie); NaN scores give an unspecified but
 * deterministic selection.
 * scores_out: optional fp32 [B,H,lh_score_rows]; when non-NULL (and scores_in is NULL) receives the scores.
 * Selection: C equal chunks per level, each keeping its min(k,N_l)/C entries of largest score (ties: lower
 * index); coarsest level whole.  Order: ascending end token (j+1)*p^l - 1, equal ends coarser level first.
 * idx_g: int32 [B,H,S] (out).  slot: int32 [B,H,lh_slot_rows] (out).  ws: scratch. */
int lh_score_topk(const lh_params* P, const void* k, const float* scores_in, float* scores_out, int32_t* idx_g,
                  int32_t* slot, void* ws, size_t ws_bytes, void* stream);

/* Step 4a, gather ([W] 核心方法 §3; [E] "Какво точно промени…").  q,k,v: bf16 [B,H,N,d];
 * q_pyr,k_pyr,v_pyr: bf16 [B,H,lh_pyramid_rows,d] from lh_pool (may be NULL when L == 1); idx_g from
 * lh_score_topk.  qg,kg,vg: fp16 [B,H,S,d] (out), row s = the bf16 pooled value of entry idx_g[s] (raw row at
 * level 0) converted to fp16, the attention's operand format: exact for magnitudes in [2^-14, 65504]; a larger
 * value records LH_ERR_RANGE in the device status word. */
int lh_gather(const lh_params* P, const void* q, const void* k, const void* v, const void* q_pyr,
              const void* k_pyr, const void* v_pyr, const int32_t* idx_g, void* qg, void* kg, void* vg,
              void* stream);

/* Step 4b, causal attention over the gathered sequence ([W] 核心方法 §3 标准 FlashAttention 调用;
 * [H] "How Lighthouse Attention Works").  og = softmax(qg kg^T / sqrt(d) + causal mask) vg, diagonal included.
 * qg,kg,vg: fp16 [B,H,S,d] (as written by lh_gather); og: fp32 [B,H,S,d] (out, accumulator precision); lse: fp32
 * [B,H,S] (out, natural log).  Runs on the tcgen05 tensor cores (TMA-fed, TMEM accumulators); P enters the PV
 * product in fp16. */
int lh_attend(const lh_params* P, const void* qg, const void* kg, const void* vg, float* og, float* lse,
              void* stream);

/* Step 5, offset scatter-back ([W] figure caption "Scatter-back"; [E] "Как four-stage pipeline…": offset that
 * preserves causality).  O[t] = sum over levels l of og[slot(l, floor((t+1)/p^l) - 1)] over selected entries
 * (entry (l,j) reaches tokens (j+1)p^l - 1 .. (j+2)p^l - 2); tokens without a selected candidate get 0.
 * og: fp32 [B,H,S,d]; slot from lh_score_topk; o: bf16 [B,H,N,d] (out, fp32 sum rounded once). */
int lh_scatter(const lh_params* P, const float* og, const int32_t* slot, void* o, void* stream);

/* ---- fused API --------------------------------------------------------------------------------------- */

/* Whole forward: q,k,v bf16 [B,H,N,d] -> o bf16 [B,H,N,d].  ctx: device buffer of lh_ctx_bytes(P) bytes that
 * receives the saved context (layout from lh_ctx_layout) and must stay untouched until lh_backward.
 * Pooled values, scores and the selection are bit-identical to the step-wise API. */
int lh_forward(const lh_params* P, const void* q, const void* k, const void* v, void* o, void* ctx, void* ws,
               size_t ws_bytes, void* stream);

/* Whole backward ([E] "Как four-stage pipeline…": gradients reach Q, K, V only through the gathered values;
 * [W] 深度洞察).  dout: bf16 [B,H,N,d]; ctx from lh_forward; dq,dk,dv: bf16 [B,H,N,d] (out).
 * dX[t] = sum_l [(l, floor(t/p^l)) selected] dX_g[slot] / p^l.
 * Determinism: dk and dv are bitwise reproducible from run to run; dq is accumulated with fp32 reduce-adds whose
 * order is not fixed, so it may differ in its last bits between runs (always within the stated tolerance). */
int lh_backward(const lh_params* P, const void* dout, const void* ctx, void* dq, void* dk, void* dv, void* ws,
                size_t ws_bytes, void* stream);

/* ---- test-only pieces of the backward ---------------------------------------------------------------- */

/* dog[s] = sum_{t=E_s}^{min(E_s + w - 1, N - 1)} dout[t] (fp32 sum) for the entry idx_g[s] with end E_s and
 * window w.  dout: bf16 [B,H,N,d]; dog: fp32 [B,H,S,d] (out). */
int lh_scatter_bwd(const lh_params* P, const void* dout, const int32_t* idx_g, float* dog, void* stream);

/* Causal attention backward over S.  qg,kg,vg: fp16 [B,H,S,d]; og: fp32 [B,H,S,d] and lse from lh_attend;
 * dog: fp32 [B,H,S,d] (gradient of og).  dqg, dkg, dvg: fp32 [B,H,S,d] (out).  ws: scratch.
 * The tensor-core operands are fp16; dog is scaled per head by a power of two before rounding (its largest
 * magnitude in [2^9, 2^10)) and the results are scaled back. */
int lh_attend_bwd(const lh_params* P, const void* qg, const void* kg, const void* vg, const float* og,
                  const float* lse, const float* dog, float* dqg, float* dkg, float* dvg, void* ws, size_t ws_bytes,
                  void* stream);

/* ---- tracing ----------------------------------------------------------------------------------------- */

/* Device time of the library's own kernels.  While enabled, every kernel the library enqueues is bracketed by two
 * CUDA events recorded on the stream it is launched on.  lh_profile_read waits for those events, writes up to
 * max_entries records {kernel name, launches, summed milliseconds} accumulated since the last read (or enable),
 * clears them and returns the number of records (or -LH_ERR_CUDA).  Events are created lazily and reused. */
typedef struct lh_kernel_time_t {
  char name[32];
  int32_t launches;
  double ms;
} lh_kernel_time_t;

int lh_profile_enable(int on);
int lh_profile_read(lh_kernel_time_t* out, int max_entries);

/* ---- selection without caller scratch ---------------------------------------------------------------- */

/* Size of the library's fixed device scratch array used by lh_score_topk_static.  No call allocates it: it is part
 * of the library's device module, so every device on which the library's kernels are loaded (the first use of any
 * entry point there) reserves these bytes until the process exits, whether or not lh_score_topk_static is called. */
#define LH_STATIC_SCRATCH_BYTES (16u << 20)

/* The pages have no counterpart to this entry point; it exists for callers that cannot allocate device memory
 * where they need the selection (for example a runtime that plans all device memory once at start-up and
 * forbids allocation on its step path, or a hook handed only the tensors it reads and writes).
 *
 * Same result as lh_score_topk (same arguments, same kernels, bit-identical idx_g, slot and scores), but the
 * scratch comes from a fixed device array inside the library instead of a caller workspace, and no device
 * memory is allocated or freed.  The scratch holds the selection lists (B*H*sum over partially selected levels
 * of k int32) and, only when both scores_in and scores_out are NULL, the scores (B*H*lh_score_rows fp32), each
 * rounded up to 256 bytes; a call that needs more than LH_STATIC_SCRATCH_BYTES returns LH_ERR_WORKSPACE before
 * any launch.  Nothing in the array has to start at zero: every call writes what it later reads.
 *
 * The first call on a device looks up the array's device address with cudaGetSymbolAddress (with that device
 * current) and caches it; make that first call before any stream capture.  All calls on a device share the one
 * array, which keeps the last call's contents: calls whose work can overlap on the GPU (different streams,
 * concurrent host threads) race on it and must be serialised by the caller. */
int lh_score_topk_static(const lh_params* P, const void* k, const float* scores_in, float* scores_out,
                         int32_t* idx_g, int32_t* slot, void* stream);

/* ---- host-resident step ------------------------------------------------------------------------------ */

/* Device bytes lh_step_host needs with chunks of `heads_per_chunk` heads (0 if P is invalid or heads_per_chunk
 * does not divide H): three chunks' eight tensors, one chunk's ctx and one chunk's workspace. */
size_t lh_step_host_bytes(const lh_params* P, int heads_per_chunk);

/* The pages have no counterpart to this entry point: it serves callers whose tensors live in host memory.
 *
 * One lh_forward + lh_backward on HOST tensors: q, k, v, dout (bf16 [B,H,N,d], read) -> o, dq, dk, dv (bf16
 * [B,H,N,d], written); results equal those of the device entry points on the same data (each head is computed
 * alone, exactly as in a call over all heads).  Heads are independent through the whole layer, so the work runs in
 * chunks of heads_per_chunk consecutive heads of one batch row (heads_per_chunk must divide H): chunk g's
 * host-to-device copies (on h2d_stream), its forward and backward (on stream) and its device-to-host copies (on
 * d2h_stream) overlap with the neighbouring chunks'.  Host buffers should be page-locked: pageable memory makes the
 * copies synchronous and serialises the pipeline (results are the same).  The three streams should be distinct
 * for the overlap (any of them may be NULL, the legacy default stream, at the cost of it).
 * dev: caller's device buffer of at least lh_step_host_bytes(P, heads_per_chunk) bytes, 256-byte aligned; it is
 * scratch only (nothing is kept in it between calls).  Everything is enqueued: the copies start after the work
 * already on `stream`, and `stream` is ordered after the last device-to-host copy, so synchronising `stream`
 * makes o, dq, dk, dv valid on the host.  Errors: LH_ERR_INVALID_ARG (sizes, heads_per_chunk, NULL or misaligned
 * pointers), LH_ERR_WORKSPACE (dev_bytes too small), LH_ERR_CUDA (a copy, event or launch failed), or the error
 * of lh_forward / lh_backward; a failure mid-way leaves the earlier chunks enqueued.  The pipeline's events are
 * created once per device (the first call, under a lock) and reused by every call, so calls on one device whose
 * work can overlap (several host threads or streams) must be serialised by the caller. */
int lh_step_host(const lh_params* P, const void* q, const void* k, const void* v, const void* dout, void* o, void* dq,
                 void* dk, void* dv, int heads_per_chunk, void* dev, size_t dev_bytes, void* stream, void* h2d_stream,
                 void* d2h_stream);

/* ---- context parallelism: one sequence split across G ranks ------------------------------------------ */

/* [E] "Може ли този подход да скалира отвъд един GPU по начин, който ops екипите ще приемат?": beyond ~100K tokens
 * the layer runs context-parallel; pooling, scoring and top-K stay local to each shard and the gathered dense
 * subsequence takes part in ordinary ring attention.  Here the N tokens of every head are split into G equal
 * shards, rank r holding tokens [r N/G, (r+1) N/G) of Q, K, V, dO, O, dQ, dK, dV as its own bf16 [B,H,N/G,d]
 * tensors.  Requirements: G | C and G | k (every chunk, so every pick, lies inside one shard: rank r's selection is
 * exactly the global selection's entries in its shard, S/G of them, and its gathered rows are rows r S/G ..
 * (r+1) S/G - 1 of the global gathered sequence); for G > 1 also S/G a multiple of 128 (LH_ERR_UNSUPPORTED
 * otherwise).  Results equal those of lh_forward / lh_backward on the whole sequence (selection and gathered rows
 * bit-exact; outputs up to the order of fp32 sums).
 *
 * The caller runs the exchanges (NCCL over NVLink, say), each into its own device memory:
 *   forward:  lh_cp_forward_select -> all-gather of each rank's K_g/V_g chunk (kv_bytes bytes at kv_offset of its
 *             ctx, rank order) into kv_all -> lh_cp_forward_attend -> all-gather of the halo blocks ->
 *             lh_cp_forward_scatter with rank r-1's block;
 *   backward: lh_cp_backward_halo -> all-gather of the halo blocks -> lh_cp_backward_attend with rank r+1's block
 *             -> reduce-scatter (sum) of dkv_part (G blocks of dkv_bytes, block g to rank g) -> lh_cp_backward_unpool.
 * ctx and ws are per rank, sized for the shard's parameters (lh_cp_layout(...).local), and ws must keep its
 * contents from lh_cp_backward_attend to lh_cp_backward_unpool (it holds the dQ_g accumulator). */
typedef struct lh_cp_layout_t {
  lh_params local;      /* the shard's parameters: N/G, k/G, C/G, the rest as given */
  int64_t S_local;      /* gathered rows per rank, S/G */
  uint64_t kv_offset;   /* byte offset, inside a rank's ctx, of the chunk it contributes to the K_g/V_g exchange */
  uint64_t kv_bytes;    /* bytes of that chunk (K_g at 0, V_g at v_offset); kv_all holds G chunks in rank order */
  uint64_t v_offset;    /* byte offset of V_g inside a chunk */
  uint64_t halo_bytes;  /* bytes of one rank's halo block, fp32 [B*H][L][d]; a halo exchange holds G blocks */
  uint64_t dkv_bytes;   /* bytes of one block of the dK_g/dV_g exchange, fp32 [2][B*H][S/G][d] (dK_g then dV_g) */
} lh_cp_layout_t;

/* Sizes of the split for global parameters P over G ranks; LH_OK or the validation error. */
int lh_cp_layout(const lh_params* P, int G, lh_cp_layout_t* out);

/* Forward steps 1-4a on rank `rank`'s shard: pool, score, top-K, order and gather of its tokens into ctx. */
int lh_cp_forward_select(const lh_params* P, int G, int rank, const void* q, const void* k, const void* v, void* ctx,
                         void* ws, size_t ws_bytes, void* stream);

/* Forward step 4b: the shard's gathered queries (global rows rank*S/G ..) attend causally over the gathered keys
 * and values of ranks 0..rank in kv_all (G chunks of kv_bytes, as exchanged); O_g and LSE go to ctx.  Then
 * halo_out (one block, fp32 [B*H][L][d]) receives, per head and level l, O_g of the shard's last level-l entry
 * (zeros when it is not selected): the next rank's tokens t < p^l - 1 take it at level l. */
int lh_cp_forward_attend(const lh_params* P, int G, int rank, void* ctx, const void* kv_all, float* halo_out,
                         void* stream);

/* Forward step 5: the offset scatter-back of the shard's tokens; halo_prev is rank rank-1's halo block (ignored,
 * may be NULL, on rank 0).  o: bf16 [B,H,N/G,d]. */
int lh_cp_forward_scatter(const lh_params* P, int G, int rank, const void* ctx, const float* halo_prev, void* o,
                          void* stream);

/* Backward exchange: halo_out (one block) receives, per head and level l, the fp32 sum of the shard's first p^l - 1
 * rows of dout: the part of the previous rank's last level-l window that lies in this shard. */
int lh_cp_backward_halo(const lh_params* P, int G, int rank, const void* dout, float* halo_out, void* stream);

/* Backward through the attention: dO_g window sums of the shard (plus halo_next, rank rank+1's halo block, in the
 * last window of each level; ignored, may be NULL, on the last rank), then the attention backward of the shard's
 * queries against the keys of ranks 0..rank.  dQ_g stays in ws; dkv_part (G blocks of dkv_bytes) receives this
 * rank's contribution to dK_g/dV_g of every rank's keys (zeros for ranks after this one).  dQ_g is accumulated
 * with fp32 reduce-adds in no fixed order. */
int lh_cp_backward_attend(const lh_params* P, int G, int rank, const void* dout, const void* ctx, const void* kv_all,
                          const float* halo_next, float* dkv_part, void* ws, size_t ws_bytes, void* stream);

/* Backward unpool: dq, dk, dv (bf16 [B,H,N/G,d]) of the shard from dQ_g (in ws) and dkv, this rank's block of the
 * summed exchange (fp32 [2][B*H][S/G][d]). */
int lh_cp_backward_unpool(const lh_params* P, int G, int rank, const void* ctx, const float* dkv, void* dq, void* dk,
                          void* dv, void* ws, size_t ws_bytes, void* stream);

/* ---- status ------------------------------------------------------------------------------------------ */

/* Synchronises `stream`, returns the first device-side error recorded since the last call (LH_OK if none)
 * on the current device, and clears it. */
int lh_get_status(void* stream);

/* Bound, in nanoseconds, on every device-side wait of the kernels launched on the current device from now on
 * (0 restores the default of 2 s).  A wait that exceeds it records LH_ERR_TIMEOUT (read with lh_get_status); the
 * block then stops, after waiting for the copies and tensor-core products it has issued, and frees its tensor
 * memory, so the context stays usable and the next call computes normally.  It exists to test that path: a short
 * limit makes ordinary waits give up.  Synchronises the device (call it while no other work of the library is in
 * flight); LH_OK or LH_ERR_CUDA. */
int lh_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* LH_H_ */
