/*
 * tls.h -- C ABI of libtls.so: the per-decode-step two-level sparse attention
 * of AsyncTLS ("AsyncTLS: Efficient Generative LLM Inference with Asynchronous
 * Two-level Sparse Attention"; method summarised in the gist.science explainers,
 * (de) section 2 "Methodik" and (es) section 2 "Metodologia") as hand-written
 * CUDA kernels for NVIDIA B200 (sm_100a).
 *
 * One decode step, per (sequence b, KV head g) "group" of G = H_q / H_kv query
 * heads (query head h uses KV head h / G):
 *   tls_block_score_topk   stages 1+2: Quest-style block bound from per-block
 *                          channel max/min, summed over the group's heads,
 *                          then the top-K_b blocks;
 *   tls_token_score_topk   stages 3+4: label-channel token scores inside the
 *                          kept blocks, then the top-K_t tokens;
 *   tls_sparse_attn_decode stage 5: exact softmax attention over the gathered
 *                          K/V rows of the kept tokens (split over tokens,
 *                          merged by log-sum-exp).
 * tls_build_block_meta builds the block summary and the label-channel slab once
 * per KV cache (set-up, not per step).  tls_prefetch_diff is the incremental
 * host->GPU block transfer of the asynchronous offload engine.
 *
 * Conventions for every entry point
 *  - All tensors are dense, row-major, C-contiguous, allocated and owned by the
 *    caller.  Device pointers must be CUDA device (or managed) memory of the
 *    current device; "pinned host" pointers must be page-locked host memory
 *    (cudaHostAlloc / torch pin_memory).  The library allocates no memory.
 *  - Element pointers (q, K, V, meta, slab, cache, host KV) must be 16-byte
 *    aligned; int32 / fp32 pointers 4-byte aligned.
 *  - Calls are asynchronous: they validate arguments on the host, enqueue
 *    kernels on `stream` (a cudaStream_t; NULL = legacy default stream) and
 *    return.  No call synchronises the device or the stream.
 *  - Errors: a failed host-side check returns TLS_ERR_INVALID_ARG /
 *    TLS_ERR_UNSUPPORTED / TLS_ERR_WORKSPACE before anything is enqueued; a
 *    CUDA launch error returns TLS_ERR_CUDA.  No call aborts the process or
 *    throws.  tls_last_error() gives a message for the calling thread.
 *  - Index outputs are int32, ascending, padded with -1.  k_b larger than the
 *    number of valid blocks, and k_t larger than the number of valid
 *    candidates, are clamped (the tail is -1).
 *  - Tokens at or beyond seq_lens[b] are never summarised, scored or selected.
 *    Device-side values are clamped into [0, max_ctx] for memory safety.
 */
#ifndef TLS_H
#define TLS_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TLS_API __attribute__((visibility("default")))
#else
#define TLS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TLS_OK = 0,
  TLS_ERR_INVALID_ARG = 1, /* null / misaligned pointer, inconsistent shape          */
  TLS_ERR_UNSUPPORTED = 2, /* shape or dtype outside the compiled kernel set          */
  TLS_ERR_WORKSPACE = 3,   /* ws too small (see tls_workspace_size)                   */
  TLS_ERR_CUDA = 4,        /* CUDA runtime / launch error (message kept)              */
  TLS_ERR_TIMEOUT = 5      /* bounded host wait ran out (tls_wait_event)              */
} tls_status;

typedef enum { TLS_F32 = 0, TLS_BF16 = 1 } tls_dtype;

/* Problem description shared by all calls. */
typedef struct tls_shape {
  int32_t batch;         /* B, sequences in the decode batch (0 = nothing to do)        */
  int32_t n_q_heads;     /* H_q, a multiple of n_kv_heads                                */
  int32_t n_kv_heads;    /* H_kv (1 for a shared latent, MLA)                            */
  int32_t d_qk;          /* channels of q and K (the latent width for MLA)               */
  int32_t d_v;           /* channels of V and of the output                              */
  int32_t v_is_k_prefix; /* 1: V = K[..., :d_v] (MLA latent); V pointers are ignored     */
  int32_t block_size;    /* bs, tokens per block                                         */
  int32_t n_label;       /* r, label channels used for token scoring                     */
  int32_t k_b;           /* K_b, blocks kept per group                                   */
  int32_t k_t;           /* K_t, tokens kept per group                                   */
  int32_t max_ctx;       /* n, token capacity: the token stride of K, V and the slab     */
  int32_t kv_dtype;      /* tls_dtype of q, K, V, meta, slab and cache                   */
  int32_t out_dtype;     /* tls_dtype of the attention output                            */
  float softmax_scale;   /* tau; <= 0 selects 1/sqrt(d_qk)                               */
  int32_t block_agg;     /* block score over the group's heads: 0 = sum of the heads'
                          * bounds (the method), 1 = their maximum (a variant)           */
  int32_t slab_bits;     /* label slab: 0 = the K dtype; 8 = int8 codes with one fp32 scale
                          * per (sequence, KV head, label channel) (bf16 K, r in {16,32,64}) */
} tls_shape;

/* Supported shapes (others return TLS_ERR_UNSUPPORTED):
 *   GQA/MQA/MHA: v_is_k_prefix = 0, kv_dtype F32 or BF16, d_qk = d_v in {64, 128},
 *                G = n_q_heads / n_kv_heads in {1, 2, 4, 8, 16, 32, 64};
 *   block_agg 1: bf16 with G <= 64 (GQA, or the latent shape), the per-head
 *                bounds as a tensor-core GEMM whose scores need room (see
 *                tls_block_score_topk); fp32 with G <= 8 on CUDA cores;
 *   MLA:         v_is_k_prefix = 1, kv_dtype BF16, d_qk = 576, d_v = 512,
 *                G a multiple of 4 up to 128;
 *   block_size >= 1, ceil(max_ctx / bs) <= 16384 blocks, 1 <= k_b <= 1024,
 *   k_b * bs <= 16384 candidates, k_t >= 1, B * H_kv <= 65535;
 *   n_label in {8, 16, 32, 64} (BF16) or {4, 8, 16, 32} (F32);
 *   slab_bits 0, or 8 with BF16 keys and n_label in {16, 32, 64}. */

/* Library version string, e.g. "tls 0.1 sm_100a". */
TLS_API const char *tls_version(void);

/* Message of the last failed call on this thread ("" if none). */
TLS_API const char *tls_last_error(void);

/* Bytes of device workspace that tls_sparse_attn_decode(_paged) and
 * tls_decode_step need for this shape on the current device (the split-KV
 * partials; tls_decode_step also keeps the step's block scores there before
 * the attention runs, and after them one readiness word per group and the
 * groups' folded queries [Q+; Q-], 2 d_qk fp32 each).  Calls that run
 * concurrently need separate buffers.  The selection stages take a workspace
 * argument too but use none (their keys stay in on-chip memory); they accept
 * NULL.  Returns 0 for an invalid shape (see tls_last_error). */
TLS_API size_t tls_workspace_size(const tls_shape *s);

/* Bytes of the label slab buffer for this shape: B*H_kv*max_ctx*r elements of
 * the K dtype (slab_bits 0), or, for slab_bits 8, B*H_kv*max_ctx*r int8 codes
 * followed (at the next multiple of 256 bytes) by B*H_kv*r fp32 scales.
 * Returns 0 for an invalid shape. */
TLS_API size_t tls_slab_bytes(const tls_shape *s);

/* Set-up: block summary and label-channel slab of a KV cache.
 * gist.science (de) section 2.A "Stufe 1": blocks are summarised by the
 * per-channel maximum and minimum of their keys; (es) section 2.A.2: token
 * scoring reads only the label channels L.
 *   K          device [B][H_kv][max_ctx][d_qk]
 *   seq_lens   device int32 [B]
 *   label_idx  device int32 [n_label], channel ids in [0, d_qk) (others read as 0)
 *   meta_out   device [B][H_kv][ceil(max_ctx/bs)][2][d_qk]: row 0 = max, row 1 = min
 *              over the block's tokens t < seq_len (a partial last block uses its
 *              valid part; blocks with no valid token are left untouched)
 *   slab_out   device [B][H_kv][max_ctx][n_label]: slab[.., t, c] = K[.., t, label_idx[c]]
 *              for t < seq_len (other rows untouched); may be NULL to skip.
 *              slab_bits 8 (the quantised variant): tls_slab_bytes(s) bytes holding
 *              the codes round-half-even(K / scale) clamped to [-127, 127] (0 where
 *              the scale is 0; rows >= seq_len untouched) and the scales
 *              max|K[.., t < seq_len, L_c]| / 127, both decided in fp32 (the max
 *              comes from the block summary, so meta_out is written first). */
TLS_API tls_status tls_build_block_meta(const tls_shape *s, const void *K, const int32_t *seq_lens,
                                const int32_t *label_idx, void *meta_out, void *slab_out, void *stream);

/* Decode-loop upkeep of the set-up structures: the caller has written the K
 * rows of tokens [old_lens[b], new_lens[b]) of every sequence b; this rebuilds
 * the summaries of the blocks those rows fall in (from all their valid rows,
 * so the result equals tls_build_block_meta at new_lens, bit for bit) and
 * writes the appended tokens' slab rows (slab_out NULL: summaries only).
 * gist.science (de) section 2.A "Stufe 1": the per-block max / min summary;
 * a new decode token only changes the last block's.
 *   old_lens, new_lens device int32 [B], 0 <= old <= new <= max_ctx
 *   max_append         host bound on new - old over all b (sizes the launch);
 *                      a sequence whose range is invalid or longer than
 *                      max_append is left untouched and sets bit 4 of the
 *                      device error word (tls_device_error)
 *   K, label_idx, meta, slab as in tls_build_block_meta.
 * An int8 label slab (slab_bits 8) is not updated here: a new token can move
 * a channel's scale and with it every code of the group.  A non-NULL slab
 * then returns TLS_ERR_UNSUPPORTED; call with slab NULL for the summaries
 * and rebuild the slab with tls_build_block_meta. */
TLS_API tls_status tls_append_tokens(const tls_shape *s, const void *K, const int32_t *old_lens,
                                     const int32_t *new_lens, int32_t max_append, const int32_t *label_idx,
                                     void *meta, void *slab, void *stream);

/* Stages 1+2: block bound and top-K_b blocks.
 * gist.science (de) section 2.A "Stufe 1" + "Optimierung", (es) section 2.A.1:
 *   u_{h,j} = sum_i max(q_{h,i} max_{j,i}, q_{h,i} min_{j,i})
 *           = q_h^+ . max_j + q_h^- . min_j          (q^+ = max(q,0), q^- = min(q,0))
 *   score_j = sum_{h in group} u_{h,j} = (sum_h q_h^+) . max_j + (sum_h q_h^-) . min_j
 * i.e. the contraction over the group's heads is folded into the query before
 * the block summary is streamed once.  Accumulation is fp32; blocks are ranked
 * on the fp32 score, equal scores to the lower block id.
 *   q              device [B][H_q][d_qk]
 *   meta           device [B][H_kv][ceil(max_ctx/bs)][2][d_qk] (tls_build_block_meta)
 *   seq_lens       device int32 [B]
 *   block_idx_out  device int32 [B][H_kv][k_b], ascending block ids, -1 padded
 *   block_score_out device fp32 [B][H_kv][ceil(max_ctx/bs)] or NULL; blocks at or
 *                  beyond ceil(seq_len/bs) hold -inf
 *   ws, ws_bytes   unused (may be NULL / 0), except for block_agg 1 with bf16
 *                  keys: the per-head bounds then run as a tcgen05 GEMM whose
 *                  block scores go to block_score_out, or when that is NULL to
 *                  ws (at least B*H_kv*ceil(max_ctx/bs)*4 bytes, 16-byte
 *                  aligned); with neither, groups of up to 8 heads take the
 *                  CUDA-core path and larger ones return TLS_ERR_WORKSPACE.
 * One launch: the blocks of each group are scored by one thread-block cluster
 * whose CTAs then select the top K_b together (block_agg 1 on the tensor
 * cores: the score launch, then the cluster launch selecting from the scores). */
TLS_API tls_status tls_block_score_topk(const tls_shape *s, const void *q, const void *meta, const int32_t *seq_lens,
                                int32_t *block_idx_out, float *block_score_out, void *ws, size_t ws_bytes,
                                void *stream);

/* Stages 3+4: label-channel token scores inside the kept blocks, top-K_t tokens.
 * gist.science (de) section 2.A "Stufe 2", (es) section 2.A.2 (Double Sparsity):
 *   s_t = sum_{h in group} sum_{c < r} q_{h, L[c]} * slab[t][c]
 * for the candidates t = block_idx[j / bs] * bs + j % bs (j < k_b * bs) with
 * block id >= 0 and t < seq_len.  fp32 accumulation; ranked on fp32, equal
 * scores to the lower token index.
 *   slab            device [B][H_kv][max_ctx][n_label] (tls_build_block_meta); with
 *                   slab_bits 8 the int8 slab, and slab[t][c] reads scale_c * code
 *                   (the kernel multiplies scale_c into the summed query channel)
 *   label_idx       device int32 [n_label]
 *   block_idx       device int32 [B][H_kv][k_b] (ids < 0 are skipped)
 *   token_idx_out   device int32 [B][H_kv][k_t], ascending token positions, -1 padded
 *   token_score_out device fp32 [B][H_kv][k_b * bs] in candidate order, or NULL;
 *                   invalid candidates hold -inf
 *   ws, ws_bytes    unused (may be NULL / 0)
 * One launch: the candidates of each group are scored by one thread-block
 * cluster whose CTAs then select the top K_t together. */
TLS_API tls_status tls_token_score_topk(const tls_shape *s, const void *q, const void *slab, const int32_t *label_idx,
                                const int32_t *block_idx, const int32_t *seq_lens, int32_t *token_idx_out,
                                float *token_score_out, void *ws, size_t ws_bytes, void *stream);

/* Stages 1-4 in one launch: exactly what tls_block_score_topk followed by
 * tls_token_score_topk compute (same arithmetic, same bits), with each
 * group's thread-block cluster going from its block selection straight to its
 * token stage instead of waiting for every group's block selection.  With
 * few groups (fewer than two clusters per SM), at least 4 MB of block
 * summary, at most 16 query heads per KV head and block_score_out given, the
 * block scores are first computed by a grid over all SMs into block_score_out
 * and the clusters select from them (two launches, same bits): one cluster
 * per group alone cannot keep HBM busy.  Each CTA of a group's cluster then
 * selects the K_b blocks itself from the group's scores (at most 4096 blocks;
 * above that the cluster selects them together).
 * Arguments as in those two calls; block_idx_out is written and then read
 * back by the same launch.  block_score_out / token_score_out may be NULL.
 * block_agg 1 with bf16 keys and more than 8 heads per group (or the latent
 * shape) needs block_score_out (tls_decode_step lends its workspace). */
TLS_API tls_status tls_select_step(const tls_shape *s, const void *q, const void *meta, const void *slab,
                                   const int32_t *label_idx, const int32_t *seq_lens, int32_t *block_idx_out,
                                   int32_t *token_idx_out, float *block_score_out, float *token_score_out,
                                   void *stream);

/* tls_select_step with tls_decode_step's workspace (ws: at least
 * tls_workspace_size(s) bytes, 256-byte aligned; checked before anything is
 * enqueued): the same launches as the selection part of tls_decode_step, so
 * that the selection can be run and timed on its own.  The two-phase
 * selection keeps the block scores in ws unless block_score_out is given, and
 * for more than 16 heads per group folds the queries into ws once per group.
 * Ids and scores are the same bits as tls_select_step's. */
TLS_API tls_status tls_select_step_ws(const tls_shape *s, const void *q, const void *meta, const void *slab,
                                      const int32_t *label_idx, const int32_t *seq_lens, int32_t *block_idx_out,
                                      int32_t *token_idx_out, float *block_score_out, float *token_score_out, void *ws,
                                      size_t ws_bytes, void *stream);

/* Stages 1-5 in one call: tls_select_step, then tls_sparse_attn_decode on its
 * token ids, for callers that want the whole decode step.  Its two-phase
 * selection (few groups, as in tls_select_step, the block scores in the
 * workspace unless block_score_out is given) also serves groups of more than
 * 16 query heads: a small launch first folds each group's queries once into
 * the workspace, which the phase-1 grid reads (the same bits as the fold each
 * CTA does otherwise).
 * gist.science (de) section 2.A and (es) section 2.A (the five stages); the
 * two calls above give the definitions.  Arguments:
 *   q, meta, slab, label_idx, seq_lens   as in tls_select_step
 *   K, V                                 as in tls_sparse_attn_decode
 *   block_idx_out, token_idx_out         device int32 [B][H_kv][k_b] / [k_t] (written)
 *   out, lse_out                         as in tls_sparse_attn_decode (lse may be NULL)
 *   block_score_out, token_score_out     as in tls_select_step, or NULL
 *   ws, ws_bytes                         as in tls_sparse_attn_decode (checked
 *                                        before anything is enqueued)
 * When the attention is the warp-MMA kernel (bf16 GQA, d in {64, 128}), the
 * two launches overlap: the selection launch resets one readiness word per
 * group in the workspace, lets the attention launch start early and marks a
 * group ready once its token ids are written; the attention's warps wait per
 * group (bounded: a wait that gives up sets bit 1 of tls_device_error) rather
 * than for the whole selection grid.  Calls on one workspace must not overlap
 * on the GPU. */
TLS_API tls_status tls_decode_step(const tls_shape *s, const void *q, const void *meta, const void *slab,
                                   const int32_t *label_idx, const int32_t *seq_lens, const void *K, const void *V,
                                   int32_t *block_idx_out, int32_t *token_idx_out, void *out, float *lse_out,
                                   float *block_score_out, float *token_score_out, void *ws, size_t ws_bytes,
                                   void *stream);

/* Stage 5: exact attention over the selected tokens.
 * gist.science (es) section 2.A.2: the final attention over the K_t kept tokens
 * at token precision.  For each query head h:
 *   a_t = tau q_h . K[t], o_h = sum_t softmax(a)_t V[t], lse_h = log sum_t exp(a_t)
 * computed by splitting the kept tokens over warps (online softmax, fp32) and
 * merging the partial (max, sum, o) by log-sum-exp.
 *   ws, ws_bytes  device workspace of tls_workspace_size(s) bytes or more,
 *              256-byte aligned; calls that run concurrently need separate
 *              workspaces.
 *   K, V       device [B][H_kv][max_ctx][d_qk] / [..][d_v] (V ignored for MLA)
 *   token_idx  device int32 [B][H_kv][k_t]; entries < 0 or >= max_ctx are skipped
 *   out        device [B][H_q][d_v] in out_dtype
 *   lse_out    device fp32 [B][H_q] (natural log) or NULL; empty selection:
 *              out = 0, lse = -inf */
TLS_API tls_status tls_sparse_attn_decode(const tls_shape *s, const void *q, const void *K, const void *V,
                                  const int32_t *token_idx, void *out, float *lse_out, void *ws, size_t ws_bytes,
                                  void *stream);

/* Stage 5 over a block cache (offloaded KV): token t of group (b, g) lives in
 * cache slot slot_of_block[b][g][t / bs] at row t % bs.
 *   cache          device [B][H_kv][n_slots][2][bs][d_qk]: K block, then V block
 *   slot_of_block  device int32 [B][H_kv][ceil(max_ctx/bs)], -1 = not resident
 *                  (tokens of non-resident blocks are skipped)
 * GQA shapes only (v_is_k_prefix = 0, d_qk = d_v). */
TLS_API tls_status tls_sparse_attn_decode_paged(const tls_shape *s, const void *q, const void *cache,
                                        const int32_t *slot_of_block, int32_t n_slots, const int32_t *token_idx,
                                        void *out, float *lse_out, void *ws, size_t ws_bytes, void *stream);

/* Offload engine: empty the block cache (all slots free, no block resident).
 *   slot_of_block device int32 [B][H_kv][ceil(max_ctx/bs)]  <- -1
 *   block_of_slot device int32 [B][H_kv][n_slots]          <- -1 */
TLS_API tls_status tls_offload_reset(const tls_shape *s, int32_t n_slots, int32_t *slot_of_block, int32_t *block_of_slot,
                             void *stream);

/* Offload engine: incremental block transfer.
 * gist.science (de) section 2.B "Inkrementelle Block-Uebertragung", (es) section
 * 2.B "Transferencia Incremental": only blocks that newly enter the selection
 * cross PCIe.  Per group (b, g):
 *   1. every resident block in neither prev_block_idx nor next_block_idx is
 *      evicted (slot freed, no transfer) -- the caller guarantees that no
 *      attention reading it is still running;
 *   2. every block of next_block_idx that is not resident gets the lowest free
 *      slot (in list order) and its 2*bs*d_qk elements are copied from host_kv
 *      into the cache by a kernel that reads pinned host memory over PCIe.
 * With n_slots >= 2*k_b the cache always holds prev and next together (fewer
 * slots: blocks that find no free slot are not loaded and n_new_out counts only
 * the loaded ones).  Ids in next_block_idx must be distinct; n_slots <= 4096.
 *   host_kv        pinned host [B][H_kv][ceil(max_ctx/bs)][2][bs][d_qk]
 *   cache          device [B][H_kv][n_slots][2][bs][d_qk]
 *   prev_block_idx device int32 [B][H_kv][k_b] or NULL (nothing kept)
 *   next_block_idx device int32 [B][H_kv][k_b]
 *   n_new_out      device int32 [B][H_kv]: blocks copied by this call
 *   jobs_ws        device int32 [B][H_kv][k_b][2] scratch for the copy list
 * Run it on a side copy stream; order it after the block selection with an
 * event.  GQA shapes only. */
TLS_API tls_status tls_prefetch_diff(const tls_shape *s, int32_t n_slots, const void *host_kv, void *cache,
                             int32_t *slot_of_block, int32_t *block_of_slot, const int32_t *prev_block_idx,
                             const int32_t *next_block_idx, int32_t *n_new_out, int32_t *jobs_ws, void *stream);

/* Stages 1+2 for callers that cannot allocate device memory (no counterpart in
 * the paper: an addition of this library).  Computes exactly what
 * tls_block_score_topk computes, needs only the inputs and block_idx_out, and
 * writes the fp32 block scores into a fixed 4 MiB array inside the library's
 * own device memory instead of a caller buffer (e.g. for code running inside
 * another runtime's launch hook, which may not call cudaMalloc).
 *   Limit: batch * n_kv_heads * ceil(max_ctx / block_size) <= 1048576 block
 *   scores; larger shapes return TLS_ERR_UNSUPPORTED with a message.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  The array exists on every GPU that loads the
 *   library until the process exits.  All calls on a device share it and it
 *   keeps the last call's scores: calls whose kernels overlap on the GPU
 *   overwrite each other's scores.  Allocates nothing. */
TLS_API tls_status tls_block_score_topk_noalloc(const tls_shape *s, const void *q, const void *meta,
                                                const int32_t *seq_lens, int32_t *block_idx_out, void *stream);

/* Copies the first `count` fp32 block scores that the last
 * tls_block_score_topk_noalloc call on the current device left in the
 * library's built-in array into dst (device or pinned host memory; layout
 * [B][H_kv][ceil(max_ctx/bs)] of that call's shape), asynchronously on
 * `stream`.  Order it after that call (same stream, or an event).  It is how
 * such a caller, which has no block_score_out buffer of its own to pass,
 * reads the scores back; it allocates nothing.
 * count > 1048576 returns TLS_ERR_INVALID_ARG. */
TLS_API tls_status tls_noalloc_read_scores(float *dst, size_t count, void *stream);

/* Device-side failure flags of the current device.  Kernels that wait on
 * other CTAs or on the tensor-core/copy engines bound every wait; when one
 * gives up (which a correct run never sees) the kernel still ends, its outputs
 * are undefined, and it sets a bit in a library-owned device word; kernels
 * that meet an argument only the device can check set a bit there too:
 *   1 = an attention kernel's wait, 2 = a selection cluster's exchange wait,
 *   4 = tls_append_tokens got a length range it could not apply.
 * Writes the word to *flags_out (0 = no failure since the last clear) and,
 * when clear != 0, zeroes it.  Reads with a synchronous cudaMemcpy, so call it
 * after the work to check has completed. */
TLS_API tls_status tls_device_error(int32_t *flags_out, int32_t clear);

/* Bounded host wait on a cudaEvent_t: polls until the event completes or
 * timeout_ms elapses.  Returns TLS_OK, TLS_ERR_TIMEOUT, or TLS_ERR_CUDA when
 * the event reports an error.  Never blocks longer than timeout_ms (+ 1 ms). */
TLS_API tls_status tls_wait_event(void *event, int32_t timeout_ms);

#ifdef __cplusplus
}
#endif

#endif /* TLS_H */
