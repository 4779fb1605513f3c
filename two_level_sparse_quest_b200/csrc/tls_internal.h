// tls_internal.h -- host-side launchers of the libtls kernels (internal, not ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "tls.h"

namespace tls {

// Launch with programmatic dependent launch enabled: the kernel's launch and
// its pre-wait prologue overlap the tail of the previous kernel in the stream
// (the kernel itself waits for that grid before touching global memory).
// cluster_x > 1 also groups the CTAs into thread-block clusters of
// (cluster_x, 1, 1); grid.x must be a multiple of it.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                      int cluster_x, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster_x > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(cluster_x);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
  return launch_pdl_cluster(kernel, grid, block, smem, st, 1, static_cast<Args &&>(args)...);
}

// Device address of the library's error word on the current device (null if
// it cannot be looked up): kernels whose bounded wait gives up set a bit in it.
int *device_error_word();

// Records a printf-style message for tls_last_error() on this thread; returns st.
tls_status set_error(tls_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));

constexpr int kMaxSelectKeys = 16384;  // keys of one selection (blocks or candidates of a group)

struct MetaArgs {
  const void *K;
  const int32_t *seq_lens;
  const int32_t *label_idx;
  void *meta;
  void *slab;
  int batch, n_kv_heads, d, block_size, n_blocks_max, max_ctx, n_label, dtype;
};
cudaError_t launch_build_meta(const MetaArgs &a, cudaStream_t st);
cudaError_t launch_build_slab(const MetaArgs &a, cudaStream_t st);
// int8 label slab (bf16 keys): scales[group][c] = max |K[t < seq, L_c]| / 127
// from the block summary a.meta, then the codes into a.slab.
cudaError_t launch_label_scales(const MetaArgs &a, float *scales, cudaStream_t st);
cudaError_t launch_build_slab_q8(const MetaArgs &a, const float *scales, cudaStream_t st);
// Incremental update after appending tokens [old_lens[b], new_lens[b]) to K:
// rebuilds the summaries of the blocks those rows fall in and their slab rows.
struct AppendArgs {
  MetaArgs m;                 // m.seq_lens unused
  const int32_t *old_lens, *new_lens;
  int max_append;
  int *err;
};
cudaError_t launch_append_tokens(const AppendArgs &a, cudaStream_t st);

struct BlockScoreArgs {
  const void *q;
  const void *meta;
  const int32_t *seq_lens;
  float *scores;      // [B*H_kv][n_blocks_max] or null (not written)
  int32_t *block_idx; // [B*H_kv][k_b]
  int batch, n_q_heads, n_kv_heads, d, block_size, n_blocks_max, max_ctx, k_b, dtype;
  int *err;           // the library's device error word
  int agg;            // 0: sum of the heads' bounds, 1: their max
  int from_scores;    // 1: scores already hold the step's block scores (the cluster only selects)
  float *qfold;       // [B*H_kv][2 d] folded queries [Q+; Q-] (written by launch_query_fold), or null
};
// Block score and top-K_b in one launch (one thread-block cluster per group).
cudaError_t launch_block_select(const BlockScoreArgs &a, cudaStream_t st);
// Whether the two-phase selection pays off for this many groups on this
// device: the block summary is then streamed by a grid over all SMs into
// a.scores first, and the clusters select from those scores.
bool select_two_phase(int groups, int heads_per_group, int num_sms, size_t summary_bytes, bool folded_queries);
// Phase 1 of the two-phase selection: every group's block scores into a.scores
// (from a.qfold when set, else every CTA folds its groups' queries itself).
cudaError_t launch_block_scores(const BlockScoreArgs &a, int num_sms, cudaStream_t st);
// [Q+; Q-] of every group into a.qfold, once per group, with the arithmetic
// of the in-kernel fold (so the scores are the same bits either way).
cudaError_t launch_query_fold(const BlockScoreArgs &a, cudaStream_t st);
// The max-over-heads block scores (block_agg 1) of every group into a.scores,
// as a tcgen05 GEMM [blocks x 2d] . [2d x heads] with a row maximum (bf16,
// d in {64, 128, 576}, up to 64 heads per group).
bool block_scores_max_tc_supported(int dtype, int d, int heads_per_group);
cudaError_t launch_block_scores_max_tc(const BlockScoreArgs &a, int num_sms, cudaStream_t st);

struct TokenArgs {
  const void *q;
  const void *slab;
  const int32_t *label_idx;
  const int32_t *block_idx;
  const int32_t *seq_lens;
  int32_t *token_idx;
  float *token_score;  // nullable
  int batch, n_q_heads, n_kv_heads, d, block_size, n_blocks_max, max_ctx, n_label, k_b, k_t, dtype;
  int *err;           // the library's device error word
  const float *scales;  // int8 slab: [B*H_kv][r] channel scales; nullptr for a slab of the K dtype
  // select_step only (nullable): per-group readiness words.  The launch resets
  // its group's word, lets the dependent launch start early, and stores `seq`
  // into it (release) once the group's token ids are written.
  int *ready;
  int seq;
};
// Token score and top-K_t in one launch (one thread-block cluster per group).
cudaError_t launch_token_select(const TokenArgs &a, cudaStream_t st);
// Stages 1-4 in one launch: the group's cluster selects its blocks, then its tokens.
cudaError_t launch_select_step(const BlockScoreArgs &a, const TokenArgs &t, cudaStream_t st);

struct AttnArgs {
  const void *q;
  const void *K;
  const void *V;
  const int32_t *token_idx;
  const int32_t *slot_of_block;  // paged only
  int n_slots;                   // paged only
  void *out;
  float *lse;
  float *part;  // workspace partials
  int *err;     // the library's device error word (kErrAttnWait when a bounded wait gave up)
  int batch, n_q_heads, n_kv_heads, d_qk, d_v, v_is_k_prefix, block_size, n_blocks_max, max_ctx, k_t;
  int dtype, out_dtype, paged;
  float scale_log2;  // softmax_scale * log2(e)
  int num_sms;
  // warp-MMA kernel only (nullable): per-group readiness words set by the
  // selection launch before it (instead of waiting for that whole grid, each
  // warp waits for its groups' words to equal seq).
  const int *ready;
  int seq;
};
// Partial-result layout chosen for a shape on a device; shared by the
// workspace query and the launch so both agree.
struct AttnPlan {
  int impl;  // 0: CUDA-core kernel, 1: tcgen05 kernel, 2: warp-MMA GQA kernel, 3: warp-MMA latent kernel,
             // 5: tcgen05 latent kernel (for 1, 3 and 5 tiles_per_warp counts tiles per CTA)
  int warps_per_cta, tokens_per_tile, head_chunk, n_head_chunks;
  int tiles_per_group, total_tiles, grid, tiles_per_warp, max_pieces;
  size_t part_floats;  // floats of workspace for partials
};
bool attn_plan(const AttnArgs &a, AttnPlan *p);
cudaError_t launch_attention(const AttnArgs &a, const AttnPlan &p, cudaStream_t st);
// tensor-core (tcgen05) attention for GQA bf16 d = 128
bool attn_mla_supported(const AttnArgs &a);
cudaError_t launch_attention_mla(const AttnArgs &a, const AttnPlan &p, cudaStream_t st);
// tcgen05 latent attention (bf16, d 576 / 512, up to 64 heads per group)
bool attn_mla_tc_supported(const AttnArgs &a);
int attn_mla_tc_tokens_per_tile();
cudaError_t launch_attention_mla_tc(const AttnArgs &a, const AttnPlan &p, cudaStream_t st);
bool attn_mma_supported(const AttnArgs &a);
int attn_mma_warps(const AttnArgs &a);
// Heads per unit of the warp-MMA kernel: the group, or 16 for larger groups.
int attn_mma_head_chunk(const AttnArgs &a);
cudaError_t launch_attention_mma(const AttnArgs &a, const AttnPlan &p, cudaStream_t st);
bool attn_tc_supported(const AttnArgs &a);
bool attn_tc_plan(const AttnArgs &a, AttnPlan *p);
cudaError_t launch_attention_tc(const AttnArgs &a, const AttnPlan &p, cudaStream_t st);
// merge kernel of the partials (shared by both attention paths)
cudaError_t launch_attention_merge(const AttnArgs &a, const AttnPlan &p, cudaStream_t st);

struct OffloadArgs {
  const void *host_kv;  // device-visible pointer of the pinned host KV
  void *cache;
  int32_t *slot_of_block;
  int32_t *block_of_slot;
  const int32_t *prev_block_idx;
  const int32_t *next_block_idx;
  int32_t *n_new;
  int32_t *jobs;
  int batch, n_kv_heads, d, block_size, n_blocks_max, k_b, n_slots, dtype;
};
cudaError_t launch_offload_reset(const OffloadArgs &a, cudaStream_t st);
cudaError_t launch_prefetch_diff(const OffloadArgs &a, cudaStream_t st);

}  // namespace tls
