// tls_api.cu -- the extern "C" entry points of libtls.so (declared in
// include/tls.h): host-side argument checks, workspace layout, kernel
// dispatch and error reporting.  Nothing here computes; every step of the
// decode path runs in the kernels of tls_meta.cu, tls_select.cu, tls_attn.cu
// and tls_offload.cu.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <mutex>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <thread>

#include "tls.h"
#include "tls_internal.h"

namespace {

thread_local std::string g_err;

tls_status fail(tls_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
tls_status fail(tls_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

tls_status cuda_status(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return TLS_OK;
  return fail(TLS_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ceil(max_ctx / block_size) in 64-bit (max_ctx near INT_MAX must not wrap);
// max_ctx <= INT_MAX keeps the quotient in int range.
int n_blocks_max(const tls_shape *s) {
  return static_cast<int>((static_cast<long long>(s->max_ctx) + s->block_size - 1) / s->block_size);
}

int device_sms() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

// Common shape checks.  `need_attn` adds the attention kernel-set checks.
tls_status check_shape(const tls_shape *s) {
  if (!s) return fail(TLS_ERR_INVALID_ARG, "shape is NULL");
  if (s->batch < 0) return fail(TLS_ERR_INVALID_ARG, "batch < 0");
  if (s->n_kv_heads < 1 || s->n_q_heads < 1 || s->n_q_heads % s->n_kv_heads)
    return fail(TLS_ERR_INVALID_ARG, "n_q_heads (%d) must be a positive multiple of n_kv_heads (%d)", s->n_q_heads,
                s->n_kv_heads);
  if (s->kv_dtype != TLS_F32 && s->kv_dtype != TLS_BF16) return fail(TLS_ERR_INVALID_ARG, "kv_dtype %d", s->kv_dtype);
  if (s->out_dtype != TLS_F32 && s->out_dtype != TLS_BF16) return fail(TLS_ERR_INVALID_ARG, "out_dtype %d", s->out_dtype);
  if (s->block_size < 1) return fail(TLS_ERR_INVALID_ARG, "block_size < 1");
  if (s->max_ctx < 1) return fail(TLS_ERR_INVALID_ARG, "max_ctx < 1");
  // kernels form seq_len + block_size - 1 in int
  if (s->max_ctx > INT32_MAX - s->block_size)
    return fail(TLS_ERR_UNSUPPORTED, "max_ctx + block_size exceeds the int32 range");
  if (s->k_b < 1 || s->k_t < 1) return fail(TLS_ERR_INVALID_ARG, "k_b and k_t must be >= 1");
  if (s->d_qk < 1 || s->d_v < 1) return fail(TLS_ERR_INVALID_ARG, "d_qk and d_v must be >= 1");
  if (s->v_is_k_prefix && s->d_v > s->d_qk) return fail(TLS_ERR_INVALID_ARG, "v_is_k_prefix needs d_v <= d_qk");
  if (s->block_agg != 0 && s->block_agg != 1) return fail(TLS_ERR_INVALID_ARG, "block_agg %d", s->block_agg);
  if (s->block_agg == 1 && s->v_is_k_prefix && s->n_q_heads / s->n_kv_heads > 64)
    return fail(TLS_ERR_UNSUPPORTED, "max-over-heads block aggregation supports up to 64 heads per latent");
  if (static_cast<long long>(s->batch) * s->n_kv_heads > 65535)
    return fail(TLS_ERR_UNSUPPORTED, "batch * n_kv_heads > 65535");
  const int G = s->n_q_heads / s->n_kv_heads;
  if (s->v_is_k_prefix) {
    if (s->kv_dtype != TLS_BF16 || s->d_qk != 576 || s->d_v != 512 || G % 4 || G > 128)
      return fail(TLS_ERR_UNSUPPORTED, "latent attention supports bf16, d_qk 576, d_v 512, G a multiple of 4 <= 128");
  } else {
    if (s->d_qk != s->d_v || (s->d_qk != 64 && s->d_qk != 128))
      return fail(TLS_ERR_UNSUPPORTED, "GQA supports d_qk = d_v in {64, 128} (got %d, %d)", s->d_qk, s->d_v);
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16 && G != 32 && G != 64)
      return fail(TLS_ERR_UNSUPPORTED, "GQA group size %d not in {1,2,4,8,16,32,64}", G);
    if (s->block_agg == 1 && G > 8 && s->kv_dtype != TLS_BF16)
      return fail(TLS_ERR_UNSUPPORTED, "max-over-heads block aggregation of fp32 keys supports up to 8 heads per group");
  }
  if (n_blocks_max(s) > tls::kMaxSelectKeys)
    return fail(TLS_ERR_UNSUPPORTED, "ceil(max_ctx / block_size) = %d > %d", n_blocks_max(s), tls::kMaxSelectKeys);
  if (s->k_b > 1024) return fail(TLS_ERR_UNSUPPORTED, "k_b %d > 1024", s->k_b);
  if (static_cast<long long>(s->k_b) * s->block_size > tls::kMaxSelectKeys)
    return fail(TLS_ERR_UNSUPPORTED, "k_b * block_size = %lld > %d", static_cast<long long>(s->k_b) * s->block_size,
                tls::kMaxSelectKeys);
  const bool r_ok = s->kv_dtype == TLS_BF16
                        ? (s->n_label == 8 || s->n_label == 16 || s->n_label == 32 || s->n_label == 64)
                        : (s->n_label == 4 || s->n_label == 8 || s->n_label == 16 || s->n_label == 32);
  if (!r_ok) return fail(TLS_ERR_UNSUPPORTED, "n_label %d unsupported for this dtype", s->n_label);
  if (s->n_label > s->d_qk) return fail(TLS_ERR_INVALID_ARG, "n_label > d_qk");
  if (s->slab_bits != 0 && s->slab_bits != 8) return fail(TLS_ERR_INVALID_ARG, "slab_bits %d", s->slab_bits);
  if (s->slab_bits == 8 && (s->kv_dtype != TLS_BF16 || s->n_label < 16))
    return fail(TLS_ERR_UNSUPPORTED, "the int8 label slab needs bf16 keys and n_label in {16, 32, 64}");
  return TLS_OK;
}

// Label slab layout: the slab of the K dtype, or int8 codes followed by the
// fp32 scales at the next multiple of 256 bytes.
size_t slab_codes_bytes(const tls_shape *s) {
  const size_t rows = static_cast<size_t>(s->batch) * s->n_kv_heads * s->max_ctx * s->n_label;
  return s->slab_bits == 8 ? rows : rows * (s->kv_dtype == TLS_BF16 ? 2 : 4);
}
size_t slab_scales_offset(const tls_shape *s) { return (slab_codes_bytes(s) + 255) / 256 * 256; }
size_t slab_total_bytes(const tls_shape *s) {
  if (s->slab_bits != 8) return slab_codes_bytes(s);
  return slab_scales_offset(s) + sizeof(float) * static_cast<size_t>(s->batch) * s->n_kv_heads * s->n_label;
}
const float *slab_scales(const tls_shape *s, const void *slab) {
  if (s->slab_bits != 8) return nullptr;
  return reinterpret_cast<const float *>(static_cast<const char *>(slab) + slab_scales_offset(s));
}

#define CHECK_PTR(p, a)                                                                          \
  do {                                                                                           \
    if (!(p)) return fail(TLS_ERR_INVALID_ARG, "%s is NULL", #p);                                \
    if (!aligned((p), (a))) return fail(TLS_ERR_INVALID_ARG, "%s is not %d-byte aligned", #p, a); \
  } while (0)

float scale_of(const tls_shape *s) {
  return s->softmax_scale > 0.f ? s->softmax_scale : 1.0f / std::sqrt(static_cast<float>(s->d_qk));
}

tls::AttnArgs attn_args(const tls_shape *s) {
  tls::AttnArgs a{};
  a.batch = s->batch;
  a.n_q_heads = s->n_q_heads;
  a.n_kv_heads = s->n_kv_heads;
  a.d_qk = s->d_qk;
  a.d_v = s->d_v;
  a.v_is_k_prefix = s->v_is_k_prefix;
  a.block_size = s->block_size;
  a.n_blocks_max = n_blocks_max(s);
  a.max_ctx = s->max_ctx;
  a.k_t = s->k_t;
  a.dtype = s->kv_dtype;
  a.out_dtype = s->out_dtype;
  a.scale_log2 = scale_of(s) * 1.4426950408889634f;
  a.num_sms = device_sms();
  return a;
}

// Workspace layout (attention only): the split-KV partials, 256-byte aligned.
struct WsLayout {
  size_t part_off, part_bytes, total;
};

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool ws_layout(const tls_shape *s, bool paged, WsLayout *w) {
  tls::AttnArgs a = attn_args(s);
  a.paged = paged;
  tls::AttnPlan p;
  if (!tls::attn_plan(a, &p)) return false;
  w->part_off = 0;
  w->part_bytes = up256(p.part_floats * sizeof(float));
  w->total = w->part_off + w->part_bytes;
  return true;
}

// tls_decode_step's workspace: the attention partials (or, before the
// attention runs, the step's block scores) from offset 0, then one readiness
// word per group at this offset.
size_t ready_words_offset(const tls_shape *s) {
  WsLayout w, wp;
  size_t body = ws_layout(s, false, &w) ? w.total : 0;
  if (!s->v_is_k_prefix && ws_layout(s, true, &wp)) body = std::max(body, wp.total);
  const size_t scores = up256(static_cast<size_t>(s->batch) * s->n_kv_heads * n_blocks_max(s) * sizeof(float));
  return up256(std::max(body, scores));
}

// Then the folded queries of the two-phase selection ([B*H_kv][2 d] fp32) at
// this offset.
size_t fold_offset(const tls_shape *s) {
  return ready_words_offset(s) + up256(static_cast<size_t>(s->batch) * s->n_kv_heads * sizeof(int));
}

// The library's device error word: one int per GPU, zero until a kernel's
// bounded wait gives up (bits kErrAttnWait, kErrSelectWait).
__device__ int g_device_error;

constexpr int kMaxDevices = 64;
std::mutex g_err_mu;
int *g_err_word[kMaxDevices] = {};

}  // namespace

namespace tls {
int *device_error_word() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_err_mu);
  if (!g_err_word[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    g_err_word[dev] = static_cast<int *>(p);
  }
  return g_err_word[dev];
}
}  // namespace tls

namespace tls {
tls_status set_error(tls_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}
}  // namespace tls

extern "C" {

const char *tls_version(void) { return "tls 0.1 sm_100a"; }

const char *tls_last_error(void) { return g_err.c_str(); }

size_t tls_workspace_size(const tls_shape *s) {
  if (check_shape(s) != TLS_OK) return 0;
  WsLayout w;
  if (!ws_layout(s, false, &w)) {
    fail(TLS_ERR_UNSUPPORTED, "no attention plan for this shape");
    return 0;
  }
  return fold_offset(s) + up256(static_cast<size_t>(s->batch) * s->n_kv_heads * 2 * s->d_qk * sizeof(float));
}

size_t tls_slab_bytes(const tls_shape *s) {
  if (check_shape(s) != TLS_OK) return 0;
  return slab_total_bytes(s);
}

tls_status tls_build_block_meta(const tls_shape *s, const void *K, const int32_t *seq_lens, const int32_t *label_idx,
                                void *meta_out, void *slab_out, void *stream) {
  tls_status st = check_shape(s);
  if (st != TLS_OK) return st;
  if (s->batch == 0) return TLS_OK;
  CHECK_PTR(K, 16);
  CHECK_PTR(seq_lens, 4);
  CHECK_PTR(meta_out, 16);
  if (slab_out) {
    CHECK_PTR(label_idx, 4);
    CHECK_PTR(slab_out, 16);
  }
  tls::MetaArgs a{K, seq_lens, label_idx, meta_out, slab_out, s->batch, s->n_kv_heads, s->d_qk, s->block_size,
                  n_blocks_max(s), s->max_ctx, s->n_label, s->kv_dtype};
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  st = cuda_status(tls::launch_build_meta(a, cs), "build_meta launch");
  if (st != TLS_OK || !slab_out) return st;
  if (s->slab_bits == 8) {
    // the scales come from the block summary just written (stream order)
    float *scales = const_cast<float *>(slab_scales(s, slab_out));
    st = cuda_status(tls::launch_label_scales(a, scales, cs), "label_scales launch");
    if (st != TLS_OK) return st;
    return cuda_status(tls::launch_build_slab_q8(a, scales, cs), "build_slab_q8 launch");
  }
  return cuda_status(tls::launch_build_slab(a, cs), "build_slab launch");
}

tls_status tls_append_tokens(const tls_shape *s, const void *K, const int32_t *old_lens, const int32_t *new_lens,
                             int32_t max_append, const int32_t *label_idx, void *meta, void *slab, void *stream) {
  tls_status st = check_shape(s);
  if (st != TLS_OK) return st;
  if (s->batch == 0 || max_append == 0) return TLS_OK;
  if (max_append < 0 || max_append > s->max_ctx)
    return fail(TLS_ERR_INVALID_ARG, "max_append %d outside [0, max_ctx]", max_append);
  CHECK_PTR(K, 16);
  CHECK_PTR(old_lens, 4);
  CHECK_PTR(new_lens, 4);
  CHECK_PTR(meta, 16);
  if (slab) {
    if (s->slab_bits == 8)  // an append can move a channel's scale and so every code of the group
      return fail(TLS_ERR_UNSUPPORTED, "tls_append_tokens does not update an int8 label slab; rebuild it");
    CHECK_PTR(label_idx, 4);
    CHECK_PTR(slab, 4);
  }
  tls::AppendArgs a{{K, nullptr, label_idx, meta, slab, s->batch, s->n_kv_heads, s->d_qk, s->block_size,
                     n_blocks_max(s), s->max_ctx, s->n_label, s->kv_dtype},
                    old_lens, new_lens, max_append, tls::device_error_word()};
  return cuda_status(tls::launch_append_tokens(a, static_cast<cudaStream_t>(stream)), "append_tokens launch");
}

// block_agg 1: the per-head bounds as a tcgen05 GEMM into `scores` (then the
// clusters only select, a.from_scores), when the shape allows it and there is
// room for the scores; otherwise the CUDA-core path (up to 8 heads per group).
// Returns TLS_OK with a.from_scores set when the scores were launched.
static tls_status agg_max_scores(const tls_shape *s, tls::BlockScoreArgs &a, float *scores, cudaStream_t cs) {
  const int G = s->n_q_heads / s->n_kv_heads;
  if (scores && tls::block_scores_max_tc_supported(s->kv_dtype, s->d_qk, G)) {
    a.scores = scores;
    tls_status st = cuda_status(tls::launch_block_scores_max_tc(a, device_sms(), cs), "block_scores_max_tc launch");
    if (st != TLS_OK) return st;
    a.from_scores = 1;
    return TLS_OK;
  }
  if (G > 8 || s->v_is_k_prefix)
    return fail(TLS_ERR_WORKSPACE,
                "max-over-heads block scores with %d heads per group need block_score_out or a workspace of "
                "tls_workspace_size bytes",
                G);
  return TLS_OK;  // CUDA-core path
}

tls_status tls_block_score_topk(const tls_shape *s, const void *q, const void *meta, const int32_t *seq_lens,
                                int32_t *block_idx_out, float *block_score_out, void *ws, size_t ws_bytes,
                                void *stream) {
  tls_status st = check_shape(s);
  if (st != TLS_OK) return st;
  if (s->batch == 0) return TLS_OK;
  CHECK_PTR(q, 16);
  CHECK_PTR(meta, 16);
  CHECK_PTR(seq_lens, 4);
  CHECK_PTR(block_idx_out, 4);
  if (block_score_out && !aligned(block_score_out, 4)) return fail(TLS_ERR_INVALID_ARG, "block_score_out misaligned");
  tls::BlockScoreArgs a{q, meta, seq_lens, block_score_out, block_idx_out, s->batch, s->n_q_heads, s->n_kv_heads,
                        s->d_qk, s->block_size, n_blocks_max(s), s->max_ctx, s->k_b, s->kv_dtype,
                        tls::device_error_word(), s->block_agg};
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (s->block_agg == 1) {
    // the scores of the tensor-core path go to block_score_out, else to the workspace
    const size_t need = static_cast<size_t>(s->batch) * s->n_kv_heads * n_blocks_max(s) * sizeof(float);
    float *scores = block_score_out ? block_score_out
                                    : (ws && ws_bytes >= need && aligned(ws, 16) ? static_cast<float *>(ws) : nullptr);
    st = agg_max_scores(s, a, scores, cs);
    if (st != TLS_OK) return st;
  }
  return cuda_status(tls::launch_block_select(a, cs), "block_select launch");
}

tls_status tls_token_score_topk(const tls_shape *s, const void *q, const void *slab, const int32_t *label_idx,
                                const int32_t *block_idx, const int32_t *seq_lens, int32_t *token_idx_out,
                                float *token_score_out, void *ws, size_t ws_bytes, void *stream) {
  tls_status st = check_shape(s);
  if (st != TLS_OK) return st;
  if (s->batch == 0) return TLS_OK;
  CHECK_PTR(q, 16);
  CHECK_PTR(slab, 16);
  CHECK_PTR(label_idx, 4);
  CHECK_PTR(block_idx, 4);
  CHECK_PTR(seq_lens, 4);
  CHECK_PTR(token_idx_out, 4);
  if (token_score_out && !aligned(token_score_out, 4)) return fail(TLS_ERR_INVALID_ARG, "token_score_out misaligned");
  tls::TokenArgs a{q, slab, label_idx, block_idx, seq_lens, token_idx_out, token_score_out, s->batch, s->n_q_heads,
                   s->n_kv_heads, s->d_qk, s->block_size, n_blocks_max(s), s->max_ctx, s->n_label, s->k_b, s->k_t,
                   s->kv_dtype, tls::device_error_word(), slab_scales(s, slab)};
  (void)ws;  // the selection keeps its keys in on-chip memory: no workspace
  (void)ws_bytes;
  return cuda_status(tls::launch_token_select(a, static_cast<cudaStream_t>(stream)), "token_select launch");
}

// Stages 1-4.  scratch: room for the step's block scores when the caller
// passes no block_score_out (tls_decode_step lends its workspace), or NULL.
static tls_status select_step_impl(const tls_shape *s, const void *q, const void *meta, const void *slab,
                                   const int32_t *label_idx, const int32_t *seq_lens, int32_t *block_idx_out,
                                   int32_t *token_idx_out, float *block_score_out, float *token_score_out,
                                   float *scratch, float *qfold, int **ready, int seq, void *stream);

tls_status tls_select_step(const tls_shape *s, const void *q, const void *meta, const void *slab,
                           const int32_t *label_idx, const int32_t *seq_lens, int32_t *block_idx_out,
                           int32_t *token_idx_out, float *block_score_out, float *token_score_out, void *stream) {
  return select_step_impl(s, q, meta, slab, label_idx, seq_lens, block_idx_out, token_idx_out, block_score_out,
                          token_score_out, nullptr, nullptr, nullptr, 0, stream);
}

static tls_status select_step_impl(const tls_shape *s, const void *q, const void *meta, const void *slab,
                                   const int32_t *label_idx, const int32_t *seq_lens, int32_t *block_idx_out,
                                   int32_t *token_idx_out, float *block_score_out, float *token_score_out,
                                   float *scratch, float *qfold, int **ready, int seq, void *stream) {
  tls_status st = check_shape(s);
  if (st != TLS_OK) return st;
  if (s->batch == 0) return TLS_OK;
  CHECK_PTR(q, 16);
  CHECK_PTR(meta, 16);
  CHECK_PTR(slab, 16);
  CHECK_PTR(label_idx, 4);
  CHECK_PTR(seq_lens, 4);
  CHECK_PTR(block_idx_out, 4);
  CHECK_PTR(token_idx_out, 4);
  if (block_score_out && !aligned(block_score_out, 4)) return fail(TLS_ERR_INVALID_ARG, "block_score_out misaligned");
  if (token_score_out && !aligned(token_score_out, 4)) return fail(TLS_ERR_INVALID_ARG, "token_score_out misaligned");
  int *err = tls::device_error_word();
  tls::BlockScoreArgs a{q, meta, seq_lens, block_score_out, block_idx_out, s->batch, s->n_q_heads, s->n_kv_heads,
                        s->d_qk, s->block_size, n_blocks_max(s), s->max_ctx, s->k_b, s->kv_dtype, err, s->block_agg};
  tls::TokenArgs t{q, slab, label_idx, block_idx_out, seq_lens, token_idx_out, token_score_out, s->batch, s->n_q_heads,
                   s->n_kv_heads, s->d_qk, s->block_size, n_blocks_max(s), s->max_ctx, s->n_label, s->k_b, s->k_t,
                   s->kv_dtype, err, slab_scales(s, slab)};
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // The readiness words (*ready, when given) are set by the select_step launch
  // only; a path without it reports NULL back so that nothing waits on them.
  t.ready = ready ? *ready : nullptr;
  t.seq = seq;
  if (s->block_agg == 1) {
    st = agg_max_scores(s, a, block_score_out ? block_score_out : scratch, cs);
    if (st != TLS_OK) return st;
    if (a.from_scores)  // tensor-core scores: the cluster launch selects blocks, then tokens
      return cuda_status(tls::launch_select_step(a, t, cs), "select_step launch");
    // CUDA-core max-over-heads scores: the two separate launches
    if (ready) *ready = nullptr;
    t.ready = nullptr;
    st = cuda_status(tls::launch_block_select(a, cs), "block_select launch");
    if (st != TLS_OK) return st;
    return cuda_status(tls::launch_token_select(t, cs), "token_select launch");
  }
  // Few groups: too few clusters to keep HBM busy streaming the summary, so a
  // grid over all SMs scores every block first and the clusters only select.
  float *scores = block_score_out ? block_score_out : scratch;
  const size_t summary_bytes = static_cast<size_t>(s->batch) * s->n_kv_heads * n_blocks_max(s) * 2 * s->d_qk *
                               (s->kv_dtype == TLS_BF16 ? 2 : 4);
  const int G = s->n_q_heads / s->n_kv_heads;
  if (G <= 16) qfold = nullptr;  // a few heads: each phase-1 CTA folds them faster than an extra launch
  if (scores && tls::select_two_phase(s->batch * s->n_kv_heads, G, device_sms(), summary_bytes, qfold != nullptr)) {
    a.scores = scores;
    if (qfold) {  // many heads: the queries folded once per group, not by every phase-1 CTA
      a.qfold = qfold;
      st = cuda_status(tls::launch_query_fold(a, cs), "query_fold launch");
      if (st != TLS_OK) return st;
    }
    st = cuda_status(tls::launch_block_scores(a, device_sms(), cs), "block_scores launch");
    if (st != TLS_OK) return st;
    a.from_scores = 1;
  }
  return cuda_status(tls::launch_select_step(a, t, cs), "select_step launch");
}

tls_status tls_select_step_ws(const tls_shape *s, const void *q, const void *meta, const void *slab,
                              const int32_t *label_idx, const int32_t *seq_lens, int32_t *block_idx_out,
                              int32_t *token_idx_out, float *block_score_out, float *token_score_out, void *ws,
                              size_t ws_bytes, void *stream) {
  tls_status st = check_shape(s);
  if (st != TLS_OK) return st;
  if (s->batch == 0) return TLS_OK;
  const size_t need = tls_workspace_size(s);
  if (!need) return fail(TLS_ERR_UNSUPPORTED, "no workspace layout for this shape");
  if (!ws || ws_bytes < need || !aligned(ws, 256))
    return fail(TLS_ERR_WORKSPACE, "workspace too small or not 256-byte aligned (need %zu bytes)", need);
  return select_step_impl(s, q, meta, slab, label_idx, seq_lens, block_idx_out, token_idx_out, block_score_out,
                          token_score_out, static_cast<float *>(ws),
                          reinterpret_cast<float *>(static_cast<char *>(ws) + fold_offset(s)), nullptr, 0, stream);
}

static tls_status attn_common(const tls_shape *s, const void *q, const void *K, const void *V,
                              const int32_t *token_idx, const int32_t *slot_of_block, int32_t n_slots, void *out,
                              float *lse_out, void *ws, size_t ws_bytes, void *stream, bool paged,
                              const int *ready = nullptr, int seq = 0) {
  tls_status st = check_shape(s);
  if (st != TLS_OK) return st;
  if (s->batch == 0) return TLS_OK;
  CHECK_PTR(q, 16);
  CHECK_PTR(K, 16);
  if (!paged && !s->v_is_k_prefix) CHECK_PTR(V, 16);
  CHECK_PTR(token_idx, 4);
  CHECK_PTR(out, 16);
  if (lse_out && !aligned(lse_out, 4)) return fail(TLS_ERR_INVALID_ARG, "lse_out misaligned");
  if (paged) {
    if (s->v_is_k_prefix) return fail(TLS_ERR_UNSUPPORTED, "the block cache holds GQA K/V blocks only");
    CHECK_PTR(slot_of_block, 4);
    if (n_slots < 1) return fail(TLS_ERR_INVALID_ARG, "n_slots < 1");
  }
  WsLayout w;
  if (!ws_layout(s, paged, &w)) return fail(TLS_ERR_UNSUPPORTED, "no attention plan for this shape");
  if (!ws || ws_bytes < w.total || !aligned(ws, 256))
    return fail(TLS_ERR_WORKSPACE, "workspace too small or not 256-byte aligned (need %zu bytes)", w.total);
  tls::AttnArgs a = attn_args(s);
  a.q = q;
  a.K = K;
  a.V = V;
  a.token_idx = token_idx;
  a.slot_of_block = slot_of_block;
  a.n_slots = n_slots;
  a.out = out;
  a.lse = lse_out;
  a.part = reinterpret_cast<float *>(static_cast<char *>(ws) + w.part_off);
  a.err = tls::device_error_word();
  a.paged = paged;
  a.ready = ready;
  a.seq = seq;
  tls::AttnPlan p;
  if (!tls::attn_plan(a, &p)) return fail(TLS_ERR_UNSUPPORTED, "no attention plan for this shape");
  return cuda_status(tls::launch_attention(a, p, static_cast<cudaStream_t>(stream)), "attention launch");
}

tls_status tls_sparse_attn_decode(const tls_shape *s, const void *q, const void *K, const void *V,
                                  const int32_t *token_idx, void *out, float *lse_out, void *ws, size_t ws_bytes,
                                  void *stream) {
  return attn_common(s, q, K, V, token_idx, nullptr, 0, out, lse_out, ws, ws_bytes, stream, false);
}

tls_status tls_sparse_attn_decode_paged(const tls_shape *s, const void *q, const void *cache,
                                        const int32_t *slot_of_block, int32_t n_slots, const int32_t *token_idx,
                                        void *out, float *lse_out, void *ws, size_t ws_bytes, void *stream) {
  return attn_common(s, q, cache, nullptr, token_idx, slot_of_block, n_slots, out, lse_out, ws, ws_bytes, stream,
                     true);
}

static tls_status offload_check(const tls_shape *s, int32_t n_slots) {
  tls_status st = check_shape(s);
  if (st != TLS_OK) return st;
  if (s->v_is_k_prefix) return fail(TLS_ERR_UNSUPPORTED, "the block cache holds GQA K/V blocks only");
  if (n_slots < 1 || n_slots > 4096) return fail(TLS_ERR_INVALID_ARG, "n_slots %d not in [1, 4096]", n_slots);
  return TLS_OK;
}

tls_status tls_offload_reset(const tls_shape *s, int32_t n_slots, int32_t *slot_of_block, int32_t *block_of_slot,
                             void *stream) {
  tls_status st = offload_check(s, n_slots);
  if (st != TLS_OK) return st;
  if (s->batch == 0) return TLS_OK;
  CHECK_PTR(slot_of_block, 4);
  CHECK_PTR(block_of_slot, 4);
  tls::OffloadArgs a{};
  a.slot_of_block = slot_of_block;
  a.block_of_slot = block_of_slot;
  a.batch = s->batch;
  a.n_kv_heads = s->n_kv_heads;
  a.n_blocks_max = n_blocks_max(s);
  a.n_slots = n_slots;
  return cuda_status(tls::launch_offload_reset(a, static_cast<cudaStream_t>(stream)), "offload_reset launch");
}

tls_status tls_prefetch_diff(const tls_shape *s, int32_t n_slots, const void *host_kv, void *cache,
                             int32_t *slot_of_block, int32_t *block_of_slot, const int32_t *prev_block_idx,
                             const int32_t *next_block_idx, int32_t *n_new_out, int32_t *jobs_ws, void *stream) {
  tls_status st = offload_check(s, n_slots);
  if (st != TLS_OK) return st;
  if (s->batch == 0) return TLS_OK;
  CHECK_PTR(host_kv, 16);
  CHECK_PTR(cache, 16);
  CHECK_PTR(slot_of_block, 4);
  CHECK_PTR(block_of_slot, 4);
  CHECK_PTR(next_block_idx, 4);
  CHECK_PTR(n_new_out, 4);
  CHECK_PTR(jobs_ws, 4);
  if (prev_block_idx && !aligned(prev_block_idx, 4)) return fail(TLS_ERR_INVALID_ARG, "prev_block_idx misaligned");
  void *dev_host = nullptr;
  cudaError_t e = cudaHostGetDevicePointer(&dev_host, const_cast<void *>(host_kv), 0);
  if (e != cudaSuccess || !dev_host) {
    cudaGetLastError();  // clear the error this query recorded
    return fail(TLS_ERR_INVALID_ARG, "host_kv is not page-locked host memory visible to the device");
  }
  tls::OffloadArgs a{};
  a.host_kv = dev_host;
  a.cache = cache;
  a.slot_of_block = slot_of_block;
  a.block_of_slot = block_of_slot;
  a.prev_block_idx = prev_block_idx;
  a.next_block_idx = next_block_idx;
  a.n_new = n_new_out;
  a.jobs = jobs_ws;
  a.batch = s->batch;
  a.n_kv_heads = s->n_kv_heads;
  a.d = s->d_qk;
  a.block_size = s->block_size;
  a.n_blocks_max = n_blocks_max(s);
  a.k_b = s->k_b;
  a.n_slots = n_slots;
  a.dtype = s->kv_dtype;
  return cuda_status(tls::launch_prefetch_diff(a, static_cast<cudaStream_t>(stream)), "prefetch_diff launch");
}

tls_status tls_decode_step(const tls_shape *s, const void *q, const void *meta, const void *slab,
                           const int32_t *label_idx, const int32_t *seq_lens, const void *K, const void *V,
                           int32_t *block_idx_out, int32_t *token_idx_out, void *out, float *lse_out,
                           float *block_score_out, float *token_score_out, void *ws, size_t ws_bytes, void *stream) {
  tls_status st = check_shape(s);
  if (st != TLS_OK) return st;
  if (s->batch == 0) return TLS_OK;
  CHECK_PTR(q, 16);
  CHECK_PTR(meta, 16);
  CHECK_PTR(slab, 16);
  CHECK_PTR(label_idx, 4);
  CHECK_PTR(seq_lens, 4);
  CHECK_PTR(K, 16);
  if (!s->v_is_k_prefix) CHECK_PTR(V, 16);
  CHECK_PTR(block_idx_out, 4);
  CHECK_PTR(token_idx_out, 4);
  CHECK_PTR(out, 16);
  if (lse_out && !aligned(lse_out, 4)) return fail(TLS_ERR_INVALID_ARG, "lse_out misaligned");
  if (block_score_out && !aligned(block_score_out, 4)) return fail(TLS_ERR_INVALID_ARG, "block_score_out misaligned");
  if (token_score_out && !aligned(token_score_out, 4)) return fail(TLS_ERR_INVALID_ARG, "token_score_out misaligned");
  const size_t need = tls_workspace_size(s);  // checked before anything is enqueued
  if (!need) return fail(TLS_ERR_UNSUPPORTED, "no workspace layout for this shape");
  if (!ws || ws_bytes < need || !aligned(ws, 256))
    return fail(TLS_ERR_WORKSPACE, "workspace too small or not 256-byte aligned (need %zu bytes)", need);
  // The block scores may borrow the workspace: they are consumed by the
  // selection launch before the attention writes its partials there.  When
  // the attention is the warp-MMA kernel, the selection launch marks each
  // group ready in the workspace's readiness words and lets the attention
  // start early: its warps wait per group instead of for the whole grid.
  tls::AttnArgs probe = attn_args(s);
  tls::AttnPlan plan;
  const bool overlap = tls::attn_plan(probe, &plan) && plan.impl == 2;
  int *ready = overlap ? reinterpret_cast<int *>(static_cast<char *>(ws) + ready_words_offset(s)) : nullptr;
  static std::atomic<int> g_seq{0};
  const int seq = overlap ? (g_seq.fetch_add(1) & 0x3fffffff) + 1 : 0;
  st = select_step_impl(s, q, meta, slab, label_idx, seq_lens, block_idx_out, token_idx_out, block_score_out,
                        token_score_out, static_cast<float *>(ws),
                        reinterpret_cast<float *>(static_cast<char *>(ws) + fold_offset(s)), &ready, seq, stream);
  if (st != TLS_OK) return st;
  return attn_common(s, q, K, V, token_idx_out, nullptr, 0, out, lse_out, ws, ws_bytes, stream, false, ready, seq);
}

tls_status tls_wait_event(void *event, int32_t timeout_ms) {
  if (!event) return fail(TLS_ERR_INVALID_ARG, "event is NULL");
  if (timeout_ms < 0) timeout_ms = 0;
  const auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    cudaError_t e = cudaEventQuery(static_cast<cudaEvent_t>(event));
    if (e == cudaSuccess) return TLS_OK;
    if (e != cudaErrorNotReady) return cuda_status(e, "event query");
    const auto ms =
        std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0).count();
    if (ms >= timeout_ms) return fail(TLS_ERR_TIMEOUT, "event not complete after %d ms", timeout_ms);
    std::this_thread::sleep_for(std::chrono::microseconds(200));
  }
}

tls_status tls_device_error(int32_t *flags_out, int32_t clear) {
  if (!flags_out) return fail(TLS_ERR_INVALID_ARG, "flags_out is NULL");
  int *w = tls::device_error_word();
  if (!w) return fail(TLS_ERR_CUDA, "the device error word could not be looked up on the current device");
  int v = 0;
  tls_status st = cuda_status(cudaMemcpy(&v, w, sizeof v, cudaMemcpyDeviceToHost), "reading the device error word");
  if (st != TLS_OK) return st;
  *flags_out = v;
  if (clear && v) return cuda_status(cudaMemset(w, 0, sizeof v), "clearing the device error word");
  return TLS_OK;
}

}  // extern "C"
