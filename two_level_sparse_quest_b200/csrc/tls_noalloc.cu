// tls_noalloc.cu -- block selection for callers that cannot allocate device memory.
//
// tls_block_score_topk_noalloc serves code that runs inside another runtime's
// launch hook (an inference-engine plugin, a serving loop that forbids device
// allocation once it is running), where cudaMalloc is not allowed or would
// synchronise the device in the middle of a step: it needs no buffer besides
// the inputs and the block_idx output, and it leaves the step's fp32 block
// scores in a fixed array that lives in the library's own device memory
// (g_noalloc_scores below).  The selection itself keeps its keys on chip, so
// the array only receives the scores; nothing here allocates.
//
// The array is 4 MiB (kNoAllocMaxScores fp32 scores) and exists on every GPU
// that loads the library, until the process exits.  It holds
// batch * n_kv_heads * ceil(max_ctx / block_size) scores at most; larger shapes
// are rejected.  Every call writes the scores of all its blocks, so nothing in
// the array has to start at zero; the array keeps the last call's scores.  All
// calls on one device share the array: calls whose kernels overlap on the GPU
// (two streams, or two threads) overwrite each other's scores.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "tls.h"
#include "tls_internal.h"

namespace {

constexpr size_t kNoAllocMaxScores = size_t(1) << 20;  // 4 MiB of fp32 scores

static __device__ __align__(256) float g_noalloc_scores[kNoAllocMaxScores];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float *g_scores_on_device[kMaxDevices] = {};

// Device address of g_noalloc_scores on the current device.  The host-side
// name is only a stand-in for the symbol; the address comes from
// cudaGetSymbolAddress, once per device, with that device current.
tls_status scratch_for_current_device(float **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tls::set_error(TLS_ERR_CUDA, "cudaGetDevice failed: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return tls::set_error(TLS_ERR_UNSUPPORTED, "device index %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scores_on_device[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scores);
    if (e != cudaSuccess || !p)
      return tls::set_error(TLS_ERR_CUDA, "cudaGetSymbolAddress of the built-in score array failed: %s",
                            cudaGetErrorString(e));
    g_scores_on_device[dev] = static_cast<float *>(p);
  }
  *out = g_scores_on_device[dev];
  return TLS_OK;
}

}  // namespace

extern "C" {

tls_status tls_block_score_topk_noalloc(const tls_shape *s, const void *q, const void *meta,
                                        const int32_t *seq_lens, int32_t *block_idx_out, void *stream) {
  // Shapes the regular entry point rejects are passed to it unchanged so that
  // the status and message are the usual ones.
  if (s && s->batch > 0 && s->n_kv_heads > 0 && s->block_size > 0 && s->max_ctx > 0) {
    const size_t n_blocks = (static_cast<size_t>(s->max_ctx) + s->block_size - 1) / s->block_size;
    const size_t need = static_cast<size_t>(s->batch) * s->n_kv_heads * n_blocks;
    if (need > kNoAllocMaxScores)
      return tls::set_error(TLS_ERR_UNSUPPORTED,
                            "tls_block_score_topk_noalloc: shape needs %zu block scores "
                            "(batch * n_kv_heads * ceil(max_ctx / block_size)); the built-in array holds %zu",
                            need, kNoAllocMaxScores);
    float *scores = nullptr;
    tls_status st = scratch_for_current_device(&scores);
    if (st != TLS_OK) return st;
    return tls_block_score_topk(s, q, meta, seq_lens, block_idx_out, scores, nullptr, 0, stream);
  }
  return tls_block_score_topk(s, q, meta, seq_lens, block_idx_out, nullptr, nullptr, 0, stream);
}

tls_status tls_noalloc_read_scores(float *dst, size_t count, void *stream) {
  if (count == 0) return TLS_OK;
  if (!dst) return tls::set_error(TLS_ERR_INVALID_ARG, "dst is NULL");
  if (count > kNoAllocMaxScores)
    return tls::set_error(TLS_ERR_INVALID_ARG, "count %zu exceeds the built-in array (%zu scores)", count,
                          kNoAllocMaxScores);
  float *scores = nullptr;
  tls_status st = scratch_for_current_device(&scores);
  if (st != TLS_OK) return st;
  cudaError_t e = cudaMemcpyAsync(dst, scores, count * sizeof(float), cudaMemcpyDefault,
                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess)
    return tls::set_error(TLS_ERR_CUDA, "copying the built-in score array: %s", cudaGetErrorString(e));
  return TLS_OK;
}

}  // extern "C"
