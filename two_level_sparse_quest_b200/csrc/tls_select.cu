// tls_select.cu -- the two selection stages of the AsyncTLS decode step.
//
// Stage 1 (block score, gist.science (de) section 2.A "Stufe 1" + "Optimierung";
// (es) section 2.A.1): the Quest-style bound of a block j for query head h,
//     u_{h,j} = sum_i max(q_{h,i} M_{j,i}, q_{h,i} m_{j,i}) = q_h^+ . M_j + q_h^- . m_j,
// summed over the heads h of one KV head.  The contraction over heads is done
// first (Q^+ = sum_h q_h^+, Q^- = sum_h q_h^-, fp32 in shared memory), so the
// block summary [M_j ; m_j] (2d values per block, contiguous) is streamed from
// HBM exactly once and dotted with [Q^+ ; Q^-]: 2 flop per stored element,
// memory-bound.  A warp owns whole summary rows; each lane loads 16-byte chunks
// (coalesced, non-allocating loads) and the row sum is a segmented warp
// reduction.
// Stage 2 (top-K_b): one CTA per group, scores as order-preserving keys in
// shared memory, block radix select, index-ordered compaction (ties -> lower id).
// Stages 3+4 (token score + top-K_t, (de) section 2.A "Stufe 2", (es) section
// 2.A.2): one CTA per group gathers the label-channel slab rows of the
// candidate tokens (a block's rows are contiguous), scores them against
// Qbar_L = sum_h q_h[L] in fp32, keeps the keys in shared memory and selects.
#include "tls_device.cuh"
#include "tls_internal.h"

namespace tls {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreUnroll = 4;

// NCH: 16-byte chunks per summary row (2 * d * bytes / 16).
template <typename E, int NCH>
__global__ void __launch_bounds__(kScoreThreads) block_score_kernel(BlockScoreArgs a, int rows_per_cta) {
  constexpr int EPC = E::kEPC;
  constexpr int LPR = NCH < 32 ? NCH : 32;            // lanes per row
  constexpr int RPW = 32 / LPR;                       // rows per warp step
  constexpr int CPL = (NCH + 31) / 32;                // chunks per lane
  constexpr int NWARP = kScoreThreads / 32;
  extern __shared__ float qpm[];                      // [2d]: Q^+ then Q^-
  const int group = blockIdx.y;
  const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int d = a.d;
  const int seq = min(max(a.seq_lens[b], 0), a.max_ctx);
  const int nb = (seq + a.block_size - 1) / a.block_size;
  // Fold the group's heads into the sign-split query.
  for (int i = threadIdx.x; i < d; i += kScoreThreads) {
    float pos = 0.f, neg = 0.f;
    for (int hh = 0; hh < G; ++hh) {
      float v = load_elem<E>(a.q, (static_cast<size_t>(b) * a.n_q_heads + g * G + hh) * d + i);
      pos += fmaxf(v, 0.f);
      neg += fminf(v, 0.f);
    }
    qpm[i] = pos;
    qpm[d + i] = neg;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPR, cl = lane % LPR;  // row within the warp step, chunk lane
  float qr[CPL][EPC];
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    const int c = cl + j * 32;
#pragma unroll
    for (int e = 0; e < EPC; ++e) qr[j][e] = (c < NCH) ? qpm[c * EPC + e] : 0.f;
  }
  const int r0 = blockIdx.x * rows_per_cta;
  const int r1 = min(r0 + rows_per_cta, a.n_blocks_max);
  const char *meta = static_cast<const char *>(a.meta) + static_cast<size_t>(group) * a.n_blocks_max * (NCH * 16);
  float *out = a.scores + static_cast<size_t>(group) * a.n_blocks_max;
  constexpr int STEP = NWARP * RPW;
  for (int rb = r0 + warp * RPW; rb < r1; rb += STEP * kScoreUnroll) {
    uint4 v[kScoreUnroll][CPL];
#pragma unroll
    for (int u = 0; u < kScoreUnroll; ++u) {
      const int row = rb + u * STEP + sub;
      const bool ok = row < r1 && row < nb;
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const int c = cl + j * 32;
        v[u][j] = (ok && c < NCH) ? ld_stream16(meta + static_cast<size_t>(row) * (NCH * 16) + c * 16)
                                  : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kScoreUnroll; ++u) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        float f[EPC];
        chunk_to_f32<E>(v[u][j], f);
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc = fmaf(qr[j][e], f[e], acc);
      }
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      const int row = rb + u * STEP + sub;
      if (cl == 0 && row < r1) out[row] = (row < nb) ? acc : -INFINITY;
    }
  }
}

constexpr int kTopkThreads = 1024;

__global__ void __launch_bounds__(kTopkThreads) block_topk_kernel(BlockScoreArgs a) {
  extern __shared__ uint32_t keys[];
  __shared__ int hist[256];
  __shared__ int sh[33];
  __shared__ int bc[2];
  const int group = blockIdx.x;
  const int b = group / a.n_kv_heads;
  const int seq = min(max(a.seq_lens[b], 0), a.max_ctx);
  const int nb = (seq + a.block_size - 1) / a.block_size;
  const float *sc = a.scores + static_cast<size_t>(group) * a.n_blocks_max;
  for (int i = threadIdx.x; i < nb; i += kTopkThreads) keys[i] = score_key(sc[i]);
  __syncthreads();
  int32_t *out = a.block_idx + static_cast<size_t>(group) * a.k_b;
  const int k = min(a.k_b, nb);
  if (k <= 0) {
    for (int i = threadIdx.x; i < a.k_b; i += kTopkThreads) out[i] = -1;
    return;
  }
  SelectResult r = block_radix_select<kTopkThreads>(keys, nb, k, hist, bc);
  block_ordered_compact<kTopkThreads>(keys, nb, r, k, out, a.k_b, [](int i) { return i; }, sh);
}

// RCH: 16-byte chunks per slab row (r * bytes / 16), 1..8.
constexpr int kTokThreads = 512;

template <typename E, int RCH>
__global__ void __launch_bounds__(kTokThreads) token_topk_kernel(TokenArgs a) {
  using S = typename E::storage;
  constexpr int EPC = E::kEPC;
  // candidates whose slab rows a thread loads before scoring them
  constexpr int kTokBatch = RCH <= 2 ? 4 : (RCH <= 4 ? 2 : 1);
  extern __shared__ uint32_t keys[];  // [k_b * bs]
  __shared__ int blk[1024];
  __shared__ float qbar[64];
  __shared__ int hist[256];
  __shared__ int sh[33];
  __shared__ int bc[2];
  const int group = blockIdx.x;
  const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int seq = min(max(a.seq_lens[b], 0), a.max_ctx);
  const int bs = a.block_size, r = a.n_label;
  for (int i = threadIdx.x; i < a.k_b; i += kTokThreads) {
    int v = a.block_idx[static_cast<size_t>(group) * a.k_b + i];
    blk[i] = (v >= 0 && v < a.n_blocks_max) ? v : -1;
  }
  for (int c = threadIdx.x; c < r; c += kTokThreads) {
    const int ch = a.label_idx[c];
    float s = 0.f;
    if (ch >= 0 && ch < a.d)
      for (int hh = 0; hh < G; ++hh)
        s += load_elem<E>(a.q, (static_cast<size_t>(b) * a.n_q_heads + g * G + hh) * a.d + ch);
    qbar[c] = s;
  }
  __syncthreads();
  float ql[RCH * EPC];
#pragma unroll
  for (int e = 0; e < RCH * EPC; ++e) ql[e] = qbar[e];  // r == RCH * EPC
  const int C = a.k_b * bs;
  const S *slab = static_cast<const S *>(a.slab) + static_cast<size_t>(group) * a.max_ctx * r;
  float *score_out = a.token_score ? a.token_score + static_cast<size_t>(group) * C : nullptr;
  int n_valid = 0;
  for (int base = 0; base < C; base += kTokThreads * kTokBatch) {
    uint4 v[kTokBatch][RCH];
    int tok[kTokBatch];
#pragma unroll
    for (int u = 0; u < kTokBatch; ++u) {
      const int j = base + u * kTokThreads + threadIdx.x;
      int t = -1;
      if (j < C) {
        const int bl = blk[j / bs];
        t = bl * bs + j % bs;
        if (bl < 0 || t >= seq) t = -1;
      }
      tok[u] = t;
#pragma unroll
      for (int c = 0; c < RCH; ++c)
        v[u][c] = t >= 0 ? ld_stream16(slab + static_cast<size_t>(t) * r + c * EPC) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kTokBatch; ++u) {
      const int j = base + u * kTokThreads + threadIdx.x;
      if (j >= C) continue;
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < RCH; ++c) {
        float f[EPC];
        chunk_to_f32<E>(v[u][c], f);
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc = fmaf(ql[c * EPC + e], f[e], acc);
      }
      const bool ok = tok[u] >= 0;
      keys[j] = ok ? score_key(acc) : 0u;
      n_valid += ok;
      if (score_out) score_out[j] = ok ? acc : -INFINITY;
    }
  }
  int total;
  block_excl_scan<kTokThreads>(n_valid, sh, total);  // also a barrier for keys[]
  int32_t *out = a.token_idx + static_cast<size_t>(group) * a.k_t;
  const int k = min(a.k_t, total);
  if (k <= 0) {
    for (int i = threadIdx.x; i < a.k_t; i += kTokThreads) out[i] = -1;
    return;
  }
  SelectResult res = block_radix_select<kTokThreads>(keys, C, k, hist, bc);
  block_ordered_compact<kTokThreads>(
      keys, C, res, k, out, a.k_t, [&](int j) { return blk[j / bs] * bs + j % bs; }, sh);
}

template <typename E, int NCH>
cudaError_t run_block_score(const BlockScoreArgs &a, cudaStream_t st) {
  const int groups = a.batch * a.n_kv_heads;
  // Enough CTAs to cover every SM several times; rows split evenly per group.
  const int want = 4 * a.num_sms;
  int splits = (want + groups - 1) / groups;
  const int min_rows = 8 * (kScoreThreads / 32);
  splits = max(1, min(splits, (a.n_blocks_max + min_rows - 1) / min_rows));
  const int rows = (a.n_blocks_max + splits - 1) / splits;
  splits = (a.n_blocks_max + rows - 1) / rows;
  dim3 grid(splits, groups);
  block_score_kernel<E, NCH><<<grid, kScoreThreads, 2 * a.d * sizeof(float), st>>>(a, rows);
  return cudaGetLastError();
}

template <typename E, int RCH>
cudaError_t run_token_topk(const TokenArgs &a, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(a.k_b) * a.block_size * sizeof(uint32_t);
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(token_topk_kernel<E, RCH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kMaxSelectKeys * static_cast<int>(sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  token_topk_kernel<E, RCH><<<a.batch * a.n_kv_heads, kTokThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_score(const BlockScoreArgs &a, cudaStream_t st) {
  const int nch = 2 * a.d * (a.dtype == 1 ? 2 : 4) / 16;
  if (a.dtype == 1) {
    switch (nch) {
      case 16: return run_block_score<BF16, 16>(a, st);
      case 32: return run_block_score<BF16, 32>(a, st);
      case 144: return run_block_score<BF16, 144>(a, st);
    }
  } else {
    switch (nch) {
      case 32: return run_block_score<F32, 32>(a, st);
      case 64: return run_block_score<F32, 64>(a, st);
    }
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_block_topk(const BlockScoreArgs &a, cudaStream_t st) {
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(block_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kMaxSelectKeys * static_cast<int>(sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const size_t smem = static_cast<size_t>(a.n_blocks_max) * sizeof(uint32_t);
  block_topk_kernel<<<a.batch * a.n_kv_heads, kTopkThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_token_topk(const TokenArgs &a, cudaStream_t st) {
  const int rch = a.n_label * (a.dtype == 1 ? 2 : 4) / 16;
  switch (rch) {
    case 1: return a.dtype == 1 ? run_token_topk<BF16, 1>(a, st) : run_token_topk<F32, 1>(a, st);
    case 2: return a.dtype == 1 ? run_token_topk<BF16, 2>(a, st) : run_token_topk<F32, 2>(a, st);
    case 4: return a.dtype == 1 ? run_token_topk<BF16, 4>(a, st) : run_token_topk<F32, 4>(a, st);
    case 8: return a.dtype == 1 ? run_token_topk<BF16, 8>(a, st) : run_token_topk<F32, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tls
