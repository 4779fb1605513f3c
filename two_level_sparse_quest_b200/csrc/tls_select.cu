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
#include <algorithm>

#include "tls_device.cuh"
#include "tls_internal.h"

namespace tls {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreCtasPerSm = 4;

// NCH: 16-byte chunks per summary row (2 * d * bytes / 16).  grid.y = group,
// grid.x = a contiguous slice of the group's rows.  A warp owns whole rows
// (16-byte chunk per lane, non-allocating loads); the first rows' loads are
// issued before the head fold so that the query reads overlap them.
template <typename E, int NCH>
__global__ void __launch_bounds__(kScoreThreads) block_score_kernel(BlockScoreArgs a, int rows_per_cta) {
  constexpr int EPC = E::kEPC;
  constexpr int LPR = NCH < 32 ? NCH : 32;            // lanes per row
  constexpr int RPW = 32 / LPR;                       // rows per warp step
  constexpr int CPL = (NCH + 31) / 32;                // chunks per lane
  constexpr int NWARP = kScoreThreads / 32;
  constexpr int STEP = NWARP * RPW;
  constexpr int U = CPL >= 4 ? 2 : 4;                 // rows in flight per warp (per lane: U * CPL loads)
  extern __shared__ float qpm[];                      // [2d]: Q^+ then Q^-
  const int group = blockIdx.y;
  const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int d = a.d;
  const int nbm = a.n_blocks_max;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPR, cl = lane % LPR;  // row within the warp step, chunk lane
  grid_dependency_wait();
  const int sq = min(max(a.seq_lens[b], 0), a.max_ctx);
  const int nb = (sq + a.block_size - 1) / a.block_size;
  const int r0 = blockIdx.x * rows_per_cta;
  const int r1 = min(r0 + rows_per_cta, nbm);
  const char *meta = static_cast<const char *>(a.meta) + static_cast<size_t>(group) * nbm * (NCH * 16);
  float *out = a.scores + static_cast<size_t>(group) * nbm;
  auto load_rows = [&](int rb, uint4 (&v)[U][CPL]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = rb + u * STEP + sub;
      const bool ok = row < r1 && row < nb;
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const int c = cl + j * 32;
        v[u][j] = (ok && c < NCH) ? ld_stream16(meta + static_cast<size_t>(row) * (NCH * 16) + c * 16)
                                  : make_uint4(0, 0, 0, 0);
      }
    }
  };
  uint4 v[U][CPL];
  int rb = r0 + warp * RPW;
  load_rows(rb, v);  // in flight while the query is folded
  for (int i = threadIdx.x; i < d; i += kScoreThreads) {
    float pos = 0.f, neg = 0.f;
    for (int hh = 0; hh < G; ++hh) {
      const float x = load_elem<E>(a.q, (static_cast<size_t>(b) * a.n_q_heads + g * G + hh) * d + i);
      pos += fmaxf(x, 0.f);
      neg += fminf(x, 0.f);
    }
    qpm[i] = pos;
    qpm[d + i] = neg;
  }
  __syncthreads();
  float qr[CPL][EPC];
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    const int c = cl + j * 32;
#pragma unroll
    for (int e = 0; e < EPC; ++e) qr[j][e] = (c < NCH) ? qpm[c * EPC + e] : 0.f;
  }
  for (; rb < r1; rb += STEP * U) {
    uint4 nv[U][CPL];
    const bool more = rb + STEP * U < r1;
    if (more) load_rows(rb + STEP * U, nv);  // next rows in flight during this batch's math
#pragma unroll
    for (int u = 0; u < U; ++u) {
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
    if (more) {
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int j = 0; j < CPL; ++j) v[u][j] = nv[u][j];
    }
  }
}

constexpr int kTopkThreads = 512;

__global__ void __launch_bounds__(kTopkThreads) block_topk_kernel(BlockScoreArgs a) {
  extern __shared__ uint32_t dyn[];  // keys[n_blocks_max], list[n_blocks_max]
  __shared__ SelectSmem S;
  uint32_t *keys = dyn;
  uint32_t *list = dyn + a.n_blocks_max;
  grid_dependency_wait();
  const int group = blockIdx.x;
  const int b = group / a.n_kv_heads;
  const int seq = min(max(a.seq_lens[b], 0), a.max_ctx);
  const int nb = (seq + a.block_size - 1) / a.block_size;
  const float *sc = a.scores + static_cast<size_t>(group) * a.n_blocks_max;
  int32_t *out = a.block_idx + static_cast<size_t>(group) * a.k_b;
  const int k = min(a.k_b, nb);
  if (k <= 0) {
    for (int i = threadIdx.x; i < a.k_b; i += kTopkThreads) out[i] = -1;
    return;
  }
  hist_clear<kTopkThreads>(S.hist);
  __syncthreads();
  for (int base = 0; base < nb; base += kTopkThreads) {
    const int i = base + threadIdx.x;
    const bool valid = i < nb;
    const uint32_t key = valid ? score_key(sc[i]) : 0u;
    if (valid) keys[i] = key;
    hist_add(S.hist, key, valid);
  }
  const SelectResult r = select_kth<kTopkThreads>(keys, nb, k, list, S);
  ordered_compact<kTopkThreads>(keys, nb, r, k, out, a.k_b, [](int i) { return i; }, S);
}

// RCH: 16-byte chunks per slab row (r * bytes / 16), 1..8.
constexpr int kTokThreads = 512;

template <typename E, int RCH>
__global__ void __launch_bounds__(kTokThreads) token_topk_kernel(TokenArgs a) {
  using S_t = typename E::storage;
  constexpr int EPC = E::kEPC;
  // candidates whose slab rows a thread loads before scoring them
  constexpr int kTokBatch = RCH <= 2 ? 8 : (RCH <= 4 ? 4 : 1);
  extern __shared__ uint32_t dyn[];  // keys[C], list[C]
  __shared__ int blk[1024];
  __shared__ float qbar[64];
  __shared__ SelectSmem S;
  grid_dependency_wait();
  const int group = blockIdx.x;
  const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int seq = min(max(a.seq_lens[b], 0), a.max_ctx);
  const int bs = a.block_size, r = a.n_label;
  const int C = a.k_b * bs;
  const bool bs_pow2 = (bs & (bs - 1)) == 0;
  const int bs_shift = __ffs(bs) - 1;
  auto blk_of = [&](int j) { return bs_pow2 ? (j >> bs_shift) : (j / bs); };
  uint32_t *keys = dyn;
  uint32_t *list = dyn + C;
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
  hist_clear<kTokThreads>(S.hist);
  __syncthreads();
  float ql[RCH * EPC];
#pragma unroll
  for (int e = 0; e < RCH * EPC; ++e) ql[e] = qbar[e];  // r == RCH * EPC
  const S_t *slab = static_cast<const S_t *>(a.slab) + static_cast<size_t>(group) * a.max_ctx * r;
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
        const int jb = blk_of(j);
        const int bl = blk[jb];
        t = bl * bs + (j - jb * bs);
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
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < RCH; ++c) {
        float f[EPC];
        chunk_to_f32<E>(v[u][c], f);
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc = fmaf(ql[c * EPC + e], f[e], acc);
      }
      const bool ok = tok[u] >= 0;
      const uint32_t key = ok ? score_key(acc) : 0u;
      if (j < C) {
        keys[j] = key;
        if (score_out) score_out[j] = ok ? acc : -INFINITY;
      }
      n_valid += ok;
      hist_add(S.hist, key, ok);
    }
  }
  int total;
  block_excl_scan<kTokThreads>(n_valid, S.sh, total);  // also a barrier for keys[] and the histogram
  int32_t *out = a.token_idx + static_cast<size_t>(group) * a.k_t;
  const int k = min(a.k_t, total);
  if (k <= 0) {
    for (int i = threadIdx.x; i < a.k_t; i += kTokThreads) out[i] = -1;
    return;
  }
  const SelectResult res = select_kth<kTokThreads>(keys, C, k, list, S);
  ordered_compact<kTokThreads>(
      keys, C, res, k, out, a.k_t, [&](int j) { const int jb = blk_of(j); return blk[jb] * bs + (j - jb * bs); }, S);
}

template <typename E, int NCH>
cudaError_t run_block_score(const BlockScoreArgs &a, cudaStream_t st) {
  // Several CTAs per SM; rows split evenly over each group's CTAs.
  const int groups = a.batch * a.n_kv_heads;
  const int want = kScoreCtasPerSm * a.num_sms;
  int splits = (want + groups - 1) / groups;
  const int min_rows = 8 * (kScoreThreads / 32);
  splits = std::max(1, std::min(splits, (a.n_blocks_max + min_rows - 1) / min_rows));
  const int rows = (a.n_blocks_max + splits - 1) / splits;
  splits = (a.n_blocks_max + rows - 1) / rows;
  return launch_pdl(block_score_kernel<E, NCH>, dim3(splits, groups), dim3(kScoreThreads), 2 * a.d * sizeof(float),
                    st, a, rows);
}

template <typename E, int RCH>
cudaError_t run_token_topk(const TokenArgs &a, cudaStream_t st) {
  const size_t smem = 2 * static_cast<size_t>(a.k_b) * a.block_size * sizeof(uint32_t);
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(token_topk_kernel<E, RCH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         2 * kMaxSelectKeys * static_cast<int>(sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  return launch_pdl(token_topk_kernel<E, RCH>, dim3(a.batch * a.n_kv_heads), dim3(kTokThreads), smem, st, a);
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
                                         2 * kMaxSelectKeys * static_cast<int>(sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const size_t smem = 2 * static_cast<size_t>(a.n_blocks_max) * sizeof(uint32_t);
  return launch_pdl(block_topk_kernel, dim3(a.batch * a.n_kv_heads), dim3(kTopkThreads), smem, st, a);
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
