// tls_select.cu -- the two selection stages of the AsyncTLS decode step, each
// one launch of one thread-block cluster per (sequence, KV head) group.
//
// Stage 1+2 (block score and top-K_b, gist.science (de) section 2.A "Stufe 1"
// + "Optimierung"; (es) section 2.A.1): the Quest-style bound of a block j for
// query head h,
//     u_{h,j} = sum_i max(q_{h,i} M_{j,i}, q_{h,i} m_{j,i}) = q_h^+ . M_j + q_h^- . m_j,
// summed over the heads h of one KV head.  The contraction over heads is done
// first (Q^+ = sum_h q_h^+, Q^- = sum_h q_h^-, fp32 in shared memory), so the
// block summary [M_j ; m_j] (2d values per block, contiguous) is streamed from
// HBM exactly once and dotted with [Q^+ ; Q^-]: 2 flop per stored element,
// memory-bound.  CTA r of the group's cluster scores the r-th contiguous slice
// of the blocks: a warp owns whole summary rows, each lane loads 16-byte
// chunks (coalesced, non-allocating loads), the row sum is a segmented warp
// reduction.  The scores become order-preserving keys in the CTA's shared
// memory and the cluster selects the top K_b (cluster_topk: 8-bit radix
// passes over histograms exchanged between the CTAs with asynchronous
// distributed-shared-memory stores, then an index-ordered compaction; ties to
// the lower block id).
// Stage 3+4 (token score and top-K_t, (de) section 2.A "Stufe 2", (es) section
// 2.A.2): CTA r scores the r-th slice of the group's K_b * bs candidates from
// the label-channel slab (a block's rows are contiguous) against
// Qbar_L = sum_h q_h[L] in fp32, and the cluster selects the top K_t the same
// way (ties to the lower token position).
#include <algorithm>

#include "tls_device.cuh"
#include "tls_internal.h"

namespace tls {
namespace {

constexpr int kClusterSize = 8;  // CTAs per group (portable cluster size)
constexpr int kSliceCap = kMaxSelectKeys / kClusterSize;  // keys per CTA
constexpr int kScoreThreads = 256;
constexpr int kTokThreads = 256;

// NCH: 16-byte chunks per summary row (2 * d * bytes / 16).  grid = (CS, groups),
// cluster = (CS, 1, 1).  The first rows' loads are issued before the head fold
// so that the query reads overlap them.
template <typename E, int NCH, int CS>
__global__ void __launch_bounds__(kScoreThreads, NCH > 32 ? 2 : 4) block_select_kernel(BlockScoreArgs a, int rows_per_cta) {
  constexpr int EPC = E::kEPC;
  constexpr int LPR = NCH < 32 ? NCH : 32;            // lanes per row
  constexpr int RPW = 32 / LPR;                       // rows per warp step
  constexpr int CPL = (NCH + 31) / 32;                // chunks per lane
  constexpr int NWARP = kScoreThreads / 32;
  constexpr int STEP = NWARP * RPW;
  constexpr int U = CPL >= 4 ? 2 : 4;                 // rows in flight per warp (per lane: U * CPL loads)
  extern __shared__ float qpm[];                      // [2d]: Q^+ then Q^-, then the slice's keys
  __shared__ ClusterSelectSmem<CS> S;
  cluster_topk_begin(S);
  const int group = blockIdx.y;
  const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int d = a.d;
  const int nbm = a.n_blocks_max;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPR, cl = lane % LPR;  // row within the warp step, chunk lane
  const int rank = static_cast<int>(cluster_ctarank());
  uint32_t *keys = reinterpret_cast<uint32_t *>(qpm + 2 * d);
  if (threadIdx.x < kCBins) S.hist[threadIdx.x] = 0;
  grid_dependency_wait();
  const int sq = min(max(a.seq_lens[b], 0), a.max_ctx);
  const int nb = (sq + a.block_size - 1) / a.block_size;
  const int r0 = rank * rows_per_cta;
  const int r1 = min(r0 + rows_per_cta, nbm);
  const char *meta = static_cast<const char *>(a.meta) + static_cast<size_t>(group) * nbm * (NCH * 16);
  float *out = a.scores ? a.scores + static_cast<size_t>(group) * nbm : nullptr;
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
      if (cl == 0 && row < r1) {
        const bool valid = row < nb;
        const uint32_t key = valid ? max(score_key(acc), 1u) : 0u;
        keys[row - r0] = key;
        hist_add(S.hist, key, valid);
        if (out) out[row] = valid ? acc : -INFINITY;
      }
    }
    if (more) {
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int j = 0; j < CPL; ++j) v[u][j] = nv[u][j];
    }
  }
  cluster_topk<kScoreThreads, CS, kSliceCap>(
      keys, max(r1 - r0, 0), a.k_b, a.block_idx + static_cast<size_t>(group) * a.k_b, a.k_b,
      [r0](int i) { return r0 + i; }, S, a.err);
}

// RCH: 16-byte chunks per slab row (r * bytes / 16), 1..8.  grid = (CS, groups),
// cluster = (CS, 1, 1); CTA r scores candidates [r*per, (r+1)*per).
template <typename E, int RCH, int CS>
__global__ void __launch_bounds__(kTokThreads, RCH > 2 ? 2 : 4) token_select_kernel(TokenArgs a, int per_cta) {
  using S_t = typename E::storage;
  constexpr int EPC = E::kEPC;
  constexpr int NT = kTokThreads;
  constexpr int kBatch = RCH <= 4 ? 4 : 2;  // candidates whose rows a thread loads at once
  extern __shared__ uint32_t keys[];  // [per_cta]
  __shared__ int blk[1024];           // block ids of the slice's blocks
  __shared__ float qbar[64];
  __shared__ ClusterSelectSmem<CS> S;
  cluster_topk_begin(S);
  const int group = blockIdx.y;
  const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int bs = a.block_size, r = a.n_label;
  const int C = a.k_b * bs;
  const int rank = static_cast<int>(cluster_ctarank());
  const int c0 = min(rank * per_cta, C), c1 = min(c0 + per_cta, C);
  const bool bs_pow2 = (bs & (bs - 1)) == 0;
  const int bs_shift = __ffs(bs) - 1;
  auto blk_of = [&](int j) { return bs_pow2 ? (j >> bs_shift) : (j / bs); };
  const int jb0 = c0 < c1 ? blk_of(c0) : 0;
  const int nblk = c0 < c1 ? blk_of(c1 - 1) - jb0 + 1 : 0;  // <= min(k_b, 1024)
  if (threadIdx.x < kCBins) S.hist[threadIdx.x] = 0;
  grid_dependency_wait();
  const int seq = min(max(a.seq_lens[b], 0), a.max_ctx);
  for (int i = threadIdx.x; i < nblk; i += NT) {
    const int v = a.block_idx[static_cast<size_t>(group) * a.k_b + jb0 + i];
    blk[i] = (v >= 0 && v < a.n_blocks_max) ? v : -1;
  }
  for (int c = threadIdx.x; c < r; c += NT) {
    const int ch = a.label_idx[c];
    float sum = 0.f;
    if (ch >= 0 && ch < a.d)
      for (int hh = 0; hh < G; ++hh)
        sum += load_elem<E>(a.q, (static_cast<size_t>(b) * a.n_q_heads + g * G + hh) * a.d + ch);
    qbar[c] = sum;
  }
  __syncthreads();
  float ql[RCH * EPC];
#pragma unroll
  for (int e = 0; e < RCH * EPC; ++e) ql[e] = qbar[e];  // r == RCH * EPC
  const S_t *slab = static_cast<const S_t *>(a.slab) + static_cast<size_t>(group) * a.max_ctx * r;
  float *score_out = a.token_score ? a.token_score + static_cast<size_t>(group) * C : nullptr;
  for (int base = c0; base < c1; base += NT * kBatch) {
    uint4 v[kBatch][RCH];
    int tok[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = base + u * NT + threadIdx.x;
      int t = -1;
      if (j < c1) {
        const int jb = blk_of(j);
        const int bl = blk[jb - jb0];
        t = bl * bs + (j - jb * bs);
        if (bl < 0 || t >= seq) t = -1;
      }
      tok[u] = t;
#pragma unroll
      for (int c = 0; c < RCH; ++c)
        v[u][c] = t >= 0 ? ld_stream16(slab + static_cast<size_t>(t) * r + c * EPC) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = base + u * NT + threadIdx.x;
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < RCH; ++c) {
        float f[EPC];
        chunk_to_f32<E>(v[u][c], f);
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc = fmaf(ql[c * EPC + e], f[e], acc);
      }
      const bool ok = tok[u] >= 0;
      const uint32_t key = ok ? max(score_key(acc), 1u) : 0u;
      if (j < c1) {
        keys[j - c0] = key;
        if (score_out) score_out[j] = ok ? acc : -INFINITY;
      }
      hist_add(S.hist, key, ok);
    }
  }
  cluster_topk<NT, CS, kSliceCap>(
      keys, c1 - c0, a.k_t, a.token_idx + static_cast<size_t>(group) * a.k_t, a.k_t,
      [&](int i) {
        const int j = c0 + i;
        const int jb = blk_of(j);
        return blk[jb - jb0] * bs + (j - jb * bs);
      },
      S, a.err);
}

template <typename E, int NCH>
cudaError_t run_block_select(const BlockScoreArgs &a, cudaStream_t st) {
  constexpr int CS = kClusterSize;
  const int rows = (a.n_blocks_max + CS - 1) / CS;  // <= kSliceCap
  const size_t smem = 2 * static_cast<size_t>(a.d) * sizeof(float) + static_cast<size_t>(rows) * sizeof(uint32_t);
  return launch_pdl_cluster(block_select_kernel<E, NCH, CS>, dim3(CS, a.batch * a.n_kv_heads), dim3(kScoreThreads),
                            smem, st, CS, a, rows);
}

template <typename E, int RCH>
cudaError_t run_token_select(const TokenArgs &a, cudaStream_t st) {
  constexpr int CS = kClusterSize;
  const int C = a.k_b * a.block_size;
  const int per = (C + CS - 1) / CS;  // <= kSliceCap
  const size_t smem = static_cast<size_t>(per) * sizeof(uint32_t);
  return launch_pdl_cluster(token_select_kernel<E, RCH, CS>, dim3(CS, a.batch * a.n_kv_heads), dim3(kTokThreads),
                            smem, st, CS, a, per);
}

}  // namespace

cudaError_t launch_block_select(const BlockScoreArgs &a, cudaStream_t st) {
  const int nch = 2 * a.d * (a.dtype == 1 ? 2 : 4) / 16;
  if (a.dtype == 1) {
    switch (nch) {
      case 16: return run_block_select<BF16, 16>(a, st);
      case 32: return run_block_select<BF16, 32>(a, st);
      case 144: return run_block_select<BF16, 144>(a, st);
    }
  } else {
    switch (nch) {
      case 32: return run_block_select<F32, 32>(a, st);
      case 64: return run_block_select<F32, 64>(a, st);
    }
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_token_select(const TokenArgs &a, cudaStream_t st) {
  const int rch = a.n_label * (a.dtype == 1 ? 2 : 4) / 16;
  switch (rch) {
    case 1: return a.dtype == 1 ? run_token_select<BF16, 1>(a, st) : run_token_select<F32, 1>(a, st);
    case 2: return a.dtype == 1 ? run_token_select<BF16, 2>(a, st) : run_token_select<F32, 2>(a, st);
    case 4: return a.dtype == 1 ? run_token_select<BF16, 4>(a, st) : run_token_select<F32, 4>(a, st);
    case 8: return a.dtype == 1 ? run_token_select<BF16, 8>(a, st) : run_token_select<F32, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tls
