// tls_select.cu -- the two selection stages of the AsyncTLS decode step, each
// run by one thread-block cluster per (sequence, KV head) group.
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
// Three kernels: stages 1+2, stages 3+4, and all four in one launch (the
// cluster goes from its block selection straight to its token stage; the
// selected block ids pass through global memory behind a release/acquire
// cluster barrier).  The arithmetic is shared, so the fused launch gives the
// same bits as the two separate ones.
#include <algorithm>

#include "tls_device.cuh"
#include "tls_internal.h"

namespace tls {
namespace {

constexpr int kClusterSize = 8;  // CTAs per group (portable cluster size)
constexpr int kSliceCap = kMaxSelectKeys / kClusterSize;  // keys per CTA
constexpr int kThreads = 256;

// ---------------------------------------------------------------- query folds
// Parts of a fold over the G heads of a group: the largest power of two P <=
// G with P * items <= kThreads (and P <= 32), so that the P threads of an
// item are consecutive lanes of one warp.
__device__ __forceinline__ int fold_parts(int G, int items) {
  int P = 1;
  while (2 * P <= G && 2 * P <= 32 && 2 * P * items <= kThreads) P *= 2;
  return P;
}

// Adds v of the P lanes of this item (lanes part 0 .. P-1, consecutive), in
// part order, starting from 0: every lane of the warp calls it.
__device__ __forceinline__ float fold_lanes(float v, int P) {
  const int lane = threadIdx.x & 31, first = lane & ~(P - 1);
  float sum = 0.f;
  for (int k = 0; k < P; ++k) sum += __shfl_sync(0xffffffffu, v, first + k);
  return sum;
}

// qpm = [Q+; Q-] (2 d floats of shared memory) of the G heads of query rows
// row0 .. row0 + G - 1: Q+_i = sum_h max(q_{h,i}, 0), Q-_i = sum_h min(q_{h,i}, 0)
// (gist.science (de) section 2.A "Stufe 1": the per-head bounds summed over
// the heads that share the KV head).  All threads of the CTA call it.  The
// G x d block is read as 16-byte chunks: thread t takes chunk column t / P and
// the heads of part t % P (consecutive heads, 8 loads in flight); the P part
// sums are then added in part order.  With P = G (small groups) the sums are
// the sequential sums over the heads.  FB: loads in flight per thread.
// Chunk columns [c_begin, c_end) only (a fold split over several CTAs), by
// the CTA's nthr threads; P depends on G and d alone, so every split gives the
// same bits.
template <typename E, int FB>
__device__ __forceinline__ void fold_group_query(const void *q, size_t row0, int G, int d, float *qpm,
                                                 int c_begin, int c_end, int nthr) {
  constexpr int EPC = E::kEPC;
  const int NC = d / EPC;
  const int P = fold_parts(G, NC);
  const int HP = (G + P - 1) / P;
  for (int base = c_begin * P; base < c_end * P; base += nthr) {
    const int t = base + static_cast<int>(threadIdx.x);
    const int c = t / P, part = t % P;
    float pos[EPC], neg[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) pos[e] = neg[e] = 0.f;
    if (c < c_end) {
      const uint4 *src = static_cast<const uint4 *>(q) + row0 * NC + c;
      const int h0 = part * HP, h1 = min(G, h0 + HP);
      for (int hb = h0; hb < h1; hb += FB) {
        uint4 v[FB];
#pragma unroll
        for (int u = 0; u < FB; ++u) v[u] = hb + u < h1 ? __ldg(src + static_cast<size_t>(hb + u) * NC) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < FB; ++u) {
          if (hb + u < h1) {
            float f[EPC];
            chunk_to_f32<E>(v[u], f);
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
              pos[e] += fmaxf(f[e], 0.f);
              neg[e] += fminf(f[e], 0.f);
            }
          }
        }
      }
    }
#pragma unroll
    for (int e = 0; e < EPC; ++e) {
      const float sp = fold_lanes(pos[e], P), sn = fold_lanes(neg[e], P);
      if (c < c_end && part == 0) {
        qpm[c * EPC + e] = sp;
        qpm[d + c * EPC + e] = sn;
      }
    }
  }
}

// The fold every path uses (so that every path's block scores are the same
// bits), by the summary row's 16-byte chunks NCH: for d <= 128 (NCH <= 64)
// thread i sums channel i over the heads in order (few heads, short rows:
// this is the cheapest), for the latent rows the parallel fold above.
template <typename E, int NCH, int FB>
__device__ __forceinline__ void fold_query(const void *q, size_t row0, int G, int d, float *qpm) {
  if constexpr (NCH > 64) {
    fold_group_query<E, FB>(q, row0, G, d, qpm, 0, d / E::kEPC, kThreads);
  } else {
    for (int i = threadIdx.x; i < d; i += kThreads) {
      float pos = 0.f, neg = 0.f;
      for (int hh = 0; hh < G; ++hh) {
        const float x = load_elem<E>(q, (row0 + hh) * d + i);
        pos += fmaxf(x, 0.f);
        neg += fminf(x, 0.f);
      }
      qpm[i] = pos;
      qpm[d + i] = neg;
    }
  }
}

// ---------------------------------------------------------------- stage 1 body
// After the grid dependency wait: folds the group's query into qpm = [Q+; Q-]
// and scores summary rows [r0, r1) into keys[row - r0] and hist (top key
// byte).  NCH: 16-byte chunks per summary row (2 * d * bytes / 16).  The first
// rows' loads are issued before the head fold so that the query reads
// overlap them.
template <typename E, int NCH, bool KEYS = true, bool QFOLD = false>
__device__ __forceinline__ void score_blocks(const BlockScoreArgs &a, int group, int nb, int r0, int r1, float *qpm,
                                             uint32_t *keys, int *hist) {
  constexpr int EPC = E::kEPC;
  constexpr int LPR = NCH < 32 ? NCH : 32;  // lanes per row
  constexpr int RPW = 32 / LPR;             // rows per warp step
  constexpr int CPL = (NCH + 31) / 32;      // chunks per lane
  constexpr int NWARP = kThreads / 32;
  constexpr int STEP = NWARP * RPW;
  constexpr int U = CPL >= 4 ? 2 : 4;  // rows in flight per warp (per lane: U * CPL loads)
  const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int d = a.d;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPR, cl = lane % LPR;  // row within the warp step, chunk lane
  const char *meta = static_cast<const char *>(a.meta) + static_cast<size_t>(group) * a.n_blocks_max * (NCH * 16);
  float *out = a.scores ? a.scores + static_cast<size_t>(group) * a.n_blocks_max : nullptr;
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
  if constexpr (QFOLD) {  // folded once per group by launch_query_fold
    const float *src = a.qfold + static_cast<size_t>(group) * 2 * d;
    for (int i = threadIdx.x; i < 2 * d; i += kThreads) qpm[i] = __ldcg(src + i);
  } else {
    fold_query<E, NCH, 8>(a.q, static_cast<size_t>(b) * a.n_q_heads + static_cast<size_t>(g) * G, G, d, qpm);
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
    float x[U];  // this lane's part of each of the batch's U rows
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
      x[u] = acc;
    }
    // The U row sums over the row group's LPR lanes in one butterfly: at each
    // of the first log2(U) steps a lane keeps half of its rows (the upper half
    // when its lane bit is set) and adds its partner's part of them, the other
    // steps add the partner's whole sum.  Afterwards lane cl holds the sum of
    // row u(cl) (its lane bits from the top); the first lane of each row
    // writes the key, so a batch's key writes and histogram adds run in one
    // pass over U lanes instead of one lane per row.
    int u_mine = 0;
#pragma unroll
    for (int o = LPR / 2, R = U; o > 0; o >>= 1) {
      if (R > 1) {
        const bool up = (cl & o) != 0;
#pragma unroll
        for (int k = 0; k < U / 2; ++k) {
          if (k < R / 2) {
            const float send = up ? x[k] : x[k + R / 2];
            const float recv = __shfl_xor_sync(0xffffffffu, send, o);
            x[k] = (up ? x[k + R / 2] : x[k]) + recv;
          }
        }
        R /= 2;
        u_mine = 2 * u_mine + (up ? 1 : 0);
      } else {
        x[0] += __shfl_xor_sync(0xffffffffu, x[0], o);
      }
    }
    {
      const int row = rb + u_mine * STEP + sub;
      if ((cl % (LPR / U)) == 0 && row < r1) {
        const float acc = x[0];
        const bool valid = row < nb;
        if constexpr (KEYS) {
          const uint32_t key = valid ? max(score_key(acc), 1u) : 0u;
          keys[row - r0] = key;
          hist_add(hist, key, valid);
        }
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
}

// [Q+; Q-] of group blockIdx.x into a.qfold.  d <= 128: one CTA per group,
// the per-channel fold.  Latent rows: blockIdx.y takes 8 of the 72 chunk
// columns (one warp, every head of a part in flight at once), so the fold of
// a group is one round trip of 72 KB spread over 9 CTAs.
template <typename E, int NCH>
__global__ void __launch_bounds__(NCH > 64 ? 32 : kThreads) query_fold_kernel(BlockScoreArgs a) {
  grid_dependency_wait();
  const int group = blockIdx.x;
  const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
  const int G = a.n_q_heads / a.n_kv_heads;
  const size_t row0 = static_cast<size_t>(b) * a.n_q_heads + static_cast<size_t>(g) * G;
  float *dst = a.qfold + static_cast<size_t>(group) * 2 * a.d;
  if constexpr (NCH > 64) {
    const int NC = a.d / E::kEPC;
    const int c0 = blockIdx.y * 8, c1 = min(NC, c0 + 8);
    fold_group_query<E, 32>(a.q, row0, G, a.d, dst, c0, c1, 32);
  } else {
    fold_query<E, NCH, 8>(a.q, row0, G, a.d, dst);
  }
}

// The stage-1 keys of rows [r0, r1) from block scores a previous launch
// wrote (the two-phase selection): the same keys score_blocks makes.
__device__ __forceinline__ void keys_from_scores(const BlockScoreArgs &a, int group, int nb, int r0, int r1,
                                                 uint32_t *keys, int *hist) {
  const float *sc = a.scores + static_cast<size_t>(group) * a.n_blocks_max;
  for (int row = r0 + threadIdx.x; row < r1; row += kThreads) {
    const bool valid = row < nb;
    const uint32_t key = valid ? max(score_key(__ldcg(sc + row)), 1u) : 0u;
    keys[row - r0] = key;
    hist_add(hist, key, valid);
  }
}

// Phase 1 of the two-phase selection: CTA c scores the c-th equal range of
// all groups' summary rows (a range may cross into the next group; the
// query fold is redone per group) into a.scores, with score_blocks' arithmetic.
template <typename E, int NCH, bool QFOLD>
__global__ void __launch_bounds__(kThreads, NCH > 32 ? 2 : 4) block_scores_kernel(BlockScoreArgs a, int rows_per_cta) {
  extern __shared__ float qpm[];  // [2d]
  grid_dependency_wait();
  const long long total = static_cast<long long>(a.batch) * a.n_kv_heads * a.n_blocks_max;
  long long r0 = static_cast<long long>(blockIdx.x) * rows_per_cta;
  const long long r1 = std::min(r0 + rows_per_cta, total);
  while (r0 < r1) {
    const int group = static_cast<int>(r0 / a.n_blocks_max);
    const long long gbase = static_cast<long long>(group) * a.n_blocks_max;
    const long long gend = std::min(r1, gbase + a.n_blocks_max);
    const int sq = min(max(a.seq_lens[group / a.n_kv_heads], 0), a.max_ctx);
    const int nb = (sq + a.block_size - 1) / a.block_size;
    score_blocks<E, NCH, false, QFOLD>(a, group, nb, static_cast<int>(r0 - gbase), static_cast<int>(gend - gbase), qpm,
                                nullptr, nullptr);
    __syncthreads();  // qpm is folded again for the next group
    r0 = gend;
  }
}

// The max-over-heads variant of the stage-1 body: qh = [q_h^+; q_h^-] per head
// (G x 2d floats), every head's bound per row, the largest one is the score.
// GQA shapes only (G <= 8).
template <typename E, int NCH>
__device__ __forceinline__ void score_blocks_max(const BlockScoreArgs &a, int group, int nb, int r0, int r1,
                                                 float *qh, uint32_t *keys, int *hist) {
  constexpr int EPC = E::kEPC;
  constexpr int LPR = NCH < 32 ? NCH : 32;
  constexpr int RPW = 32 / LPR;
  constexpr int CPL = (NCH + 31) / 32;
  constexpr int NWARP = kThreads / 32;
  constexpr int STEP = NWARP * RPW;
  constexpr int MAXG = 8;
  const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int d = a.d;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPR, cl = lane % LPR;
  const char *meta = static_cast<const char *>(a.meta) + static_cast<size_t>(group) * a.n_blocks_max * (NCH * 16);
  float *out = a.scores ? a.scores + static_cast<size_t>(group) * a.n_blocks_max : nullptr;
  for (int i = threadIdx.x; i < G * d; i += kThreads) {
    const int hh = i / d, c = i % d;
    const float x = load_elem<E>(a.q, (static_cast<size_t>(b) * a.n_q_heads + g * G + hh) * d + c);
    qh[hh * 2 * d + c] = fmaxf(x, 0.f);
    qh[hh * 2 * d + d + c] = fminf(x, 0.f);
  }
  __syncthreads();
  for (int rb = r0 + warp * RPW; rb < r1; rb += STEP) {
    const int row = rb + sub;
    const bool ok = row < r1 && row < nb;
    float acc[MAXG];
#pragma unroll
    for (int h = 0; h < MAXG; ++h) acc[h] = 0.f;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      const int c = cl + j * 32;
      if (c < NCH) {
        const uint4 v = ok ? ld_stream16(meta + static_cast<size_t>(row) * (NCH * 16) + c * 16) : make_uint4(0, 0, 0, 0);
        float f[EPC];
        chunk_to_f32<E>(v, f);
#pragma unroll
        for (int h = 0; h < MAXG; ++h)
          if (h < G) {
            const float *qp = qh + h * 2 * d + c * EPC;
#pragma unroll
            for (int e = 0; e < EPC; ++e) acc[h] = fmaf(qp[e], f[e], acc[h]);
          }
      }
    }
    float best = -INFINITY;
#pragma unroll
    for (int h = 0; h < MAXG; ++h) {
      float x = acc[h];
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (h < G) best = fmaxf(best, x);
    }
    if (cl == 0 && row < r1) {
      const bool valid = row < nb;
      const uint32_t key = valid ? max(score_key(best), 1u) : 0u;
      keys[row - r0] = key;
      hist_add(hist, key, valid);
      if (out) out[row] = valid ? best : -INFINITY;
    }
  }
}

// Qbar_L[c] = sum_h q_h[L[c]] (fp32, heads in order) into qbar[0..r); with an
// int8 slab the channel's scale is folded in: qbar[c] = scale_c * Qbar_L[c].
// All threads of the CTA call it.  PAR (the latent rows, many heads): thread
// t takes label t / P and the heads of part t % P (4 loads in flight) and the
// part sums are added in part order; otherwise thread c sums label c over the
// heads in order.  Every kernel of a shape takes the same PAR (d > 128).
template <typename E, bool PAR>
__device__ __forceinline__ void fold_label_query(const TokenArgs &a, int group, float *qbar) {
  const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
  const int G = a.n_q_heads / a.n_kv_heads;
  if constexpr (!PAR) {
    for (int c = threadIdx.x; c < a.n_label; c += kThreads) {
      const int ch = a.label_idx[c];
      float sum = 0.f;
      if (ch >= 0 && ch < a.d)
        for (int hh = 0; hh < G; ++hh)
          sum += load_elem<E>(a.q, (static_cast<size_t>(b) * a.n_q_heads + g * G + hh) * a.d + ch);
      qbar[c] = a.scales ? sum * a.scales[static_cast<size_t>(group) * a.n_label + c] : sum;
    }
    return;
  }
  const int P = fold_parts(G, a.n_label);
  const int HP = (G + P - 1) / P;
  const size_t row0 = static_cast<size_t>(b) * a.n_q_heads + static_cast<size_t>(g) * G;
  for (int base = 0; base < a.n_label * P; base += kThreads) {
    const int t = base + static_cast<int>(threadIdx.x);
    const int c = t / P, part = t % P;
    const int ch = c < a.n_label ? a.label_idx[c] : -1;
    float sum = 0.f;
    if (ch >= 0 && ch < a.d) {
      const int h0 = part * HP, h1 = min(G, h0 + HP);
      for (int hb = h0; hb < h1; hb += 4) {
        float x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) x[u] = hb + u < h1 ? load_elem<E>(a.q, (row0 + hb + u) * a.d + ch) : 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (hb + u < h1) sum += x[u];
      }
    }
    const float tot = fold_lanes(sum, P);
    if (c < a.n_label && part == 0)
      qbar[c] = a.scales ? tot * a.scales[static_cast<size_t>(group) * a.n_label + c] : tot;
  }
}

// ---------------------------------------------------------------- stage 3 body
// Scores candidates [c0, c1) of the group (blk[j / bs - jb0] = kept block id,
// < 0 for none; qbar in shared memory, complete) into keys[j - c0] and hist.
// SE: the slab's storage (the K dtype, or I8 codes); RCH: 16-byte chunks per
// slab row (r * bytes / 16), 1..8.
template <int RCH, int EPC>
constexpr int token_min_blocks() { return (RCH > 2 || RCH * EPC > 16) ? 2 : 4; }

template <typename E, int RCH>
__device__ __forceinline__ void score_tokens(const TokenArgs &a, int group, int seq, int c0, int c1, const int *blk,
                                             int jb0, const float *qbar, uint32_t *keys, int *hist) {
  using S_t = typename E::storage;
  constexpr int EPC = E::kEPC;
  constexpr int kBatch = (RCH <= 4 && RCH * EPC <= 32) ? 4 : 2;  // candidates whose rows a thread loads at once
  const int bs = a.block_size, r = a.n_label;
  const int C = a.k_b * bs;
  const bool bs_pow2 = (bs & (bs - 1)) == 0;
  const int bs_shift = __ffs(bs) - 1;
  auto blk_of = [&](int j) { return bs_pow2 ? (j >> bs_shift) : (j / bs); };
  float ql[RCH * EPC];
#pragma unroll
  for (int e = 0; e < RCH * EPC; ++e) ql[e] = qbar[e];  // r == RCH * EPC
  const S_t *slab = static_cast<const S_t *>(a.slab) + static_cast<size_t>(group) * a.max_ctx * r;
  float *score_out = a.token_score ? a.token_score + static_cast<size_t>(group) * C : nullptr;
  for (int base = c0; base < c1; base += kThreads * kBatch) {
    uint4 v[kBatch][RCH];
    int tok[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = base + u * kThreads + threadIdx.x;
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
      const int j = base + u * kThreads + threadIdx.x;
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
      hist_add(hist, key, ok);
    }
  }
}

// Candidate slice [c0, c1) of cluster rank `rank` and the range of kept-block
// list entries it covers: [jb0, jb0 + nblk), nblk <= min(k_b, 1024).
struct TokenSlice {
  int c0, c1, jb0, nblk;
};
__device__ __forceinline__ TokenSlice token_slice(const TokenArgs &a, int rank, int per_cta) {
  const int bs = a.block_size, C = a.k_b * bs;
  TokenSlice s;
  s.c0 = min(rank * per_cta, C);
  s.c1 = min(s.c0 + per_cta, C);
  s.jb0 = s.c0 < s.c1 ? s.c0 / bs : 0;
  s.nblk = s.c0 < s.c1 ? (s.c1 - 1) / bs - s.jb0 + 1 : 0;
  return s;
}

// ---------------------------------------------------------------- kernels
// grid = (CS, groups), cluster = (CS, 1, 1) for all three.
template <typename E, int NCH, int CS, bool AGG_MAX>
__global__ void __launch_bounds__(kThreads, NCH > 32 ? 2 : 4) block_select_kernel(BlockScoreArgs a, int rows_per_cta) {
  extern __shared__ float qpm[];  // [2d] Q^+, Q^- (max variant: [G][2d] per head), then the slice's keys
  __shared__ ClusterSelectSmem<CS> S;
  cluster_topk_begin(S);
  const int group = blockIdx.y;
  const int rank = static_cast<int>(cluster_ctarank());
  const int G = a.n_q_heads / a.n_kv_heads;
  uint32_t *keys = reinterpret_cast<uint32_t *>(qpm + (AGG_MAX ? G : 1) * 2 * a.d);
  if (threadIdx.x < kCBins) S.hist[threadIdx.x] = 0;
  grid_dependency_wait();
  const int b = group / a.n_kv_heads;
  const int sq = min(max(a.seq_lens[b], 0), a.max_ctx);
  const int nb = (sq + a.block_size - 1) / a.block_size;
  const int r0 = rank * rows_per_cta;
  const int r1 = min(r0 + rows_per_cta, a.n_blocks_max);
  if (a.from_scores) keys_from_scores(a, group, nb, r0, r1, keys, S.hist);
  else if constexpr (AGG_MAX) score_blocks_max<E, NCH>(a, group, nb, r0, r1, qpm, keys, S.hist);
  else score_blocks<E, NCH>(a, group, nb, r0, r1, qpm, keys, S.hist);
  cluster_topk<kThreads, CS, kSliceCap>(
      keys, max(r1 - r0, 0), a.k_b, a.block_idx + static_cast<size_t>(group) * a.k_b, a.k_b,
      [r0](int i) { return r0 + i; }, S, a.err);
}

template <typename E, typename SE, int RCH, int CS, bool PAR>
__global__ void __launch_bounds__(kThreads, token_min_blocks<RCH, SE::kEPC>())
    token_select_kernel(TokenArgs a, int per_cta) {
  extern __shared__ uint32_t keys[];  // [per_cta]
  __shared__ int blk[1024];           // block ids of the slice's blocks
  __shared__ float qbar[64];
  __shared__ ClusterSelectSmem<CS> S;
  cluster_topk_begin(S);
  const int group = blockIdx.y;
  const int rank = static_cast<int>(cluster_ctarank());
  const TokenSlice sl = token_slice(a, rank, per_cta);
  if (threadIdx.x < kCBins) S.hist[threadIdx.x] = 0;
  grid_dependency_wait();
  const int seq = min(max(a.seq_lens[group / a.n_kv_heads], 0), a.max_ctx);
  for (int i = threadIdx.x; i < sl.nblk; i += kThreads) {
    const int v = a.block_idx[static_cast<size_t>(group) * a.k_b + sl.jb0 + i];
    blk[i] = (v >= 0 && v < a.n_blocks_max) ? v : -1;
  }
  fold_label_query<E, PAR>(a, group, qbar);
  __syncthreads();
  score_tokens<SE, RCH>(a, group, seq, sl.c0, sl.c1, blk, sl.jb0, qbar, keys, S.hist);
  const int bs = a.block_size, jb0 = sl.jb0, c0 = sl.c0;
  cluster_topk<kThreads, CS, kSliceCap>(
      keys, sl.c1 - sl.c0, a.k_t, a.token_idx + static_cast<size_t>(group) * a.k_t, a.k_t,
      [&](int i) {
        const int j = c0 + i;
        const int jb = j / bs;
        return blk[jb - jb0] * bs + (j - jb * bs);
      },
      S, a.err);
}

struct StepArgs {
  BlockScoreArgs blk;
  TokenArgs tok;
};

// local_n > 0 (block scores in global memory, a.from_scores, at most
// kLocalBlockKeys blocks): every CTA selects the group's K_b blocks itself from
// all local_n scores (no cluster exchange); rank 0 writes the block ids.
constexpr int kLocalBlockKeys = 4096;

template <typename E, typename SE, int NCH, int RCH, int CS, bool LOCAL>
__global__ void __launch_bounds__(kThreads, NCH > 32 ? 2 : token_min_blocks<RCH, SE::kEPC>())
    select_step_kernel(StepArgs s, int rows_per_cta, int per_cta, int local_n) {
  // dynamic: [max(2d Q^+ Q^- + rows_per_cta block keys, local_n block keys)][per_cta token keys]
  extern __shared__ float qpm[];
  __shared__ ClusterSelectSmem<CS> SB, ST;
  __shared__ int blk[1024];
  __shared__ float qbar[64];
  const BlockScoreArgs &a = s.blk;
  const TokenArgs &t = s.tok;
  cluster_topk_arm(SB);
  cluster_topk_arm(ST);
  cluster_arrive_relaxed();
  const int group = blockIdx.y;
  const int rank = static_cast<int>(cluster_ctarank());
  uint32_t *bkeys = reinterpret_cast<uint32_t *>(qpm + 2 * a.d);
  uint32_t *tkeys = reinterpret_cast<uint32_t *>(qpm) + max(2 * a.d + rows_per_cta, local_n);
  if (threadIdx.x < kCBins) {
    SB.hist[threadIdx.x] = 0;
    ST.hist[threadIdx.x] = 0;
  }
  grid_dependency_wait();
  if (t.ready) {  // the attention after this launch waits per group on these words, not on the grid
    if (rank == 0 && threadIdx.x == 0) {
      t.ready[group] = 0;
      __threadfence();
    }
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  const int b = group / a.n_kv_heads;
  const int sq = min(max(a.seq_lens[b], 0), a.max_ctx);
  const int nb = (sq + a.block_size - 1) / a.block_size;
  fold_label_query<E, (NCH > 64)>(t, group, qbar);  // independent of the block stage; complete by the next barrier
  int32_t *bout = a.block_idx + static_cast<size_t>(group) * a.k_b;
  TokenSlice sl;
  if constexpr (LOCAL) {
    // ---- stages 1 + 2 from the scores in global memory, in every CTA
    uint32_t *lkeys = reinterpret_cast<uint32_t *>(qpm);
    const int nbm = min(local_n, a.n_blocks_max);
    keys_from_scores(a, group, nb, 0, nbm, lkeys, SB.hist);  // (the cluster histogram stays unused)
    const int k = cta_topk<kThreads, kLocalBlockKeys>(lkeys, nbm, a.k_b, blk, [](int i) { return i; }, SB.hist,
                                                      SB.bc, SB.sh);
    for (int i = max(k, 0) + threadIdx.x; i < a.k_b; i += kThreads) blk[i] = -1;
    sl = token_slice(t, rank, per_cta);
    __syncthreads();
    if (rank == 0)
      for (int i = threadIdx.x; i < a.k_b; i += kThreads) bout[i] = blk[i];
    // this CTA's slice of the kept-block list moves to the front of blk
    int v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = u * kThreads + threadIdx.x;
      v[u] = i < sl.nblk ? blk[sl.jb0 + i] : -1;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = u * kThreads + threadIdx.x;
      if (i < sl.nblk) blk[i] = (v[u] >= 0 && v[u] < t.n_blocks_max) ? v[u] : -1;
    }
  } else {
    // ---- stages 1 + 2
    const int r0 = rank * rows_per_cta;
    const int r1 = min(r0 + rows_per_cta, a.n_blocks_max);
    if (a.from_scores) keys_from_scores(a, group, nb, r0, r1, bkeys, SB.hist);
    else score_blocks<E, NCH>(a, group, nb, r0, r1, qpm, bkeys, SB.hist);
    cluster_topk<kThreads, CS, kSliceCap>(
        bkeys, max(r1 - r0, 0), a.k_b, bout, a.k_b, [r0](int i) { return r0 + i; }, SB, a.err);
    // every CTA's block ids are in global memory and visible to the cluster
    cluster_arrive_release();
    cluster_wait();
    sl = token_slice(t, rank, per_cta);
    for (int i = threadIdx.x; i < sl.nblk; i += kThreads) {
      const int v = __ldcg(bout + sl.jb0 + i);
      blk[i] = (v >= 0 && v < t.n_blocks_max) ? v : -1;
    }
  }
  // ---- stages 3 + 4
  __syncthreads();
  score_tokens<SE, RCH>(t, group, sq, sl.c0, sl.c1, blk, sl.jb0, qbar, tkeys, ST.hist);
  const int bs = t.block_size, jb0 = sl.jb0, c0 = sl.c0;
  cluster_topk<kThreads, CS, kSliceCap>(
      tkeys, sl.c1 - sl.c0, t.k_t, t.token_idx + static_cast<size_t>(group) * t.k_t, t.k_t,
      [&](int i) {
        const int j = c0 + i;
        const int jb = j / bs;
        return blk[jb - jb0] * bs + (j - jb * bs);
      },
      ST, t.err, /*entry_wait=*/LOCAL);
  if (t.ready) {  // every CTA's token ids are written: the group is ready for its attention
    __threadfence();
    cluster_arrive_release();
    cluster_wait();
    if (rank == 0 && threadIdx.x == 0)
      asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(t.ready + group), "r"(t.seq) : "memory");
  }
}

// ---------------------------------------------------------------- launchers
// Raises the kernel's dynamic shared-memory limit to `bytes` when a launch
// needs more than the previous ones on this device (static + dynamic above
// 48 KB needs the opt-in).  One cache per kernel instantiation (the caller's
// static array).
template <typename K>
cudaError_t allow_smem(K kern, size_t bytes, int (&allowed)[64]) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || allowed[dev] >= static_cast<int>(bytes)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) allowed[dev] = static_cast<int>(bytes);
  return e;
}

template <typename E, int NCH, bool AGG_MAX>
cudaError_t run_block_select_agg(const BlockScoreArgs &a, cudaStream_t st) {
  constexpr int CS = kClusterSize;
  const int rows = (a.n_blocks_max + CS - 1) / CS;  // <= kSliceCap
  const int qrows = AGG_MAX ? a.n_q_heads / a.n_kv_heads : 1;
  const size_t smem =
      static_cast<size_t>(qrows) * 2 * a.d * sizeof(float) + static_cast<size_t>(rows) * sizeof(uint32_t);
  static int allowed[64] = {};
  cudaError_t e = allow_smem(block_select_kernel<E, NCH, CS, AGG_MAX>, smem, allowed);
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(block_select_kernel<E, NCH, CS, AGG_MAX>, dim3(CS, a.batch * a.n_kv_heads),
                            dim3(kThreads), smem, st, CS, a, rows);
}
template <typename E, int NCH>
cudaError_t run_block_select(const BlockScoreArgs &a, cudaStream_t st) {
  if (a.from_scores) return run_block_select_agg<E, NCH, false>(a, st);  // selection only: no query in smem
  if (a.agg == 1) {
    if constexpr (NCH <= 64) return run_block_select_agg<E, NCH, true>(a, st);
    return cudaErrorInvalidValue;  // latent shapes: max aggregation not offered
  }
  return run_block_select_agg<E, NCH, false>(a, st);
}

template <typename E, typename SE, int RCH>
cudaError_t run_token_select(const TokenArgs &a, cudaStream_t st) {
  constexpr int CS = kClusterSize;
  const int per = (a.k_b * a.block_size + CS - 1) / CS;  // <= kSliceCap
  const size_t smem = static_cast<size_t>(per) * sizeof(uint32_t);
  auto kern = a.d > 128 ? token_select_kernel<E, SE, RCH, CS, true> : token_select_kernel<E, SE, RCH, CS, false>;
  static int allowed[2][64] = {};
  cudaError_t e = allow_smem(kern, smem, allowed[a.d > 128]);
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(kern, dim3(CS, a.batch * a.n_kv_heads), dim3(kThreads), smem, st, CS, a, per);
}

template <typename E, typename SE, int NCH, int RCH>
cudaError_t run_select_step(const BlockScoreArgs &a, const TokenArgs &t, cudaStream_t st) {
  constexpr int CS = kClusterSize;
  const int rows = (a.n_blocks_max + CS - 1) / CS;
  const int per = (t.k_b * t.block_size + CS - 1) / CS;
  // each CTA selecting the blocks itself pays off while the clusters do not
  // fill the GPU (few groups); with many groups the cluster exchange is cheaper
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const bool few_groups = static_cast<long long>(a.batch) * a.n_kv_heads * CS < 2LL * sms;
  const int local_n = a.from_scores && few_groups && a.n_blocks_max <= kLocalBlockKeys ? a.n_blocks_max : 0;
  const size_t head = std::max<size_t>(2 * static_cast<size_t>(a.d) + rows, static_cast<size_t>(local_n));
  const size_t smem = (head + static_cast<size_t>(per)) * sizeof(uint32_t);
  auto kern = local_n > 0 ? select_step_kernel<E, SE, NCH, RCH, CS, true> : select_step_kernel<E, SE, NCH, RCH, CS, false>;
  static int allowed[2][64] = {};
  cudaError_t e = allow_smem(kern, smem, allowed[local_n > 0]);
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(kern, dim3(CS, a.batch * a.n_kv_heads), dim3(kThreads), smem, st, CS, StepArgs{a, t},
                            rows, per, local_n);
}

template <typename E, int NCH>
cudaError_t step_by_rch(const BlockScoreArgs &a, const TokenArgs &t, cudaStream_t st) {
  if constexpr (sizeof(typename E::storage) == 2) {
    if (t.scales) {  // int8 label slab
      switch (t.n_label / 16) {
        case 1: return run_select_step<E, I8, NCH, 1>(a, t, st);
        case 2: return run_select_step<E, I8, NCH, 2>(a, t, st);
        case 4: return run_select_step<E, I8, NCH, 4>(a, t, st);
      }
      return cudaErrorInvalidValue;
    }
  }
  if (t.scales) return cudaErrorInvalidValue;
  switch (t.n_label * E::kBytes / 16) {
    case 1: return run_select_step<E, E, NCH, 1>(a, t, st);
    case 2: return run_select_step<E, E, NCH, 2>(a, t, st);
    case 4: return run_select_step<E, E, NCH, 4>(a, t, st);
    case 8: return run_select_step<E, E, NCH, 8>(a, t, st);
  }
  return cudaErrorInvalidValue;
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
  if (a.scales) {  // int8 label slab (bf16 queries)
    if (a.dtype != 1) return cudaErrorInvalidValue;
    switch (a.n_label / 16) {
      case 1: return run_token_select<BF16, I8, 1>(a, st);
      case 2: return run_token_select<BF16, I8, 2>(a, st);
      case 4: return run_token_select<BF16, I8, 4>(a, st);
    }
    return cudaErrorInvalidValue;
  }
  const int rch = a.n_label * (a.dtype == 1 ? 2 : 4) / 16;
  switch (rch) {
    case 1: return a.dtype == 1 ? run_token_select<BF16, BF16, 1>(a, st) : run_token_select<F32, F32, 1>(a, st);
    case 2: return a.dtype == 1 ? run_token_select<BF16, BF16, 2>(a, st) : run_token_select<F32, F32, 2>(a, st);
    case 4: return a.dtype == 1 ? run_token_select<BF16, BF16, 4>(a, st) : run_token_select<F32, F32, 4>(a, st);
    case 8: return a.dtype == 1 ? run_token_select<BF16, BF16, 8>(a, st) : run_token_select<F32, F32, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

bool select_two_phase(int groups, int heads_per_group, int num_sms, size_t summary_bytes, bool folded_queries) {
  // One cluster of kClusterSize CTAs per group: with fewer clusters than fill
  // the SMs twice over, the summary stream is short of loads in flight.  Below
  // a few MB of summary the extra launch costs more than it saves.  With many
  // heads per group the queries must be folded once per group beforehand
  // (launch_query_fold): folded by every phase-1 CTA, the fold costs more than
  // the stream (measured: gqa48k 21.9 -> 18.4 us; the 64-head latent
  // 33.8 -> 37.7 us without the separate fold).
  return static_cast<long long>(groups) * kClusterSize < 2LL * num_sms && summary_bytes >= (size_t(4) << 20) &&
         (heads_per_group <= 16 || folded_queries);
}

cudaError_t launch_query_fold(const BlockScoreArgs &a, cudaStream_t st) {
  if (!a.qfold) return cudaErrorInvalidValue;
  const unsigned groups = static_cast<unsigned>(a.batch * a.n_kv_heads);
  if (a.dtype == 1 && a.d > 128)  // the fold of score_blocks<BF16, 144>: parallel, 8 chunk columns per CTA
    return launch_pdl(query_fold_kernel<BF16, 144>, dim3(groups, (a.d / 8 + 7) / 8), dim3(32), 0, st, a);
  if (a.dtype == 1) return launch_pdl(query_fold_kernel<BF16, 32>, dim3(groups), dim3(kThreads), 0, st, a);
  return launch_pdl(query_fold_kernel<F32, 32>, dim3(groups), dim3(kThreads), 0, st, a);
}

namespace {
template <typename E, int NCH>
cudaError_t run_block_scores(const BlockScoreArgs &a, int num_sms, cudaStream_t st) {
  const long long total = static_cast<long long>(a.batch) * a.n_kv_heads * a.n_blocks_max;
  // one wave: the kernel's resident CTAs per SM (2 for the latent rows' 128 registers, else 4)
  const int ctas = static_cast<int>(std::max<long long>(1, std::min<long long>((NCH > 32 ? 2LL : 4LL) * num_sms, total)));
  const int rows = static_cast<int>((total + ctas - 1) / ctas);
  const int grid = static_cast<int>((total + rows - 1) / rows);
  const size_t smem = 2 * static_cast<size_t>(a.d) * sizeof(float);
  if (a.qfold) return launch_pdl(block_scores_kernel<E, NCH, true>, dim3(grid), dim3(kThreads), smem, st, a, rows);
  return launch_pdl(block_scores_kernel<E, NCH, false>, dim3(grid), dim3(kThreads), smem, st, a, rows);
}
}  // namespace

cudaError_t launch_block_scores(const BlockScoreArgs &a, int num_sms, cudaStream_t st) {
  if (!a.scores) return cudaErrorInvalidValue;
  const int nch = 2 * a.d * (a.dtype == 1 ? 2 : 4) / 16;
  if (a.dtype == 1) {
    switch (nch) {
      case 16: return run_block_scores<BF16, 16>(a, num_sms, st);
      case 32: return run_block_scores<BF16, 32>(a, num_sms, st);
      case 144: return run_block_scores<BF16, 144>(a, num_sms, st);
    }
  } else {
    switch (nch) {
      case 32: return run_block_scores<F32, 32>(a, num_sms, st);
      case 64: return run_block_scores<F32, 64>(a, num_sms, st);
    }
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_select_step(const BlockScoreArgs &a, const TokenArgs &t, cudaStream_t st) {
  const int nch = 2 * a.d * (a.dtype == 1 ? 2 : 4) / 16;
  if (a.dtype == 1) {
    switch (nch) {
      case 16: return step_by_rch<BF16, 16>(a, t, st);
      case 32: return step_by_rch<BF16, 32>(a, t, st);
      case 144: return step_by_rch<BF16, 144>(a, t, st);
    }
  } else {
    switch (nch) {
      case 32: return step_by_rch<F32, 32>(a, t, st);
      case 64: return step_by_rch<F32, 64>(a, t, st);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace tls
