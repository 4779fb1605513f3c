// tls_attn_mma.cu -- stage 5 of the AsyncTLS decode step for bf16 GQA shapes:
// exact softmax attention over the gathered K/V rows of the selected tokens
// (gist.science (es) section 2.A.2: the final attention runs at token
// precision on the K_t kept tokens), with the two per-tile contractions on
// the tensor cores through warp-level MMAs.
//
// Work split, gather pipeline and partial layout are those of the CUDA-core
// kernel in tls_attn.cu (persistent grid, one contiguous range of 16-token
// tiles per warp, a private cp.async ring per warp, partial (max, sum, o)
// per unit and piece, log-sum-exp merge kernel).  Per tile, one warp:
//   S = Q K^T   mma m16n8k16 (bf16 in, fp32 accumulate): M = the unit's heads
//               (up to 8 heads use rows 0-7 and leave rows 8-15 zero; a unit
//               of 16 heads fills all 16 rows, two per lane quad; Q fragments
//               stay in registers for the unit), N = 8 tokens x 2, K = d in
//               steps of 16; K fragments come from the XOR-swizzled stage
//               buffer through ldmatrix.
//   online softmax in the log2 domain on the S accumulators (a row = a head
//               lives in one lane quad: max and sum are two quad shuffles).
//   O += P V    the S accumulator layout of two 8-token blocks is exactly the
//               A-fragment layout of P over 16 tokens, so P never leaves the
//               registers; P is split into bf16 hi + lo parts (two MMAs, about
//               2^-17 relative error on P) and V fragments come from the
//               swizzled stage buffer through ldmatrix.trans.
// The tensor cores replace ~40 FMA-pipe instructions per token and head
// group with 3 MMAs, which moves the kernel from issue-bound to HBM-bound on
// the gathered rows.  Groups of 32 or 64 heads (MQA-like shapes) are cut
// into units of 16 heads that gather the group's rows each; the units of one
// group sit in adjacent warps, so the repeated gathers mostly hit L2.
#include <cuda_bf16.h>

#include <algorithm>

#include "tls_device.cuh"
#include "tls_internal.h"
#include "tls_mma.cuh"

namespace tls {
namespace {

template <int D, int HG, bool PAGED, int NS>
__global__ void __launch_bounds__(MmaLayout<D, NS>::W * 32, 1) attn_mma_kernel(AttnArgs a, AttnPlan p) {
  using L = MmaLayout<D, NS>;
  constexpr int KS = D / 16;  // k-steps of S = Q K^T
  constexpr int NB = D / 8;   // 8-channel blocks of O
  constexpr int R = HG > 8 ? 2 : 1;  // MMA rows per lane: lane/4 (and lane/4 + 8)
  static_assert(HG <= 16, "a unit's heads fit the 16 MMA rows");
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned char *wbase = smem + warp * L::kWarpBytes;
  long long *Off = reinterpret_cast<long long *>(wbase + NS * L::kStageBytes);  // [NS][kMT] byte offsets
  uint32_t *Mask = reinterpret_cast<uint32_t *>(Off + NS * kMT);                 // [NS] valid-token bits

  // With readiness words the selection launch before this one let it start
  // early; each warp then waits for its groups (issue_next) instead of the grid.
  if (!a.ready) grid_dependency_wait();
  const int gw = blockIdx.x * L::W + warp;
  const int t_begin = gw * p.tiles_per_warp;
  const int t_end = min(t_begin + p.tiles_per_warp, p.total_tiles);
  if (t_begin >= t_end) return;

  const unsigned char *Kb = static_cast<const unsigned char *>(a.K);
  const unsigned char *Vb = PAGED ? Kb : static_cast<const unsigned char *>(a.V);
  const long long v_delta = PAGED ? static_cast<long long>(a.block_size) * L::RB : 0;
  const int Gt = a.n_q_heads / a.n_kv_heads;

  // Gather the K and V rows of tile t into stage st (the caller commits).
  // Issue cursor: tile iss_t (its group, head chunk, tile within the unit,
  // ring stage) advances by counting, so no integer division sits on the
  // per-tile path.  A unit is one head chunk of one group.
  const int nhc = p.n_head_chunks;
  const int unit0 = t_begin / p.tiles_per_group;
  int iss_t = t_begin, iss_group = unit0 / nhc, iss_hc = unit0 % nhc, iss_tile = t_begin % p.tiles_per_group,
      iss_st = 0;
  int ready_group = -1;  // the last group whose readiness word this warp has seen
  auto issue_next = [&]() {
    const int t = iss_t, st = iss_st, tile = iss_tile, group = iss_group;
    if (++iss_tile == p.tiles_per_group) {
      iss_tile = 0;
      if (++iss_hc == nhc) {
        iss_hc = 0;
        ++iss_group;
      }
    }
    ++iss_t;
    if (++iss_st == NS) iss_st = 0;
    if (t < t_end) {
      if (a.ready && group != ready_group) {  // bounded wait for the group's token ids
        if (lane == 0) {
          bool ok = false;
          for (uint32_t i = 0; i < (1u << 22) && !ok; ++i) {
            int v;
            asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(a.ready + group) : "memory");
            ok = v == a.seq;
            if (!ok) __nanosleep(i < 16 ? 32 : 256);
          }
          if (!ok && a.err) atomicOr(a.err, kErrAttnWait);
        }
        __syncwarp();
        ready_group = group;
      }
      long long off = -1;
      if (lane < kMT) {
        const int j = tile * kMT + lane;
        if (j < a.k_t) {
          const int tok = __ldcg(a.token_idx + static_cast<size_t>(group) * a.k_t + j);
          if (tok >= 0 && tok < a.max_ctx) {
            if constexpr (PAGED) {
              const int slot = a.slot_of_block[static_cast<size_t>(group) * a.n_blocks_max + tok / a.block_size];
              if (slot >= 0 && slot < a.n_slots)
                off = ((static_cast<long long>(group) * a.n_slots + slot) * 2 * a.block_size + tok % a.block_size) *
                      L::RB;
            } else {
              off = (static_cast<long long>(group) * a.max_ctx + tok) * L::RB;
            }
          }
        }
        Off[st * kMT + lane] = off;
      }
      const unsigned vm = __ballot_sync(0xffffffffu, off >= 0);
      if (lane == 0) Mask[st] = vm;
      __syncwarp();
      unsigned char *Ks = wbase + st * L::kStageBytes;
      unsigned char *Vs = Ks + kMT * L::RB;
#pragma unroll
      for (int i = 0; i < kMT * L::CH / 32; ++i) {
        const int idx = i * 32 + lane;
        const int row = idx / L::CH, c = idx % L::CH;
        const long long o = Off[st * kMT + row];
        const bool ok = o >= 0;
        const long long ob = ok ? o : 0;
        const int sw = (c ^ (row & 7)) << 4;
        cp_async16(Ks + row * L::RB + sw, Kb + ob + (c << 4), ok);
        cp_async16(Vs + row * L::RB + sw, Vb + ob + v_delta + (c << 4), ok);
      }
    }
  };

  const int g = lane >> 2;          // MMA row of this lane = head within the unit (and g + 8 when R = 2)
  const int tq = 2 * (lane & 3);    // first of this lane's token (or channel) pair
  // A fragments of Q: R = 1 {rows g: ch tq, ch 8 + tq}; R = 2 {g, g + 8, g: 8 + tq, g + 8: 8 + tq}
  uint32_t qa[KS][2 * R];
  float o[NB][2 * R];               // O[g (+ 8 r)][8j + tq .. + 1] at [j][2r .. 2r + 1]
  float m_run[R], l_run[R];
  int cur_unit = -1;

  auto flush = [&](int unit) {
    const int first = (unit * p.tiles_per_group) / p.tiles_per_warp;
    const int piece = gw - first;
    const size_t units = static_cast<size_t>(a.batch) * a.n_kv_heads * p.n_head_chunks;
    float *ml = a.part + (static_cast<size_t>(unit) * p.max_pieces + piece) * HG * 2;
    float *po = a.part + units * p.max_pieces * HG * 2 + (static_cast<size_t>(unit) * p.max_pieces + piece) * HG * D;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float lt = l_run[r];
      lt += __shfl_xor_sync(0xffffffffu, lt, 1);
      lt += __shfl_xor_sync(0xffffffffu, lt, 2);
      const int h = g + 8 * r;
      if (h < HG) {
        if ((lane & 3) == 0) {
          ml[h * 2] = m_run[r];
          ml[h * 2 + 1] = lt;
        }
#pragma unroll
        for (int j = 0; j < NB; ++j)
          *reinterpret_cast<float2 *>(po + h * D + 8 * j + tq) = make_float2(o[j][2 * r], o[j][2 * r + 1]);
      }
    }
  };

  auto start_unit = [&](int unit) {  // unit = group * n_head_chunks + head chunk
    const int group = unit / nhc, hc = unit % nhc;
    const int b = group / a.n_kv_heads, gk = group % a.n_kv_heads;
    const uint32_t *q = static_cast<const uint32_t *>(a.q);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int h = g + 8 * r;
      const size_t row = (static_cast<size_t>(b) * a.n_q_heads + gk * Gt + hc * HG + h) * D;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        qa[kk][r] = h < HG ? q[(row + 16 * kk + tq) / 2] : 0u;
        qa[kk][R + r] = h < HG ? q[(row + 16 * kk + 8 + tq) / 2] : 0u;
      }
      m_run[r] = -INFINITY;
      l_run[r] = 0.f;
    }
#pragma unroll
    for (int j = 0; j < NB; ++j)
#pragma unroll
      for (int i = 0; i < 2 * R; ++i) o[j][i] = 0.f;
  };

  const int mi = lane >> 3, mr = lane & 7;  // ldmatrix: matrix index and row of this lane's address
#pragma unroll
  for (int s = 0; s < NS - 1; ++s) {
    issue_next();
    cp_async_commit();
  }

  // compute cursor: tile t, its unit and ring stage
  int unit = t_begin / p.tiles_per_group, tile_in_unit = t_begin % p.tiles_per_group, st = 0;
  for (int t = t_begin; t < t_end; ++t) {
    issue_next();
    cp_async_commit();
    cp_async_wait<NS - 1>();
    __syncwarp();
    if (unit != cur_unit) {
      if (cur_unit >= 0) flush(cur_unit);
      start_unit(unit);
      cur_unit = unit;
    }
    const unsigned char *Ks = wbase + st * L::kStageBytes;
    const unsigned char *Vs = Ks + kMT * L::RB;
    const uint32_t vmask = Mask[st];

    // ---- S = Q K^T: tokens 0-7 -> s0, 8-15 -> s1 (row g at [0..1], row g + 8 at [2..3])
    float s0[2 * R], s1[2 * R];
#pragma unroll
    for (int i = 0; i < 2 * R; ++i) s0[i] = s1[i] = 0.f;
    {
      const int tok = (mi >> 1) * 8 + mr;
      const uint32_t rowa = smem_addr(Ks + tok * L::RB);
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        const int ch = 2 * kk + (mi & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(rowa + ((ch ^ (tok & 7)) << 4), b0, b1, b2, b3);
        mma_r<R>(s0, qa[kk], b0, b1);
        mma_r<R>(s1, qa[kk], b2, b3);
      }
    }
    // ---- online softmax, log2 domain; lanes of a quad share a row (head)
    const int tk[4] = {tq, tq + 1, 8 + tq, 9 + tq};
    float alpha[R], pr[R][4];
    bool rescale = false;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float sc[4] = {s0[2 * r], s0[2 * r + 1], s1[2 * r], s1[2 * r + 1]};
#pragma unroll
      for (int i = 0; i < 4; ++i) sc[i] = ((vmask >> tk[i]) & 1u) ? sc[i] * a.scale_log2 : -INFINITY;
      float mt = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
      const float mn = fmaxf(m_run[r], mt);
      alpha[r] = 1.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) pr[r][i] = 0.f;
      if (mn != -INFINITY) {
        alpha[r] = ex2(m_run[r] - mn);
#pragma unroll
        for (int i = 0; i < 4; ++i) pr[r][i] = ex2(sc[i] - mn);
      }
      l_run[r] = l_run[r] * alpha[r] + ((pr[r][0] + pr[r][1]) + (pr[r][2] + pr[r][3]));
      m_run[r] = mn;
      rescale |= alpha[r] != 1.f;
    }
    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
      for (int j = 0; j < NB; ++j)
#pragma unroll
        for (int r = 0; r < R; ++r) {
          o[j][2 * r] *= alpha[r];
          o[j][2 * r + 1] *= alpha[r];
        }
    }
    // P as the A operand over 16 tokens, hi and lo parts: the same fragment
    // order as Q ({row g: tokens tq.., (row g + 8: tokens tq..), row g: 8 + tq.., (row g + 8: 8 + tq..)})
    uint32_t ph[2 * R], pl[2 * R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      split_bf16(pr[r][0], pr[r][1], ph[r], pl[r]);
      split_bf16(pr[r][2], pr[r][3], ph[R + r], pl[R + r]);
    }
    // ---- O += P V
    {
      const int tok = (mi & 1) * 8 + mr;
      const uint32_t rowa = smem_addr(Vs + tok * L::RB);
#pragma unroll
      for (int j = 0; j < NB; j += 2) {
        const int ch = j + (mi >> 1);
        uint32_t v0, v1, v2, v3;
        ldsm_x4_t(rowa + ((ch ^ (tok & 7)) << 4), v0, v1, v2, v3);
        mma_r<R>(o[j], ph, v0, v1);
        mma_r<R>(o[j], pl, v0, v1);
        mma_r<R>(o[j + 1], ph, v2, v3);
        mma_r<R>(o[j + 1], pl, v2, v3);
      }
    }
    __syncwarp();
    if (++tile_in_unit == p.tiles_per_group) {
      tile_in_unit = 0;
      ++unit;
    }
    if (++st == NS) st = 0;
  }
  if (cur_unit >= 0) flush(cur_unit);
  cp_async_wait<0>();
}

template <int D, int HG, bool PAGED>
cudaError_t run_mma(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  using L = MmaLayout<D, kMmaStages>;
  auto kern = attn_mma_kernel<D, HG, PAGED, kMmaStages>;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  return launch_pdl(kern, dim3(p.grid), dim3(L::W * 32), L::kSmem, st, a, p);
}

template <int D, bool PAGED>
cudaError_t dispatch_mma(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  switch (p.head_chunk) {
    case 1: return run_mma<D, 1, PAGED>(a, p, st);
    case 2: return run_mma<D, 2, PAGED>(a, p, st);
    case 4: return run_mma<D, 4, PAGED>(a, p, st);
    case 8: return run_mma<D, 8, PAGED>(a, p, st);
    case 16: return run_mma<D, 16, PAGED>(a, p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool attn_mma_supported(const AttnArgs &a) {
  const int G = a.n_q_heads / a.n_kv_heads;
  return a.dtype == 1 && !a.v_is_k_prefix && a.d_qk == a.d_v && (a.d_qk == 64 || a.d_qk == 128) &&
         (G == 1 || G == 2 || G == 4 || G == 8 || G == 16 || G == 32 || G == 64);
}

int attn_mma_head_chunk(const AttnArgs &a) { return std::min(a.n_q_heads / a.n_kv_heads, 16); }

int attn_mma_warps(const AttnArgs &a) {
  return a.d_qk == 64 ? MmaLayout<64, kMmaStages>::W : MmaLayout<128, kMmaStages>::W;
}

cudaError_t launch_attention_mma(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  if (a.d_qk == 128) return a.paged ? dispatch_mma<128, true>(a, p, st) : dispatch_mma<128, false>(a, p, st);
  return a.paged ? dispatch_mma<64, true>(a, p, st) : dispatch_mma<64, false>(a, p, st);
}

}  // namespace tls
