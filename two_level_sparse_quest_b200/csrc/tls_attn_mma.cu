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
//               (rows padded to 16; Q fragments stay in registers for the
//               unit), N = 8 tokens x 2, K = d in steps of 16; K fragments come
//               from the XOR-swizzled stage buffer through ldmatrix.
//   online softmax in the log2 domain on the S accumulators (a row = a head
//               lives in one lane quad: max and sum are two quad shuffles).
//   O += P V    the S accumulator layout of two 8-token blocks is exactly the
//               A-fragment layout of P over 16 tokens, so P never leaves the
//               registers; P is split into bf16 hi + lo parts (two MMAs, about
//               2^-17 relative error on P) and V fragments come from the
//               swizzled stage buffer through ldmatrix.trans.
// The tensor cores replace ~40 FMA-pipe instructions per token and head
// group with 3 MMAs, which moves the kernel from issue-bound to HBM-bound on
// the gathered rows.
#include <cuda_bf16.h>

#include <algorithm>

#include "tls_device.cuh"
#include "tls_internal.h"

namespace tls {
namespace {

constexpr int kMT = 16;  // tokens per tile
constexpr int kMmaStages = 3;

template <int D, int NS>
struct MmaLayout {
  static constexpr int RB = D * 2;                 // bytes of one K (or V) row
  static constexpr int CH = RB / 16;               // 16-byte chunks per row
  static constexpr int kStageBytes = 2 * kMT * RB;  // K tile then V tile
  // ring, row offsets, valid-token masks; rounded to 128 bytes so that every
  // warp's ring (cp.async and ldmatrix targets) stays 16-byte aligned
  static constexpr int kWarpBytes = (NS * kStageBytes + NS * kMT * 8 + NS * 8 + 127) / 128 * 128;
  static constexpr int kMaxSmem = 227 * 1024;
  static constexpr int W = (kMaxSmem / kWarpBytes) < 16 ? (kMaxSmem / kWarpBytes) : 16;  // warps per CTA
  static constexpr int kSmem = W * kWarpBytes;
  static_assert(CH % 8 == 0, "the row swizzle permutes groups of 8 chunks");
  static_assert((kMT * CH) % 32 == 0, "the issue loop covers whole warps");
  static_assert(W >= 1, "one warp's ring must fit in shared memory");
  static_assert(kWarpBytes % 16 == 0 && kStageBytes % 16 == 0 && RB % 16 == 0, "16-byte aligned rows and rings");
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// c[0..1] += A B for the rows of this lane (row lane/4); the A rows lane/4 + 8
// are zero (a1 = a3 = 0) and the matching accumulator halves are discarded.
__device__ __forceinline__ void mma_rows(float (&c)[2], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  float d2, d3;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %10, %11};"
      : "+f"(c[0]), "+f"(c[1]), "=f"(d2), "=f"(d3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(0.f), "f"(0.f));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}
// x = bf16 hi part + bf16 lo part (the lo part holds the rounding error of hi)
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  hi = pack_bf16(x0, x1);
  lo = pack_bf16(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
}

template <int D, int HG, bool PAGED, int NS>
__global__ void __launch_bounds__(MmaLayout<D, NS>::W * 32, 1) attn_mma_kernel(AttnArgs a, AttnPlan p) {
  using L = MmaLayout<D, NS>;
  constexpr int KS = D / 16;  // k-steps of S = Q K^T
  constexpr int NB = D / 8;   // 8-channel blocks of O
  static_assert(HG <= 8, "a head group fits the first 8 MMA rows");
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned char *wbase = smem + warp * L::kWarpBytes;
  long long *Off = reinterpret_cast<long long *>(wbase + NS * L::kStageBytes);  // [NS][kMT] byte offsets
  uint32_t *Mask = reinterpret_cast<uint32_t *>(Off + NS * kMT);                 // [NS] valid-token bits

  grid_dependency_wait();
  const int gw = blockIdx.x * L::W + warp;
  const int t_begin = gw * p.tiles_per_warp;
  const int t_end = min(t_begin + p.tiles_per_warp, p.total_tiles);
  if (t_begin >= t_end) return;

  const unsigned char *Kb = static_cast<const unsigned char *>(a.K);
  const unsigned char *Vb = PAGED ? Kb : static_cast<const unsigned char *>(a.V);
  const long long v_delta = PAGED ? static_cast<long long>(a.block_size) * L::RB : 0;
  const int Gt = a.n_q_heads / a.n_kv_heads;

  // Gather the K and V rows of tile t into stage st (the caller commits).
  // Issue cursor: tile iss_t (its unit = group, tile within the group, ring
  // stage) advances by counting, so no integer division sits on the per-tile
  // path.  A unit is one GQA group (the plan has one head chunk per group).
  int iss_t = t_begin, iss_group = t_begin / p.tiles_per_group, iss_tile = t_begin % p.tiles_per_group, iss_st = 0;
  auto issue_next = [&]() {
    const int t = iss_t, st = iss_st, tile = iss_tile, group = iss_group;
    if (++iss_tile == p.tiles_per_group) {
      iss_tile = 0;
      ++iss_group;
    }
    ++iss_t;
    if (++iss_st == NS) iss_st = 0;
    if (t < t_end) {
      long long off = -1;
      if (lane < kMT) {
        const int j = tile * kMT + lane;
        if (j < a.k_t) {
          const int tok = a.token_idx[static_cast<size_t>(group) * a.k_t + j];
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

  const int g = lane >> 2;          // MMA row of this lane = head within the unit
  const int tq = 2 * (lane & 3);    // first of this lane's token (or channel) pair
  uint32_t qa[KS][2];               // A fragments of Q (rows g; rows g + 8 are zero)
  float o[NB][2];                   // O[g][8j + tq .. + 1]
  float m_run = -INFINITY, l_run = 0.f;
  int cur_unit = -1;

  auto flush = [&](int unit) {
    float lt = l_run;
    lt += __shfl_xor_sync(0xffffffffu, lt, 1);
    lt += __shfl_xor_sync(0xffffffffu, lt, 2);
    const int first = (unit * p.tiles_per_group) / p.tiles_per_warp;
    const int piece = gw - first;
    const size_t units = static_cast<size_t>(a.batch) * a.n_kv_heads * p.n_head_chunks;
    float *ml = a.part + (static_cast<size_t>(unit) * p.max_pieces + piece) * HG * 2;
    float *po = a.part + units * p.max_pieces * HG * 2 + (static_cast<size_t>(unit) * p.max_pieces + piece) * HG * D;
    if (g < HG) {
      if ((lane & 3) == 0) {
        ml[g * 2] = m_run;
        ml[g * 2 + 1] = lt;
      }
#pragma unroll
      for (int j = 0; j < NB; ++j)
        *reinterpret_cast<float2 *>(po + g * D + 8 * j + tq) = make_float2(o[j][0], o[j][1]);
    }
  };

  auto start_unit = [&](int unit) {  // unit = group
    const int b = unit / a.n_kv_heads, gk = unit % a.n_kv_heads;
    const uint32_t *q = static_cast<const uint32_t *>(a.q);
    const size_t row = (static_cast<size_t>(b) * a.n_q_heads + gk * Gt + g) * D;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      qa[kk][0] = g < HG ? q[(row + 16 * kk + tq) / 2] : 0u;
      qa[kk][1] = g < HG ? q[(row + 16 * kk + 8 + tq) / 2] : 0u;
    }
#pragma unroll
    for (int j = 0; j < NB; ++j) o[j][0] = o[j][1] = 0.f;
    m_run = -INFINITY;
    l_run = 0.f;
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

    // ---- S = Q K^T: tokens 0-7 -> s0, 8-15 -> s1
    float s0[2] = {0.f, 0.f}, s1[2] = {0.f, 0.f};
    {
      const int tok = (mi >> 1) * 8 + mr;
      const uint32_t rowa = smem_addr(Ks + tok * L::RB);
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        const int ch = 2 * kk + (mi & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(rowa + ((ch ^ (tok & 7)) << 4), b0, b1, b2, b3);
        mma_rows(s0, qa[kk][0], qa[kk][1], b0, b1);
        mma_rows(s1, qa[kk][0], qa[kk][1], b2, b3);
      }
    }
    // ---- online softmax, log2 domain; lanes of a quad share a row (head)
    float sc[4] = {s0[0], s0[1], s1[0], s1[1]};
    const int tk[4] = {tq, tq + 1, 8 + tq, 9 + tq};
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[i] = ((vmask >> tk[i]) & 1u) ? sc[i] * a.scale_log2 : -INFINITY;
    float mt = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
    const float mn = fmaxf(m_run, mt);
    float alpha = 1.f, pr[4] = {0.f, 0.f, 0.f, 0.f};
    if (mn != -INFINITY) {
      alpha = ex2(m_run - mn);
#pragma unroll
      for (int i = 0; i < 4; ++i) pr[i] = ex2(sc[i] - mn);
    }
    l_run = l_run * alpha + ((pr[0] + pr[1]) + (pr[2] + pr[3]));
    m_run = mn;
    if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
      for (int j = 0; j < NB; ++j) {
        o[j][0] *= alpha;
        o[j][1] *= alpha;
      }
    }
    uint32_t ph0, pl0, ph1, pl1;  // P over tokens tq..tq+1 (0) and 8+tq..9+tq (1), hi and lo parts
    split_bf16(pr[0], pr[1], ph0, pl0);
    split_bf16(pr[2], pr[3], ph1, pl1);
    // ---- O += P V
    {
      const int tok = (mi & 1) * 8 + mr;
      const uint32_t rowa = smem_addr(Vs + tok * L::RB);
#pragma unroll
      for (int j = 0; j < NB; j += 2) {
        const int ch = j + (mi >> 1);
        uint32_t v0, v1, v2, v3;
        ldsm_x4_t(rowa + ((ch ^ (tok & 7)) << 4), v0, v1, v2, v3);
        mma_rows(o[j], ph0, ph1, v0, v1);
        mma_rows(o[j], pl0, pl1, v0, v1);
        mma_rows(o[j + 1], ph0, ph1, v2, v3);
        mma_rows(o[j + 1], pl0, pl1, v2, v3);
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
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool attn_mma_supported(const AttnArgs &a) {
  const int G = a.n_q_heads / a.n_kv_heads;
  return a.dtype == 1 && !a.v_is_k_prefix && a.d_qk == a.d_v && (a.d_qk == 64 || a.d_qk == 128) &&
         (G == 1 || G == 2 || G == 4 || G == 8);
}

int attn_mma_warps(const AttnArgs &a) {
  return a.d_qk == 64 ? MmaLayout<64, kMmaStages>::W : MmaLayout<128, kMmaStages>::W;
}

cudaError_t launch_attention_mma(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  if (p.n_head_chunks != 1) return cudaErrorInvalidValue;  // the kernel takes a unit to be a whole group
  if (a.d_qk == 128) return a.paged ? dispatch_mma<128, true>(a, p, st) : dispatch_mma<128, false>(a, p, st);
  return a.paged ? dispatch_mma<64, true>(a, p, st) : dispatch_mma<64, false>(a, p, st);
}

}  // namespace tls
