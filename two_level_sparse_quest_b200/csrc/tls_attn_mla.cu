// tls_attn_mla.cu -- stage 5 of the AsyncTLS decode step for latent (MLA)
// shapes: every query head attends over the same 576-channel latent rows of
// the kept tokens, V being the first 512 channels of each row (gist.science
// (es) section 2.A.2: the final attention runs at token precision on the K_t
// kept tokens).  64 heads x 576 channels per kept token is a real dense
// contraction (~120 flop per byte gathered), so both products run on the
// tensor cores through warp-level MMAs, and each row is gathered once for all
// heads.
//
//   * A CTA owns a contiguous range of 16-token tiles of the flattened
//     (group, tile) space.  The group's queries (G x 576 bf16) and a 4-stage
//     ring of gathered rows (16 x 1152 bytes per stage) sit in shared memory,
//     chunks XOR-swizzled by row inside groups of 8 so that ldmatrix reads
//     are conflict-free.  All 256 threads gather a stage with 16-byte cp.async
//     copies (zero-fill for masked tokens).
//   * Warp w owns 16 heads (head tile w % HT) and a slice of the 512 output
//     channels (part w / HT of 8 / HT).  Per tile it computes S = Q K^T for its
//     16 heads (mma m16n8k16, bf16 in, fp32 accumulate; 36 k-steps, Q and K
//     fragments through ldmatrix), the online softmax of its two rows per lane
//     (log2 domain), and O += P V over its channels, with P split into bf16
//     hi + lo parts and V fragments through ldmatrix.trans of the same rows.
//   * When the CTA's range leaves a group, each warp writes its partial
//     (max, sum, o) for its heads and channels; the log-sum-exp merge kernel of
//     tls_attn.cu combines the CTAs' pieces.
#include <cuda_bf16.h>

#include <algorithm>

#include "tls_device.cuh"
#include "tls_internal.h"

namespace tls {
namespace {

constexpr int kD = 576, kDV = 512;
constexpr int kRB = kD * 2;          // bytes of one latent row
constexpr int kCH = kRB / 16;        // 72 chunks of 16 bytes
constexpr int kT = 16;               // tokens per tile
constexpr int kNS = 4;               // ring stages
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kStageBytes = kT * kRB;
constexpr int kMaxG = 64;
constexpr int kQBytes = kMaxG * kRB;
constexpr int kOffOff = kQBytes + kNS * kStageBytes;
constexpr int kMaskOff = kOffOff + kNS * kT * 8;
constexpr int kSmem = kMaskOff + kNS * 4;
static_assert(kSmem <= 227 * 1024, "fits in shared memory");
static_assert(kCH % 8 == 0, "the swizzle permutes groups of 8 chunks");

// physical 16-byte chunk of logical chunk c in row r
__device__ __forceinline__ int swz(int c, int r) { return (c & ~7) | ((c ^ r) & 7); }

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
// c += A B over a full m16n8k16 tile (all 16 A rows real)
__device__ __forceinline__ void mma16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                      uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  hi = pack_bf16(x0, x1);
  lo = pack_bf16(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
}

// HT: head tiles of 16 (G = 16 * HT); a warp covers 512 / (8 / HT) channels.
template <int HT>
__global__ void __launch_bounds__(kThreads, 1) attn_mla_kernel(AttnArgs a, AttnPlan p) {
  constexpr int G = 16 * HT;
  constexpr int NCP = kWarps / HT;     // channel parts
  constexpr int CPW = kDV / NCP;       // channels per warp
  constexpr int NBW = CPW / 8;         // 8-channel blocks per warp
  static_assert(NBW % 2 == 0, "ldmatrix.x4.trans covers two channel blocks");
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char *Qs = smem;
  unsigned char *stages = smem + kQBytes;
  long long *Off = reinterpret_cast<long long *>(smem + kOffOff);
  uint32_t *Mask = reinterpret_cast<uint32_t *>(smem + kMaskOff);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ht = warp % HT, cpart = warp / HT;
  grid_dependency_wait();
  const int tpc = p.tiles_per_warp;  // tiles per CTA
  const int t_begin = blockIdx.x * tpc;
  const int t_end = min(t_begin + tpc, p.total_tiles);
  if (t_begin >= t_end) return;
  const unsigned char *Kb = static_cast<const unsigned char *>(a.K);
  const unsigned char *qb = static_cast<const unsigned char *>(a.q);

  // issue cursor
  int iss_t = t_begin, iss_group = t_begin / p.tiles_per_group, iss_tile = t_begin % p.tiles_per_group, iss_st = 0;
  auto issue_next = [&]() {  // whole CTA; contains __syncthreads
    const int t = iss_t, st = iss_st, tile = iss_tile, group = iss_group;
    if (++iss_tile == p.tiles_per_group) {
      iss_tile = 0;
      ++iss_group;
    }
    ++iss_t;
    if (++iss_st == kNS) iss_st = 0;
    if (t >= t_end) return;
    if (warp == 0) {
      long long off = -1;
      if (lane < kT) {
        const int j = tile * kT + lane;
        if (j < a.k_t) {
          const int tok = a.token_idx[static_cast<size_t>(group) * a.k_t + j];
          if (tok >= 0 && tok < a.max_ctx) off = (static_cast<long long>(group) * a.max_ctx + tok) * kRB;
        }
        Off[st * kT + lane] = off;
      }
      const unsigned vm = __ballot_sync(0xffffffffu, off >= 0);
      if (lane == 0) Mask[st] = vm;
    }
    __syncthreads();
    unsigned char *S = stages + st * kStageBytes;
    for (int idx = tid; idx < kT * kCH; idx += kThreads) {
      const int row = idx / kCH, c = idx % kCH;
      const long long o = Off[st * kT + row];
      const bool ok = o >= 0;
      cp_async16(S + row * kRB + (swz(c, row) << 4), Kb + (ok ? o : 0) + (c << 4), ok);
    }
  };
  auto load_q = [&](int group) {  // whole CTA, cp.async into Qs
    const int b = group / a.n_kv_heads, gk = group % a.n_kv_heads;
    const unsigned char *src = qb + (static_cast<size_t>(b) * a.n_q_heads + gk * G) * kRB;
    for (int idx = tid; idx < G * kCH; idx += kThreads) {
      const int row = idx / kCH, c = idx % kCH;
      cp_async16(Qs + row * kRB + (swz(c, row) << 4), src + static_cast<size_t>(row) * kRB + (c << 4), true);
    }
  };

  const int g = lane >> 2, tq = 2 * (lane & 3);
  const int mi = lane >> 3, mr = lane & 7;
  float o[NBW][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows g and g + 8
  auto reset = [&]() {
#pragma unroll
    for (int j = 0; j < NBW; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
  };
  auto flush = [&](int unit) {
    float t0 = l0, t1 = l1;
    t0 += __shfl_xor_sync(0xffffffffu, t0, 1);
    t0 += __shfl_xor_sync(0xffffffffu, t0, 2);
    t1 += __shfl_xor_sync(0xffffffffu, t1, 1);
    t1 += __shfl_xor_sync(0xffffffffu, t1, 2);
    const int first = (unit * p.tiles_per_group) / tpc;
    const int piece = blockIdx.x - first;
    const size_t units = static_cast<size_t>(a.batch) * a.n_kv_heads;
    float *ml = a.part + (static_cast<size_t>(unit) * p.max_pieces + piece) * G * 2;
    float *po = a.part + units * p.max_pieces * G * 2 + (static_cast<size_t>(unit) * p.max_pieces + piece) * G * kDV;
    const int h0 = ht * 16 + g, h1 = h0 + 8;
    if (cpart == 0 && (lane & 3) == 0) {
      ml[h0 * 2] = m0;
      ml[h0 * 2 + 1] = t0;
      ml[h1 * 2] = m1;
      ml[h1 * 2 + 1] = t1;
    }
#pragma unroll
    for (int j = 0; j < NBW; ++j) {
      const int ch = cpart * CPW + 8 * j + tq;
      *reinterpret_cast<float2 *>(po + h0 * kDV + ch) = make_float2(o[j][0], o[j][1]);
      *reinterpret_cast<float2 *>(po + h1 * kDV + ch) = make_float2(o[j][2], o[j][3]);
    }
  };

  int unit = t_begin / p.tiles_per_group, tile_in_unit = t_begin % p.tiles_per_group, st = 0;
  load_q(unit);
  reset();
  for (int s = 0; s < kNS - 1; ++s) {
    issue_next();
    cp_async_commit();
  }
  int cur_unit = unit;
  for (int t = t_begin; t < t_end; ++t) {
    issue_next();
    cp_async_commit();
    cp_async_wait<kNS - 1>();
    __syncthreads();  // stage st (and the unit's queries) landed for every thread's copies
    if (unit != cur_unit) {
      flush(cur_unit);
      __syncthreads();  // every warp is done with the old queries
      load_q(unit);
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
      reset();
      cur_unit = unit;
    }
    const unsigned char *S = stages + st * kStageBytes;
    const uint32_t vmask = Mask[st];
    // ---- S = Q K^T for this warp's 16 heads: tokens 0-7 -> s0, 8-15 -> s1
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    {
      const int qrow = ht * 16 + (mi & 1) * 8 + mr;
      const uint32_t qa = smem_addr(Qs + qrow * kRB);
      const int tok = (mi >> 1) * 8 + mr;
      const uint32_t ka = smem_addr(S + tok * kRB);
#pragma unroll 6
      for (int kk = 0; kk < kD / 16; ++kk) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        ldsm_x4(qa + (swz(2 * kk + (mi >> 1), qrow) << 4), a0, a1, a2, a3);
        ldsm_x4(ka + (swz(2 * kk + (mi & 1), tok) << 4), b0, b1, b2, b3);
        mma16(s0, a0, a1, a2, a3, b0, b1);
        mma16(s1, a0, a1, a2, a3, b2, b3);
      }
    }
    // ---- online softmax on rows g (c0, c1) and g + 8 (c2, c3), log2 domain
    const bool v0 = (vmask >> tq) & 1u, v1 = (vmask >> (tq + 1)) & 1u;
    const bool v2 = (vmask >> (8 + tq)) & 1u, v3 = (vmask >> (9 + tq)) & 1u;
    float r0[4] = {v0 ? s0[0] * a.scale_log2 : -INFINITY, v1 ? s0[1] * a.scale_log2 : -INFINITY,
                   v2 ? s1[0] * a.scale_log2 : -INFINITY, v3 ? s1[1] * a.scale_log2 : -INFINITY};
    float r1[4] = {v0 ? s0[2] * a.scale_log2 : -INFINITY, v1 ? s0[3] * a.scale_log2 : -INFINITY,
                   v2 ? s1[2] * a.scale_log2 : -INFINITY, v3 ? s1[3] * a.scale_log2 : -INFINITY};
    float mt0 = fmaxf(fmaxf(r0[0], r0[1]), fmaxf(r0[2], r0[3]));
    float mt1 = fmaxf(fmaxf(r1[0], r1[1]), fmaxf(r1[2], r1[3]));
    mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, 1));
    mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, 2));
    mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, 1));
    mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, 2));
    const float n0 = fmaxf(m0, mt0), n1 = fmaxf(m1, mt1);
    float al0 = 1.f, al1 = 1.f, p0[4] = {0.f, 0.f, 0.f, 0.f}, p1[4] = {0.f, 0.f, 0.f, 0.f};
    if (n0 != -INFINITY) {
      al0 = ex2(m0 - n0);
#pragma unroll
      for (int e = 0; e < 4; ++e) p0[e] = ex2(r0[e] - n0);
    }
    if (n1 != -INFINITY) {
      al1 = ex2(m1 - n1);
#pragma unroll
      for (int e = 0; e < 4; ++e) p1[e] = ex2(r1[e] - n1);
    }
    l0 = l0 * al0 + ((p0[0] + p0[1]) + (p0[2] + p0[3]));
    l1 = l1 * al1 + ((p1[0] + p1[1]) + (p1[2] + p1[3]));
    m0 = n0;
    m1 = n1;
    if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
      for (int j = 0; j < NBW; ++j) {
        o[j][0] *= al0;
        o[j][1] *= al0;
        o[j][2] *= al1;
        o[j][3] *= al1;
      }
    }
    // P as A fragments: rows g / g + 8 x tokens tq.. (k 0-7) and 8+tq.. (k 8-15)
    uint32_t h0, l0p, h1, l1p, h2, l2p, h3, l3p;
    split_bf16(p0[0], p0[1], h0, l0p);  // row g, tokens tq, tq+1
    split_bf16(p1[0], p1[1], h1, l1p);  // row g+8
    split_bf16(p0[2], p0[3], h2, l2p);  // row g, tokens 8+tq, 9+tq
    split_bf16(p1[2], p1[3], h3, l3p);  // row g+8
    // ---- O += P V over this warp's channels (V = first 512 channels of the row)
    {
      const int tok = (mi & 1) * 8 + mr;
      const uint32_t va = smem_addr(S + tok * kRB);
      const int cb = cpart * (CPW / 8);
#pragma unroll
      for (int j = 0; j < NBW; j += 2) {
        uint32_t w0, w1, w2, w3;
        ldsm_x4_t(va + (swz(cb + j + (mi >> 1), tok) << 4), w0, w1, w2, w3);
        mma16(o[j], h0, h1, h2, h3, w0, w1);
        mma16(o[j], l0p, l1p, l2p, l3p, w0, w1);
        mma16(o[j + 1], h0, h1, h2, h3, w2, w3);
        mma16(o[j + 1], l0p, l1p, l2p, l3p, w2, w3);
      }
    }
    __syncthreads();  // every warp is done with stage st before it is refilled
    if (++tile_in_unit == p.tiles_per_group) {
      tile_in_unit = 0;
      ++unit;
    }
    if (++st == kNS) st = 0;
  }
  flush(cur_unit);
  cp_async_wait<0>();
}

template <int HT>
cudaError_t run_mla(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_mla_kernel<HT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  return launch_pdl(attn_mla_kernel<HT>, dim3(p.grid), dim3(kThreads), kSmem, st, a, p);
}

}  // namespace

bool attn_mla_supported(const AttnArgs &a) {
  const int G = a.n_q_heads / a.n_kv_heads;
  return a.v_is_k_prefix && a.dtype == 1 && a.d_qk == kD && a.d_v == kDV && !a.paged &&
         (G == 16 || G == 32 || G == 64);
}

cudaError_t launch_attention_mla(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  switch (p.head_chunk) {
    case 16: return run_mla<1>(a, p, st);
    case 32: return run_mla<2>(a, p, st);
    case 64: return run_mla<4>(a, p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tls
