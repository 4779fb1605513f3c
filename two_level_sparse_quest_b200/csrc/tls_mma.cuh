// tls_mma.cuh -- warp-level tensor-core helpers shared by the bf16 attention
// kernels (tls_attn_mma.cu and the fused decode step in tls_step.cu): the
// per-warp gather ring layout, ldmatrix / mma.sync wrappers and the bf16
// hi + lo split of the softmax weights.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "tls_device.cuh"

namespace tls {

static constexpr int kMT = 16;  // tokens per tile
static constexpr int kMmaStages = 3;

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

static __device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

static __device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
static __device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// c[0..1] += A B for the rows of this lane (row lane/4); the A rows lane/4 + 8
// are zero (a1 = a3 = 0) and the matching accumulator halves are discarded.
static __device__ __forceinline__ void mma_rows(float (&c)[2], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  float d2, d3;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %10, %11};"
      : "+f"(c[0]), "+f"(c[1]), "=f"(d2), "=f"(d3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(0.f), "f"(0.f));
}

// c[0..3] += A B over all 16 rows (rows lane/4 and lane/4 + 8).
static __device__ __forceinline__ void mma_full(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// R = 1: rows lane/4 only (A fragment {a0, a2}); R = 2: both row halves
// (A fragment {a0, a1, a2, a3}); c holds 2 R accumulators.
template <int R>
static __device__ __forceinline__ void mma_r(float (&c)[2 * R], const uint32_t (&a)[2 * R], uint32_t b0, uint32_t b1) {
  if constexpr (R == 1) mma_rows(c, a[0], a[1], b0, b1);
  else mma_full(c, a[0], a[1], a[2], a[3], b0, b1);
}

static __device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}
// x = bf16 hi part + bf16 lo part (the lo part holds the rounding error of hi)
static __device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t &hi, uint32_t &lo) {
  hi = pack_bf16(x0, x1);
  lo = pack_bf16(x0 - bf16_lo(hi), x1 - bf16_hi(hi));
}

}  // namespace tls
