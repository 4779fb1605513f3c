// tls_device.cuh -- device helpers shared by the libtls kernels (sm_100a).
//
// Element access for fp32 / bf16 storage, order-preserving score keys,
// cp.async staging, warp / block reductions and scans, and the block-wide
// radix select + index-ordered compaction used by both selection stages.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tls {

// ---------------------------------------------------------------- element types
// Storage tags.  kEPC = elements per 16-byte chunk.
struct F32 {
  using storage = float;
  static constexpr int kBytes = 4;
  static constexpr int kEPC = 4;
};
struct BF16 {
  using storage = uint16_t;
  static constexpr int kBytes = 2;
  static constexpr int kEPC = 8;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// One 16-byte chunk -> kEPC floats (exact widening).
template <typename E>
__device__ __forceinline__ void chunk_to_f32(const uint4 &c, float *f);
template <>
__device__ __forceinline__ void chunk_to_f32<F32>(const uint4 &c, float *f) {
  f[0] = __uint_as_float(c.x);
  f[1] = __uint_as_float(c.y);
  f[2] = __uint_as_float(c.z);
  f[3] = __uint_as_float(c.w);
}
template <>
__device__ __forceinline__ void chunk_to_f32<BF16>(const uint4 &c, float *f) {
  f[0] = bf16_lo(c.x); f[1] = bf16_hi(c.x);
  f[2] = bf16_lo(c.y); f[3] = bf16_hi(c.y);
  f[4] = bf16_lo(c.z); f[5] = bf16_hi(c.z);
  f[6] = bf16_lo(c.w); f[7] = bf16_hi(c.w);
}

template <typename E>
__device__ __forceinline__ float load_elem(const void *base, size_t i);
template <>
__device__ __forceinline__ float load_elem<F32>(const void *base, size_t i) {
  return static_cast<const float *>(base)[i];
}
template <>
__device__ __forceinline__ float load_elem<BF16>(const void *base, size_t i) {
  return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t *>(base)[i]) << 16);
}

// fp32 -> bf16 bits, round to nearest even (inputs are finite here).
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7fffu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

// Streaming 16-byte global load that bypasses L1 allocation.
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Packed fp32x2 FMA (sm_100+): d = a * b + d, two lanes at once.
__device__ __forceinline__ void ffma2(float2 &d, const float2 a, const float2 b) {
  unsigned long long dd, aa, bb;
  aa = *reinterpret_cast<const unsigned long long *>(&a);
  bb = *reinterpret_cast<const unsigned long long *>(&b);
  dd = *reinterpret_cast<unsigned long long *>(&d);
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(dd) : "l"(aa), "l"(bb));
  d = *reinterpret_cast<float2 *>(&dd);
}

// ---------------------------------------------------------------- score keys
// Order-preserving map fp32 -> uint32 (larger float -> larger key).  -0 is
// folded onto +0 so that equal scores give equal keys.  Key 0 is below every
// non-NaN float and marks an invalid candidate.
__device__ __forceinline__ uint32_t score_key(float f) {
  f += 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- cp.async
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool pred) {
  unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  int n = pred ? 16 : 0;  // 0 source bytes -> the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- warp / block collectives
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// Exclusive prefix sum over the whole thread block (NT threads, NT % 32 == 0).
// `sh` needs 33 ints of shared memory.  Returns the exclusive prefix; `total`
// receives the block total.  Contains __syncthreads(); call uniformly.
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int *sh, int &total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = warp_incl_scan(v);
  if (lane == 31) sh[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int w = (lane < NW) ? sh[lane] : 0;
    w = warp_incl_scan(w);
    if (lane < NW) sh[lane] = w;
  }
  __syncthreads();
  const int base = wid ? sh[wid - 1] : 0;
  total = sh[NW - 1];
  __syncthreads();
  return base + incl - v;
}

// ---------------------------------------------------------------- top-k select
struct SelectResult {
  uint32_t thr;  // the k-th largest key
  int take_eq;   // how many keys equal to thr are kept (the lowest-indexed ones)
};

// Block-wide radix select (8-bit digits, most significant first) of the k-th
// largest key among keys[0..n).  Requires 1 <= k <= (number of keys > 0).
// `hist` needs 256 ints and `bc` 2 ints of shared memory.  Histogram updates are
// aggregated per warp with match.any so that many equal digits do not
// serialise on one shared-memory address.
template <int NT>
__device__ SelectResult block_radix_select(const uint32_t *keys, int n, int k, int *hist, int *bc) {
  uint32_t prefix = 0, mask = 0;
  int krem = k;
  const int tid = threadIdx.x, lane = tid & 31;
  const int iters = (n + NT - 1) / NT;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
#pragma unroll 1
    for (int it = 0; it < iters; ++it) {
      const int i = it * NT + tid;
      const uint32_t key = (i < n) ? keys[i] : 0u;
      const bool match = (i < n) && ((key & mask) == prefix);
      const int digit = match ? static_cast<int>((key >> shift) & 255u) : 256;
      const unsigned peers = __match_any_sync(0xffffffffu, digit);
      if (match && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
    }
    __syncthreads();
    if (tid < 32) {
      int c[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[lane * 8 + j];
        tot += c[j];
      }
      int suf = tot;  // keys in bins owned by lanes >= lane
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += t;
      }
      const int above = suf - tot;
      const unsigned own = __ballot_sync(0xffffffffu, above < krem && krem <= suf);
      if (lane == __ffs(own) - 1) {
        int acc = above, dsel = lane * 8;
        for (int j = 7; j >= 0; --j) {
          if (acc + c[j] >= krem) { dsel = lane * 8 + j; break; }
          acc += c[j];
        }
        bc[0] = dsel;
        bc[1] = acc;
      }
    }
    __syncthreads();
    const int dsel = bc[0];
    krem -= bc[1];
    prefix |= static_cast<uint32_t>(dsel) << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  return {prefix, krem};
}

// Writes the ids of the selected keys (key > thr, or key == thr among the first
// take_eq such keys in index order) in ascending index order to out[0..k) and
// -1 to out[k..cap).  id_of(i) maps a key position to the id written.
// `sh` needs 33 ints of shared memory.
template <int NT, typename IdOf>
__device__ void block_ordered_compact(const uint32_t *keys, int n, SelectResult r, int k, int32_t *out, int cap,
                                      IdOf id_of, int *sh) {
  const int tid = threadIdx.x;
  const int E = (n + NT - 1) / NT;
  const int i0 = min(tid * E, n), i1 = min(i0 + E, n);
  int n_eq = 0;
  for (int i = i0; i < i1; ++i) n_eq += (keys[i] == r.thr);
  int tot;
  const int eq_before = block_excl_scan<NT>(n_eq, sh, tot);
  int n_sel = 0, eq_rank = eq_before;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = keys[i];
    if (key > r.thr) ++n_sel;
    else if (key == r.thr) { n_sel += (eq_rank < r.take_eq); ++eq_rank; }
  }
  int pos = block_excl_scan<NT>(n_sel, sh, tot);
  eq_rank = eq_before;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = keys[i];
    bool sel = key > r.thr;
    if (key == r.thr) { sel = eq_rank < r.take_eq; ++eq_rank; }
    if (sel && pos < k) out[pos++] = id_of(i);  // pos < k always holds; the guard keeps writes in bounds
  }
  for (int i = k + tid; i < cap; i += NT) out[i] = -1;
}

}  // namespace tls
