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

// ---------------------------------------------------------------- programmatic dependent launch
// Kernels are launched with programmatic stream serialization, so a kernel may
// be scheduled while the previous one in the stream finishes.  Every kernel
// calls this before its first global-memory access: it returns once the
// previous grid has completed and its writes are visible (a no-op when the
// launch had no programmatic dependency).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------- mbarriers and bulk copies
__device__ __forceinline__ uint32_t smem_addr(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void mbarrier_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbarrier_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ bool mbarrier_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      " .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of the given parity; false when it gave up (after
// about a second), so that no kernel can spin forever.
__device__ __forceinline__ bool mbarrier_wait(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < (1u << 24); ++i) {
    if (mbarrier_try_wait(bar, parity)) return true;
    if (i > 32) __nanosleep(64);
  }
  return false;
}

__device__ __forceinline__ void mbarrier_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbarrier_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

// Contiguous global -> shared copy by the TMA engine (16-byte aligned, size a
// multiple of 16), completing its bytes on the mbarrier.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
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
//
// Selection of the k largest keys among keys[0..n) held in shared memory
// (key 0 = invalid, never selected; requires 1 <= k <= number of keys > 0),
// ties to the lower index, output ids ascending.  Steps:
//   1. histogram of the top 11 key bits (2048 bins), usually fused into the
//      pass that produces the keys (hist_add);
//   2. the bin b1 holding the k-th largest key, by a block scan over the bins
//      taken from the top;
//   3. the keys of bin b1 are gathered into a short list;
//   4. two more radix passes (11 then 10 bits) over that list only give the
//      exact k-th key thr and how many keys equal to thr are kept;
//   5. an index-ordered compaction: warp w owns a contiguous run of indices
//      (lane-striped, conflict-free), ranks come from ballots and one block
//      scan over the warp totals.
struct SelectResult {
  uint32_t thr;  // the k-th largest key
  int take_eq;   // how many keys equal to thr are kept (the lowest-indexed ones)
};

constexpr int kHistBins = 2048;

struct SelectSmem {
  int hist[kHistBins];
  int sh[33];
  int bc[4];
};

// Adds one key's top-11-bit digit to the histogram (`valid` false contributes
// nothing).  Plain shared-memory atomics: 11-bit digits of score keys are
// spread, so lanes rarely collide on one bin.
__device__ __forceinline__ void hist_add(int *hist, uint32_t key, bool valid) {
  if (valid) atomicAdd(&hist[key >> 21], 1);
}

template <int NT>
__device__ __forceinline__ void hist_clear(int *hist) {
  for (int i = threadIdx.x; i < kHistBins; i += NT) hist[i] = 0;
}

// Over bins [0, nbins): the bin holding the krem-th largest element, and the
// number of elements in higher bins.  Thread t owns nbins/NT consecutive bins
// counted from the top.  Result in bc[0] (bin), bc[1] (count above).
template <int NT>
__device__ __forceinline__ void find_bin_from_top(const int *hist, int nbins, int krem, SelectSmem &S) {
  const int per = nbins / NT;  // nbins is a multiple of NT
  const int top = nbins - threadIdx.x * per;  // owns bins [top - per, top)
  int sum = 0;
  for (int i = 1; i <= per; ++i) sum += hist[top - i];
  int tot;
  const int above = block_excl_scan<NT>(sum, S.sh, tot);
  if (above < krem && krem <= above + sum) {
    int acc = above;
    for (int i = 1; i <= per; ++i) {
      const int c = hist[top - i];
      if (acc + c >= krem) {
        S.bc[0] = top - i;
        S.bc[1] = acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
}

// Steps 2-4.  hist must hold the step-1 histogram of keys[0..n).  list needs n
// entries of shared memory.  Contains __syncthreads(); call uniformly.
template <int NT>
__device__ SelectResult select_kth(const uint32_t *keys, int n, int k, uint32_t *list, SelectSmem &S) {
  static_assert(kHistBins % NT == 0 || NT > kHistBins, "bins split evenly over threads");
  __syncthreads();  // histogram complete
  find_bin_from_top<NT>(S.hist, kHistBins, k, S);
  const uint32_t b1 = static_cast<uint32_t>(S.bc[0]);
  int krem = k - S.bc[1];
  // gather the keys of bin b1
  if (threadIdx.x == 0) S.bc[2] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  for (int base = 0; base < n; base += NT) {
    const int i = base + threadIdx.x;
    const uint32_t key = i < n ? keys[i] : 0u;
    const bool in = i < n && key != 0u && (key >> 21) == b1;
    const unsigned mask = __ballot_sync(0xffffffffu, in);
    int slot = 0;
    if (lane == 0 && mask) slot = atomicAdd(&S.bc[2], __popc(mask));
    slot = __shfl_sync(0xffffffffu, slot, 0);
    if (in) list[slot + __popc(mask & ((1u << lane) - 1u))] = key;
  }
  __syncthreads();
  const int m = S.bc[2];
  // bits 20..10 over the list
  hist_clear<NT>(S.hist);
  __syncthreads();
  for (int i = threadIdx.x; i < m; i += NT) atomicAdd(&S.hist[(list[i] >> 10) & 2047u], 1);
  __syncthreads();
  find_bin_from_top<NT>(S.hist, kHistBins, krem, S);
  const uint32_t b2 = static_cast<uint32_t>(S.bc[0]);
  krem -= S.bc[1];
  // bits 9..0 over the list entries of bin b2
  hist_clear<NT>(S.hist);
  __syncthreads();
  for (int i = threadIdx.x; i < m; i += NT) {
    const uint32_t key = list[i];
    if (((key >> 10) & 2047u) == b2) atomicAdd(&S.hist[key & 1023u], 1);
  }
  __syncthreads();
  find_bin_from_top<NT>(S.hist, 1024 < NT ? NT : 1024, krem, S);
  const uint32_t b3 = static_cast<uint32_t>(S.bc[0]);
  krem -= S.bc[1];
  return {(b1 << 21) | (b2 << 10) | b3, krem};
}

// Step 5: ids of the kept keys (key > thr, or key == thr among the first
// take_eq such keys in index order) in ascending index order to out[0..k), -1
// to out[k..cap).  id_of(i) maps a key position to the id written.  Warp w owns
// the contiguous index run [w*seg, (w+1)*seg), read lane-striped; ranks come
// from ballots and two block scans over the warp totals.
template <int NT, typename IdOf>
__device__ void ordered_compact(const uint32_t *keys, int n, SelectResult r, int k, int32_t *out, int cap,
                                IdOf id_of, SelectSmem &S) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int seg = ((n + NW - 1) / NW + 31) & ~31;  // indices per warp, a multiple of 32
  const int i0 = wid * seg, i1 = min(i0 + seg, n);
  const unsigned lt = (1u << lane) - 1u;
  int n_gt = 0, n_eq = 0;
#pragma unroll 1
  for (int base = i0; base < i0 + seg; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < i1 ? keys[i] : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, key > r.thr));
    n_eq += __popc(__ballot_sync(0xffffffffu, i < i1 && key == r.thr));
  }
  int tot;
  const int eq_base = __shfl_sync(0xffffffffu, block_excl_scan<NT>(lane == 0 ? n_eq : 0, S.sh, tot), 0);
  const int eq_kept = max(0, min(n_eq, r.take_eq - eq_base));
  int pos = __shfl_sync(0xffffffffu, block_excl_scan<NT>(lane == 0 ? (n_gt + eq_kept) : 0, S.sh, tot), 0);
  int eq_seen = eq_base;
#pragma unroll 1
  for (int base = i0; base < i0 + seg; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < i1 ? keys[i] : 0u;
    const unsigned gtm = __ballot_sync(0xffffffffu, key > r.thr);
    const unsigned eqm = __ballot_sync(0xffffffffu, i < i1 && key == r.thr);
    // equal keys of this run that are still within take_eq (lowest lanes first)
    const int room = max(0, r.take_eq - eq_seen);
    unsigned keep_eq = eqm;
    if (__popc(eqm) > room) {
      keep_eq = 0;
      unsigned rest = eqm;
      for (int c = 0; c < room; ++c) {
        keep_eq |= rest & (~rest + 1u);  // lowest set bit
        rest &= rest - 1u;
      }
    }
    eq_seen += __popc(eqm);
    const unsigned selm = gtm | keep_eq;
    if ((selm >> lane) & 1u) {
      const int p = pos + __popc(selm & lt);
      if (p < k) out[p] = id_of(i);  // p < k always holds; the guard keeps writes in bounds
    }
    pos += __popc(selm);
  }
  for (int i = k + threadIdx.x; i < cap; i += NT) out[i] = -1;
}

}  // namespace tls
