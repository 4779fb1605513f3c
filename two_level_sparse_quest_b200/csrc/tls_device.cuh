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
struct I8 {  // int8 codes of the quantised label slab
  using storage = int8_t;
  static constexpr int kBytes = 1;
  static constexpr int kEPC = 16;
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
template <>
__device__ __forceinline__ void chunk_to_f32<I8>(const uint4 &c, float *f) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k) f[4 * i + k] = static_cast<float>(static_cast<int32_t>(w[i] << (24 - 8 * k)) >> 24);
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

// ---------------------------------------------------------------- thread-block clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Split cluster barrier: every thread of every CTA of the cluster arrives once
// and waits once.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t local_smem_addr, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(local_smem_addr), "r"(rank));
  return a;
}
// Asynchronous store into (possibly another CTA's) shared memory that counts
// its bytes on that CTA's mbarrier (complete_tx).
__device__ __forceinline__ void st_async_v4(uint32_t cluster_addr, uint4 v, uint32_t cluster_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   cluster_addr),
               "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(cluster_bar)
               : "memory");
}
__device__ __forceinline__ void st_async_b32(uint32_t cluster_addr, uint32_t v, uint32_t cluster_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(cluster_addr), "r"(v),
               "r"(cluster_bar)
               : "memory");
}
__device__ __forceinline__ void mbarrier_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}
// Bounded wait (cluster-scope acquire: the awaited bytes were written by other
// CTAs); false when it gave up after about a second.
__device__ __forceinline__ bool mbarrier_wait_cluster(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < (1u << 24); ++i) {
    uint32_t ok;
    asm volatile(
        "{\n"
        " .reg .pred p;\n"
        " mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
    if (i > 32) __nanosleep(32);
  }
  return false;
}

// Bits of the library's device error word (set by kernels whose bounded wait
// gave up; read by tls_device_error).
constexpr int kErrAttnWait = 1;
constexpr int kErrSelectWait = 2;
constexpr int kErrAppendRange = 4;  // an appended range outside [0, max_ctx] or longer than max_append

// ---------------------------------------------------------------- cluster top-k
//
// Selection of the k largest of a group's keys (key 0 = invalid, never
// selected), ties to the lower index, output ids ascending.  The keys are
// spread over the CS CTAs of one thread-block cluster: CTA r holds the r-th
// contiguous slice of the index space in its own shared memory.  Steps:
//   1. each CTA builds a 256-bin histogram of the top key byte over its slice
//      while it produces the keys (hist_add);
//   2. four radix passes of 8 bits (bits 31..24, 23..16, 15..8, 7..0): warp 0
//      of every CTA packs its histogram as 16-bit counts and sends it with
//      asynchronous stores into a per-pass inbox of every CTA of the cluster,
//      counting the bytes on that CTA's per-pass mbarrier; once its own
//      mbarrier has all CS histograms, warp 0 sums them and finds the digit of
//      the k-th largest key (every CTA finds the same one); the next pass
//      histograms only the keys that share the digits found so far.  After
//      pass 4 the k-th key thr is exact, and take_eq says how many keys equal
//      to thr are kept (the lowest-indexed ones);
//   3. an index-ordered compaction: inside a CTA, warp w owns a contiguous run
//      of indices read lane-striped; one pass records ballot masks (lane j
//      keeps those of steps j, j+32, ...), a block scan of packed
//      (equal << 16 | greater) counts ranks the steps, every CTA sends its
//      packed total to every CTA (one more mbarrier), and the sum over lower
//      ranks is the CTA's offset; a second pass writes the ids.
// A CTA only waits for bytes addressed to it, so no CTA exits while a store to
// its shared memory is outstanding; the one cluster barrier (entry arrive,
// wait before the first send) makes every CTA's mbarriers initialised before
// anyone sends.  Counts fit 16 bits: a group has at most kSelectCapacity keys.
constexpr int kCBins = 256;
constexpr int kSelectCapacity = 16384;

template <int CS>
struct ClusterSelectSmem {
  int hist[kCBins];           // this CTA's histogram of the current digit
  uint4 inbox[4][CS][32];     // per pass, per source CTA: lane l's 8 bins (top-down) as 16-bit counts
  int counts[CS];             // packed (equal << 16 | greater) totals sent by each CTA
  uint64_t bar[5];            // passes 0..3, counts
  int sh[33];
  int bc[4];
};

// At kernel entry, before anything else touches S: the mbarriers are armed for
// the bytes every pass will receive; then the entry cluster arrive.
template <int CS>
__device__ __forceinline__ void cluster_topk_arm(ClusterSelectSmem<CS> &S) {
  if (threadIdx.x == 0) {
#pragma unroll
    for (int i = 0; i < 5; ++i) mbarrier_init(&S.bar[i], 1);
    mbarrier_init_fence();
#pragma unroll
    for (int i = 0; i < 4; ++i) mbarrier_arrive_expect_tx(&S.bar[i], CS * 32 * 16);
    mbarrier_arrive_expect_tx(&S.bar[4], CS * 4);
  }
}
template <int CS>
__device__ __forceinline__ void cluster_topk_begin(ClusterSelectSmem<CS> &S) {
  cluster_topk_arm(S);
  cluster_arrive_relaxed();
}

// Adds one valid key's top byte to the histogram.
__device__ __forceinline__ void hist_add(int *hist, uint32_t key, bool valid) {
  if (valid) atomicAdd(&hist[key >> 24], 1);
}

struct SelectResult {
  uint32_t thr;  // the k-th largest key
  int take_eq;   // how many keys equal to thr are kept (the lowest-indexed ones)
};

// Step 3 inside one CTA.  keys[0..n), n <= CAP.  cta_base(total) receives the
// CTA's packed (equal << 16 | greater) total and returns the packed total of
// all lower-indexed keys of the group held elsewhere (0 for a lone CTA).
// Writes out[p] = id_of(i) for the kept keys at their group-wide ranks p < k.
template <int NT, int CAP, typename IdOf, typename BaseFn>
__device__ void ordered_compact(const uint32_t *keys, int n, SelectResult r, int k, int32_t *out, IdOf id_of,
                                int *sh, BaseFn cta_base) {
  constexpr int NW = NT / 32;
  constexpr int R = (CAP + NW * 1024 - 1) / (NW * 1024);  // mask slots per lane
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int seg = ((n + NW - 1) / NW + 31) & ~31;  // indices per warp, a multiple of 32
  const int iters = min(seg >> 5, 32 * R);         // seg >> 5 <= 32 * R when n <= CAP
  const int i0 = wid * seg, i1 = min(i0 + seg, n);
  unsigned gt[R], eq[R];
#pragma unroll
  for (int s = 0; s < R; ++s) gt[s] = eq[s] = 0u;
#pragma unroll 4
  for (int it = 0; it < iters; ++it) {
    const int i = i0 + it * 32 + lane;
    const uint32_t key = i < i1 ? keys[i] : 0u;
    const unsigned g = __ballot_sync(0xffffffffu, key > r.thr);
    const unsigned e = __ballot_sync(0xffffffffu, i < i1 && key == r.thr);
    if ((it & 31) == lane) {
#pragma unroll
      for (int s = 0; s < R; ++s)
        if ((it >> 5) == s) {
          gt[s] = g;
          eq[s] = e;
        }
    }
  }
  int pre[R];
  int run = 0;
#pragma unroll
  for (int s = 0; s < R; ++s) {
    const int pc = (__popc(eq[s]) << 16) | __popc(gt[s]);
    const int incl = warp_incl_scan(pc);
    pre[s] = run + incl - pc;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  int total;
  const int wexcl = __shfl_sync(0xffffffffu, block_excl_scan<NT>(lane == 0 ? run : 0, sh, total), 0);
  const int wbase = wexcl + cta_base(total);
  unsigned sel[R];
  int pos[R];
#pragma unroll
  for (int s = 0; s < R; ++s) {
    const int before = wbase + pre[s];
    const int gt_before = before & 0xffff, eq_before = before >> 16;
    const int room = r.take_eq - eq_before;  // equal keys still to keep at this step
    unsigned keep = eq[s];
    if (__popc(keep) > room) {
      keep = 0u;
      unsigned rest = eq[s];
      for (int c = 0; c < room; ++c) {
        keep |= rest & (~rest + 1u);  // lowest set bit
        rest &= rest - 1u;
      }
    }
    sel[s] = gt[s] | keep;
    pos[s] = gt_before + min(r.take_eq, eq_before);
  }
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll 4
  for (int it = 0; it < iters; ++it) {
    unsigned vs = sel[0];
    int vp = pos[0];
#pragma unroll
    for (int s = 1; s < R; ++s)
      if ((it >> 5) == s) {
        vs = sel[s];
        vp = pos[s];
      }
    const unsigned selm = __shfl_sync(0xffffffffu, vs, it & 31);
    const int p0 = __shfl_sync(0xffffffffu, vp, it & 31);
    if ((selm >> lane) & 1u) {
      const int p = p0 + __popc(selm & lt);
      if (p < k) out[p] = id_of(i0 + it * 32 + lane);  // p < k always holds; the guard keeps writes in bounds
    }
  }
}

// The same selection by one CTA over keys[0..n) in its own shared memory
// (n <= CAP): four radix passes of 8 bits over a shared-memory histogram, then
// the index-ordered compaction into out[0..k) (ascending ids; the caller pads).
// Returns k (the wanted count clamped to the valid keys).  Every thread of the
// CTA calls it; hist must hold kCBins ints, bc 4 ints, sh 33 ints.
template <int NT, int CAP, typename IdOf>
__device__ int cta_topk(const uint32_t *keys, int n, int k_req, int32_t *out, IdOf id_of, int *hist, int *bc,
                        int *sh) {
  static_assert(NT >= kCBins && NT % 32 == 0, "one histogram bin per thread");
  const int tid = threadIdx.x, lane = tid & 31;
  uint32_t prefix = 0;
  int krem = 0, k = 0;
  __syncthreads();  // the keys are complete and nothing still adds to hist
#pragma unroll 1
  for (int p = 0; p < 4; ++p) {
    const int shift = 24 - 8 * p;
    if (tid < kCBins) hist[tid] = 0;
    __syncthreads();  // the previous pass's decision is read
    const uint32_t want = p == 0 ? 0u : prefix >> (shift + 8);
    for (int i = tid; i < n; i += NT) {
      const uint32_t key = keys[i];
      if (key != 0u && (p == 0 || (key >> (shift + 8)) == want)) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid < 32) {  // lane l owns bins 255-8l .. 248-8l, from the top
      const int top = kCBins - 1 - 8 * lane;
      int cnt[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = hist[top - j];
        sum += cnt[j];
      }
      const int incl = warp_incl_scan(sum);
      int kr = krem;
      if (p == 0) kr = min(k_req, __shfl_sync(0xffffffffu, incl, 31));  // valid keys
      int acc = incl - sum;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (acc < kr && acc + cnt[j] >= kr) {  // exactly one (lane, bin) satisfies this
          bc[0] = top - j;
          bc[1] = acc;
          bc[3] = cnt[j];
        }
        acc += cnt[j];
      }
      if (p == 0 && lane == 0) bc[2] = kr;
    }
    __syncthreads();
    if (p == 0) {
      k = bc[2];
      krem = k;
      if (k <= 0) break;  // no valid key
    }
    krem -= bc[1];
    prefix |= static_cast<uint32_t>(bc[0]) << shift;
    if (krem == bc[3] && prefix != 0u) {  // exact fit: every key of the bin is kept
      prefix -= 1u;
      krem = 0;
      break;
    }
  }
  if (k > 0)
    ordered_compact<NT, CAP>(keys, n, SelectResult{prefix, krem}, k, out, id_of, sh, [](int) { return 0; });
  __syncthreads();
  return k;
}

// The whole selection for one cluster (steps 2-3; step 1 done by the caller
// into S.hist).  keys[0..n): this CTA's slice, n <= CAP; k_req: wanted count
// (clamped to the number of valid keys of the group); out[0..cap): ids in
// ascending order, -1 padded (cap >= k_req).  Every thread of every CTA of the
// cluster calls it once per ClusterSelectSmem, after cluster_topk_begin() on
// that smem at kernel entry; entry_wait = false for a later selection whose
// mbarriers were armed before an earlier call's entry wait.  A wait
// that gives up sets kErrSelectWait in *err (the results are then undefined;
// the kernel still ends).
template <int NT, int CS, int CAP, typename IdOf>
__device__ void cluster_topk(const uint32_t *keys, int n, int k_req, int32_t *out, int cap, IdOf id_of,
                             ClusterSelectSmem<CS> &S, int *err, bool entry_wait = true) {
  static_assert(NT >= kCBins && NT % 32 == 0, "one histogram bin per thread");
  static_assert(CS * CAP <= kSelectCapacity, "16-bit bin counts");
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  __syncthreads();  // this CTA's keys and histogram are complete
  if (entry_wait) cluster_wait();  // every CTA of the cluster has armed its mbarriers
  uint32_t prefix = 0;
  int krem = k_req, k = 0;
  bool ok = true;
#pragma unroll 1
  for (int p = 0; p < 4; ++p) {
    const int shift = 24 - 8 * p;
    if (tid < 32) {  // warp 0: lane l owns bins 255-8l .. 248-8l, from the top
      const int top = kCBins - 1 - 8 * lane;
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        w[j] = static_cast<uint32_t>(S.hist[top - 2 * j]) | (static_cast<uint32_t>(S.hist[top - 2 * j - 1]) << 16);
#pragma unroll
      for (int j = 0; j < 8; ++j) S.hist[top - j] = 0;  // cleared for the next digit
      const uint32_t la = smem_addr(&S.inbox[p][rank][lane]);
      const uint32_t lb = smem_addr(&S.bar[p]);
      const uint4 v = make_uint4(w[0], w[1], w[2], w[3]);
#pragma unroll
      for (int c = 0; c < CS; ++c) st_async_v4(cluster_map(la, c), v, cluster_map(lb, c));
      ok = mbarrier_wait_cluster(&S.bar[p], 0) && ok;
      uint32_t sm[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int c = 0; c < CS; ++c) {
        const uint4 x = S.inbox[p][c][lane];
        sm[0] += x.x;
        sm[1] += x.y;
        sm[2] += x.z;
        sm[3] += x.w;
      }
      int cnt[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        cnt[2 * j] = static_cast<int>(sm[j] & 0xffffu);
        cnt[2 * j + 1] = static_cast<int>(sm[j] >> 16);
        sum += cnt[2 * j] + cnt[2 * j + 1];
      }
      const int incl = warp_incl_scan(sum);
      if (p == 0) krem = min(k_req, __shfl_sync(0xffffffffu, incl, 31));  // valid keys of the group
      int acc = incl - sum;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (acc < krem && acc + cnt[i] >= krem) {  // exactly one (lane, bin) satisfies this
          S.bc[0] = top - i;
          S.bc[1] = acc;
          S.bc[3] = cnt[i];
        }
        acc += cnt[i];
      }
      if (p == 0 && lane == 0) S.bc[2] = krem;
    }
    __syncthreads();
    if (p == 0) {
      k = S.bc[2];
      krem = k;
      if (k <= 0) break;  // the group has no valid key: same decision in every CTA
    }
    const uint32_t digit = static_cast<uint32_t>(S.bc[0]);
    krem -= S.bc[1];
    prefix |= digit << shift;
    // Exact fit: the bin holds exactly the keys still wanted, so every key at
    // or above the bin's lowest key is kept and no further digit is needed
    // (thr = that key - 1, no equal keys taken).  Same decision in every CTA.
    if (krem == S.bc[3] && prefix != 0u) {
      prefix -= 1u;
      krem = 0;
      break;
    }
    if (p < 3) {  // next digit over this CTA's keys that share the digits found so far
      const uint32_t want = prefix >> shift;
      const int nshift = shift - 8;
      constexpr int U = 8;
      for (int base = 0; base < n; base += NT * U) {
        uint32_t kv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int i = base + u * NT + tid;
          kv[u] = i < n ? keys[i] : 0u;
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (kv[u] != 0u && (kv[u] >> shift) == want) atomicAdd(&S.hist[(kv[u] >> nshift) & 255u], 1);
      }
      __syncthreads();
    }
  }
  if (k > 0) {
    ordered_compact<NT, CAP>(keys, n, SelectResult{prefix, krem}, k, out, id_of, S.sh, [&](int total) {
      if (tid < CS)
        st_async_b32(cluster_map(smem_addr(&S.counts[rank]), tid), static_cast<uint32_t>(total),
                     cluster_map(smem_addr(&S.bar[4]), tid));
      ok = mbarrier_wait_cluster(&S.bar[4], 0) && ok;
      int base = 0;
      for (uint32_t c = 0; c < rank; ++c) base += S.counts[c];
      return base;
    });
  }
  if (rank == 0)
    for (int i = max(k, 0) + tid; i < cap; i += NT) out[i] = -1;
  if (!ok && err) atomicOr(err, kErrSelectWait);
}

}  // namespace tls
