// tls_score_tc.cu -- the max-over-heads block score on the 5th-generation
// tensor cores (tcgen05.mma, operands in shared memory, accumulator in TMEM).
//
// Stage 1 with block_agg = 1 (the variant of gist.science (de) section 2.A
// "Stufe 1" / "Optimierung"; (es) section 2.A.1): every head h of a group
// bounds block j by u_{h,j} = q_h^+ . max_j + q_h^- . min_j, and the block's
// score is the largest of the G bounds.  Unlike the sum over heads (which
// folds into one query vector), the G bounds are a real contraction:
//   U[blocks x G] = [max_j ; min_j]  .  [q_h^+ ; q_h^-]^T      (K = 2 d)
// One CTA (one warpgroup; two per SM for d <= 128) walks a contiguous range of
// (group, 128-block tile) work items:
//   A = the tile's 128 summary rows, K-major, staged 64 channels (128 B) at a
//       time into a ring of 128B-swizzled 16 KB regions by 16-byte cp.async;
//   B = [q^+ ; q^-] of the group's heads as bf16 rows (exact: each element is
//       q or 0), rows padded with zeros to N = a multiple of 16, resident in
//       shared memory for the group;
//   D = U in TMEM (128 lanes = the tile's blocks, N fp32 columns); thread t
//       reads block t's row (tcgen05.ld) and writes max_{h < G} to the scores.
// bf16 x bf16 products are exact; the tensor cores accumulate in fp32.
// Every wait is bounded; a wait that gives up sets the attention/selection
// error bit 2 and stops the CTA after freeing its TMEM.
#include <algorithm>

#include "tls_device.cuh"
#include "tls_internal.h"

namespace tls {
namespace {

constexpr int kSThreads = 128;
constexpr int kSTile = 128;                  // blocks per tile (MMA M)
constexpr int kSRegion = kSTile * 128;       // 64 channels of 128 rows: 16 KB
constexpr int kSStages = 4;                  // ring of A regions
constexpr uint32_t kSWait = 1u << 24;

__device__ __forceinline__ bool s_mbar_wait(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < kSWait; ++i) {
    if (mbarrier_try_wait(bar, parity)) return true;
    if (i > 32) __nanosleep(64);
  }
  return false;
}
__device__ __forceinline__ void s_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void s_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void s_fence_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle, K-major (sm_100 format).
__device__ __forceinline__ uint64_t s_desc(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(16 >> 4) << 16;      // leading byte offset (unused for K-major swizzled)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;    // stride byte offset: 8 rows x 128 B
  d |= static_cast<uint64_t>(1) << 46;            // descriptor version
  d |= static_cast<uint64_t>(2) << 61;            // 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16, bf16 x bf16 -> f32, both operands K-major.
constexpr uint32_t s_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void s_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                      uint32_t accumulate) {
  asm volatile(
      "{\n"
      " .reg .pred p;\n"
      " setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void s_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void s_tmem_ld16(uint32_t taddr, float *v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Byte offset of 16-byte chunk c (0-7) of row r inside a 128B-swizzled region.
__device__ __forceinline__ uint32_t s_sw(int r, int c) { return r * 128 + (((c ^ r) & 7) << 4); }

// Shared memory: [ring of kSStages A regions][B: K/64 regions of NP rows x 128 B][mbarriers, TMEM slot].
constexpr int score_tc_smem(int np, int kr) { return kSStages * kSRegion + kr * np * 128 + 256 + 1024 /*align*/; }
static_assert(score_tc_smem(64, 18) <= 227 * 1024, "shared memory budget of the latent shape");

// NP: padded heads (MMA N).  KR: 64-channel regions of K = 2 d.
template <int NP, int KR>
__global__ void __launch_bounds__(kSThreads, 1) block_scores_max_tc_kernel(BlockScoreArgs a, int n_items,
                                                                          int items_per_cta) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem =
      reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char *ring = smem;                                  // [kSStages][16 KB]
  unsigned char *bmat = ring + kSStages * kSRegion;            // [KR][NP rows x 128 B]
  uint64_t *bar = reinterpret_cast<uint64_t *>(bmat + KR * NP * 128);  // [kSStages] MMA of a stage done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + kSStages);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int d = a.d;
  const int RB = 2 * d * 2;  // summary row bytes
  const int G = a.n_q_heads / a.n_kv_heads;
  const int tiles_per_group = (a.n_blocks_max + kSTile - 1) / kSTile;
  // this CTA's work items: a contiguous range, so that consecutive tiles
  // mostly belong to the same group and share its B
  const int item0 = blockIdx.x * items_per_cta;
  const int my_items = max(0, min(items_per_cta, n_items - item0));
  if (my_items == 0) return;

  constexpr uint32_t kCols = NP <= 32 ? 32 : (NP <= 64 ? 64 : (NP <= 128 ? 128 : 256));
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(kCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < kSStages; ++i) mbarrier_init(&bar[i], 1);
    mbarrier_init_fence();
  }
  s_fence_before();
  __syncthreads();
  s_fence_after();
  grid_dependency_wait();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  constexpr uint32_t kIdesc = s_idesc(kSTile, NP);

  // A region r of item it: 128 rows, 16-byte chunks (8 per row) of channels
  // [64 r, 64 r + 64) of K; rows at or beyond the capacity are zero-filled.
  auto issue_region = [&](int step, int st) {
    const int it = step / KR, r = step % KR;
    const int item = item0 + it;
    const int group = item / tiles_per_group, j0 = (item % tiles_per_group) * kSTile;
    const char *base = static_cast<const char *>(a.meta) + (static_cast<size_t>(group) * a.n_blocks_max) * RB;
    unsigned char *dst = ring + st * kSRegion;
#pragma unroll
    for (int i = 0; i < kSTile * 8 / kSThreads; ++i) {
      const int idx = i * kSThreads + tid;
      const int row = idx >> 3, c = idx & 7;
      const int j = j0 + row;
      const bool ok = j < a.n_blocks_max;
      cp_async16(dst + s_sw(row, c), base + static_cast<size_t>(ok ? j : 0) * RB + r * 128 + c * 16, ok);
    }
  };
  // B for a group: row h (< G) = [q_h^+ (d) ; q_h^- (d)] as bf16 (q^+ = max(q, 0),
  // q^- = min(q, 0), taken from the sign bit of each bf16; -0 reads as 0).  The
  // q rows are read as 16-byte chunks of 8 channels, kBLoads chunks in flight
  // per thread; chunk c of row h lands in chunk c % 8 of region c / 8 (q^+)
  // and of region (d / 64) + c / 8 (q^-).  Rows G .. NP-1 stay zero.
  constexpr int kBLoads = 8;
  auto build_b = [&](int group) {
    const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
    const uint4 *q4 = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(a.q) +
                                                      (static_cast<size_t>(b) * a.n_q_heads + g * G) * d);
    const int cpr = d / 8, n = G * cpr, half = d / 64;
    for (int base = 0; base < n; base += kSThreads * kBLoads) {
      uint4 v[kBLoads];
#pragma unroll
      for (int u = 0; u < kBLoads; ++u) {
        const int idx = base + u * kSThreads + tid;
        v[u] = idx < n ? q4[idx] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kBLoads; ++u) {
        const int idx = base + u * kSThreads + tid;
        if (idx < n) {
          const int h = idx / cpr, c = idx % cpr;
          uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w}, pw[4], nw[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t m = ((w[i] >> 15) & 0x00010001u) * 0xFFFFu;  // 0xFFFF in each negative half
            nw[i] = w[i] & m;
            pw[i] = w[i] & ~m;
          }
          *reinterpret_cast<uint4 *>(bmat + (c >> 3) * NP * 128 + s_sw(h, c & 7)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
          *reinterpret_cast<uint4 *>(bmat + (half + (c >> 3)) * NP * 128 + s_sw(h, c & 7)) =
              make_uint4(nw[0], nw[1], nw[2], nw[3]);
        }
      }
    }
  };
  // rows G .. NP-1 of every region: zero for the whole launch
  for (int i = tid; i < KR * NP * 8; i += kSThreads) {
    const int r = i / (NP * 8), h = (i / 8) % NP, c = i % 8;
    if (h >= G) *reinterpret_cast<uint4 *>(bmat + r * NP * 128 + s_sw(h, c)) = make_uint4(0, 0, 0, 0);
  }

  const int n_steps = my_items * KR;
  int cur_group = -1;
  bool failed = false;
  uint32_t phase = 0;        // bit s: parity of the next completion of bar[s]
  bool prev_waited = false;  // the previous step's completion was consumed by its tile epilogue
  // prologue: regions 0 .. kSStages - 2
#pragma unroll
  for (int s = 0; s < kSStages - 1; ++s) {
    if (s < n_steps) issue_region(s, s);
    cp_async_commit();
  }
  for (int step = 0; step < n_steps && !failed; ++step) {
    const int st = step % kSStages;
    const int it = step / KR, r = step % KR;
    const int item = item0 + it;
    const int group = item / tiles_per_group;
    // the stage that region step + kSStages - 1 reuses held region step - 1:
    // its MMA must be complete before the copies overwrite it
    if (step >= 1 && !prev_waited) {
      const int ps = (step - 1) % kSStages;
      if (!s_mbar_wait(&bar[ps], (phase >> ps) & 1u)) failed = true;
      phase ^= 1u << ps;
      s_fence_after();
    }
    prev_waited = false;
    if (r == 0 && group != cur_group) {  // new group: its B (every MMA reading the old B is complete)
      build_b(group);
      cur_group = group;
    }
    const int nxt = step + kSStages - 1;
    if (nxt < n_steps) issue_region(nxt, nxt % kSStages);
    cp_async_commit();
    cp_async_wait<kSStages - 1>();  // region `step` has landed
    s_fence_async();
    failed = __syncthreads_or(failed);
    if (failed) break;
    if (tid == 0) {
      s_fence_after();
      const uint32_t abase = smem_addr(ring + st * kSRegion), bbase = smem_addr(bmat + r * NP * 128);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)  // 4 k-steps of 16 channels (32 bytes) per region
        s_mma(tmem, s_desc(abase + kk * 32), s_desc(bbase + kk * 32), kIdesc, (r > 0 || kk > 0) ? 1u : 0u);
      s_commit(&bar[st]);
    }
    if (r == KR - 1) {  // last region of the tile: wait for its MMAs, then the row maxima
      if (!s_mbar_wait(&bar[st], (phase >> st) & 1u)) failed = true;
      phase ^= 1u << st;
      s_fence_after();
      float best = -INFINITY;
#pragma unroll
      for (int c0 = 0; c0 < NP; c0 += 16) {
        float v[16];
        s_tmem_ld16(tmem + lane_base + c0, v);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (c0 + i < G) best = fmaxf(best, v[i]);
      }
      const int j = (item % tiles_per_group) * kSTile + tid;
      const int sq = min(max(a.seq_lens[group / a.n_kv_heads], 0), a.max_ctx);
      const int nb = (sq + a.block_size - 1) / a.block_size;
      if (j < a.n_blocks_max) a.scores[static_cast<size_t>(group) * a.n_blocks_max + j] = j < nb ? best : -INFINITY;
      s_fence_before();
      failed = __syncthreads_or(failed);  // every lane's row is read before the next tile overwrites D
      prev_waited = true;                 // this completion is consumed: the next step does not wait on it
    }
  }
  cp_async_wait<0>();
  if (failed && tid == 0 && a.err) atomicOr(a.err, kErrSelectWait);
  s_fence_before();
  __syncthreads();
  if (warp == 0) {
    s_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols) : "memory");
  }
}

template <int NP, int KR>
cudaError_t run_score_tc(const BlockScoreArgs &a, int num_sms, cudaStream_t st) {
  auto kern = block_scores_max_tc_kernel<NP, KR>;
  constexpr int smem = score_tc_smem(NP, KR);
  static int configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  const long long items = static_cast<long long>(a.batch) * a.n_kv_heads * ((a.n_blocks_max + kSTile - 1) / kSTile);
  if (items <= 0 || items > (1LL << 30)) return cudaErrorInvalidValue;
  // two warpgroups per SM where their shared memory fits (d <= 128), so that
  // twice the summary bytes are in flight; the latent rows' B leaves room for one
  const int ctas = smem <= 113 * 1024 ? 2 * num_sms : num_sms;
  const int per = static_cast<int>((items + ctas - 1) / ctas);  // contiguous items per CTA
  const int grid = static_cast<int>((items + per - 1) / per);
  return launch_pdl(kern, dim3(grid), dim3(kSThreads), static_cast<size_t>(smem), st, a, static_cast<int>(items), per);
}

template <int KR>
cudaError_t score_tc_by_heads(const BlockScoreArgs &a, int num_sms, cudaStream_t st) {
  const int G = a.n_q_heads / a.n_kv_heads;
  if (G <= 16) return run_score_tc<16, KR>(a, num_sms, st);
  if (G <= 32) return run_score_tc<32, KR>(a, num_sms, st);
  if (G <= 64) return run_score_tc<64, KR>(a, num_sms, st);
  return cudaErrorInvalidValue;
}

}  // namespace

bool block_scores_max_tc_supported(int dtype, int d, int heads_per_group) {
  return dtype == 1 && (d == 64 || d == 128 || d == 576) && heads_per_group >= 1 && heads_per_group <= 64;
}

cudaError_t launch_block_scores_max_tc(const BlockScoreArgs &a, int num_sms, cudaStream_t st) {
  if (!a.scores) return cudaErrorInvalidValue;
  switch (a.d) {
    case 64: return score_tc_by_heads<2>(a, num_sms, st);
    case 128: return score_tc_by_heads<4>(a, num_sms, st);
    case 576: return score_tc_by_heads<18>(a, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tls
