// tls_attn_mla_tc.cu -- stage 5 of the AsyncTLS decode step for the latent
// (MLA) shape on the 5th-generation tensor cores: tcgen05.mma with operands in
// shared memory and fp32 accumulators in tensor memory (TMEM).
//
// Every query head of a group attends over the same 576-channel latent rows of
// the kept tokens, V being the first 512 channels of each row (gist.science
// (es) section 2.A.2: the final attention runs at token precision on the K_t
// kept tokens).  64 heads x (576 + 512) channels per kept token is a real
// dense contraction.
//
// Work: the flattened (group, 32-token tile) space is cut into equal
// contiguous ranges, one per CTA (one warpgroup, 128 threads).  TMEM holds S
// (32 fp32 columns) and O (256 columns): O row h holds head h's channels
// 0-255 and row 64 + h its channels 256-511.  Per tile:
//   gather   every thread copies a quarter of one of the tile's 32 latent rows
//            (1152 B each) with 16-byte cp.async into a 3-stage ring (the
//            tile after next is requested as soon as the tile before it is
//            done); a stage is 9 regions of 32 rows x 128 B (64 channels),
//            128-byte swizzled, zero-filled for masked tokens.
//   MMA 1    S[128 x 32] = Q[128 x 576] . K^T: A = the group's queries, K-major,
//            9 regions of 64 rows; M = 128 reads rows 64-127 from the bytes
//            after each region (the next region, or the ring after the last),
//            and those rows of S are never read.  B = the stage (N = 32
//            tokens, K-major).  36 k-steps of 16 channels, one issuing thread.
//   softmax  thread h < 64 reads head h's 32 scores (tcgen05.ld), scales them
//            by tau log2(e), masks invalid tokens and keeps the head's
//            reference max and sum.  The reference max moves only when the
//            tile's max exceeds it by more than 8 (log2 units), and only then
//            is O rescaled: the weights 2^(s - m) stay below 256.  Each weight
//            is split into a bf16 part and the bf16 of its remainder, so the
//            product keeps ~16 bits of it.
//   MMA 2    O += P . V, both channel halves: A = P (row h = head h's hi parts
//            of the 32 tokens, then its lo parts: K = 64 as four k-steps),
//            B = V = channels of the same staged rows (MN-major, N = 256).
//            For channels 0-255 the A rows 0-63 are P and rows 64-127 zero,
//            for channels 256-511 the reverse, so both products accumulate
//            into the same 256 columns without disturbing each other's rows.
// When the range leaves a group, the CTA writes the group's partial (max, sum
// and 512 channels per head) in the layout of the warp-MMA latent kernel, and
// the log-sum-exp merge kernel of tls_attn.cu combines the pieces.  Completion
// of each MMA batch is signalled by tcgen05.commit on an mbarrier; every wait
// is bounded (on expiry the CTA records an error and stops, freeing its TMEM).
#include <algorithm>

#include "tls_device.cuh"
#include "tls_internal.h"

namespace tls {
namespace {

constexpr int kLD = 576, kLDV = 512;
constexpr int kLRB = kLD * 2;                     // bytes of one latent row
constexpr int kLThreads = 128;
constexpr int kLT = 32;                           // tokens per tile (N of MMA 1, K of MMA 2)
constexpr int kLStages = 3;
constexpr int kLRegions = kLD / 64;               // 9 regions of 64 channels
constexpr int kLHalf = kLDV / 2;                  // channels per MMA 2 product (N)
constexpr int kLHeads = 64;                       // heads per group (MMA rows 0-63)
constexpr int kQRegion = kLHeads * 128;           // 8 KB: 64 rows x 128 B
constexpr int kKRegion = kLT * 128;               // 4 KB: 32 rows x 128 B
constexpr int kQBytes = kLRegions * kQRegion;     // 72 KB
constexpr int kStageBytes = kLRegions * kKRegion; // 36 KB
constexpr int kLMisc = 1024;                      // stage masks, mbarriers, TMEM slot, alpha
constexpr int kLStaging = 4 * 32 * 128;           // flush: one 32 x 32 fp32 block per warp
constexpr int kLSmem = kQBytes + kLStages * kStageBytes + 3 * kQRegion + kLStaging + kLMisc + 1024 /*align*/;
static_assert(kLSmem <= 227 * 1024, "shared memory budget");
constexpr uint32_t kLCols = 512;                  // S: cols 0-31, O: cols 256-511
constexpr uint32_t kLWait = 1u << 24;
constexpr float kRescaleAt = 8.f;                 // log2 units a head's max may grow before O is rescaled

__device__ __forceinline__ bool l_mbar_wait(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < kLWait; ++i) {
    if (mbarrier_try_wait(bar, parity)) return true;
    if (i > 32) __nanosleep(64);
  }
  return false;
}
__device__ __forceinline__ void l_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void l_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void l_fence_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format).
__device__ __forceinline__ uint64_t l_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor: kind::f16, bf16 x bf16 -> f32.
constexpr uint32_t l_idesc(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void l_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
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

__device__ __forceinline__ void l_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void l_ld32(uint32_t taddr, float *v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void l_st32(uint32_t taddr, const float *v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
      "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
      "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
      "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
      "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float l_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of 16-byte chunk c (0-7) of row r inside a 128B-swizzled region.
__device__ __forceinline__ uint32_t l_sw(int r, int c) { return r * 128 + (((c ^ r) & 7) << 4); }

// Shared memory (1024-byte aligned):
//   [Q: 9 regions x 64 rows x 128 B][ring: 3 stages x 9 regions x 32 rows x 128 B]
//   [P buffer: Z0 | P | Z1, 3 x 64 rows x 128 B][flush staging: 4 x 4 KB]
//   [stage masks, mbarriers, TMEM slot, alpha]
// P row h = [hi of tokens 0-31 | lo of tokens 0-31] (64 bf16 = one 128-byte row).
// The A operand of MMA 2 for channels 0-255 starts at P (rows 64-127 = Z1 = 0),
// for channels 256-511 at Z0 (rows 0-63 = 0, rows 64-127 = P), so the two
// products accumulate into the same 256 TMEM columns without touching each
// other's rows: O row h = head h channels 0-255, row 64 + h = head h channels
// 256-511.
constexpr int kOffRing = kQBytes;
constexpr int kOffP = kOffRing + kLStages * kStageBytes;
constexpr int kOffStaging = kOffP + 3 * kQRegion;
constexpr int kOffMisc = kOffStaging + kLStaging;

__global__ void __launch_bounds__(kLThreads, 1) attn_mla_tc_kernel(AttnArgs a, AttnPlan p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem =
      reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char *Qs = smem;
  unsigned char *ring = smem + kOffRing;
  unsigned char *Pb = smem + kOffP;
  uint32_t *mask = reinterpret_cast<uint32_t *>(smem + kOffMisc);        // [kLStages] valid tokens of a stage
  uint64_t *bar_s = reinterpret_cast<uint64_t *>(smem + kOffMisc + 64);   // MMA 1 (and all before it) done
  uint64_t *bar_o = bar_s + 1;                                            // flush: every MMA done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc + 96);
  float *alpha_s = reinterpret_cast<float *>(smem + kOffMisc + 128);     // [64] rescale factors of O rows
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.n_q_heads / a.n_kv_heads;
  const int tpc = p.tiles_per_warp;  // tiles per CTA
  const int t_begin = blockIdx.x * tpc;
  const int t_end = min(t_begin + tpc, p.total_tiles);
  if (t_begin >= t_end) return;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(kLCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    mbarrier_init(bar_s, 1);
    mbarrier_init(bar_o, 1);
    mbarrier_init_fence();
  }
  // Z0 and Z1 stay zero for the whole launch
  for (int i = tid; i < kQRegion / 16; i += kLThreads) {
    reinterpret_cast<uint4 *>(Pb)[i] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4 *>(Pb + 2 * kQRegion)[i] = make_uint4(0, 0, 0, 0);
  }
  l_fence_before();
  __syncthreads();
  l_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t tmem_s = tmem, tmem_o = tmem + 256;
  grid_dependency_wait();

  const unsigned char *Kb = static_cast<const unsigned char *>(a.K);
  const unsigned char *qb = static_cast<const unsigned char *>(a.q);

  // the group's queries: row h < G = head h, rows G..63 zero; chunk c of a
  // row lands in region c / 8, chunk c % 8 (swizzled by the row)
  auto load_q = [&](int group) {
    const int b = group / a.n_kv_heads, gk = group % a.n_kv_heads;
    const unsigned char *src = qb + (static_cast<size_t>(b) * a.n_q_heads + static_cast<size_t>(gk) * G) * kLRB;
    for (int idx = tid; idx < kLHeads * (kLRB / 16); idx += kLThreads) {
      const int h = idx / (kLRB / 16), c = idx % (kLRB / 16);
      const bool ok = h < G;
      cp_async16(Qs + (c >> 3) * kQRegion + l_sw(h, c & 7), src + static_cast<size_t>(ok ? h : 0) * kLRB + c * 16,
                 ok);
    }
  };
  // gather of flattened tile tt into stage st: thread t copies row t / 4,
  // chunks t % 4 + 4 i (i < 18); masked tokens are zero-filled
  auto issue_tile = [&](int tt, int st) {
    if (tt >= t_end) return;
    const int group = tt / p.tiles_per_group, tile = tt % p.tiles_per_group;
    const int row = tid >> 2, sub = tid & 3;
    const int j = tile * kLT + row;
    long long off = -1;
    if (j < a.k_t) {
      const int tok = __ldcg(a.token_idx + static_cast<size_t>(group) * a.k_t + j);
      if (tok >= 0 && tok < a.max_ctx) off = (static_cast<long long>(group) * a.max_ctx + tok) * kLRB;
    }
    const bool ok = off >= 0;
    const unsigned vb = __ballot_sync(0xffffffffu, ok && sub == 0);
    if (lane == 0) {
      uint32_t byte = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) byte |= ((vb >> (4 * k)) & 1u) << k;
      reinterpret_cast<unsigned char *>(&mask[st])[warp] = static_cast<unsigned char>(byte);
    }
    unsigned char *S = ring + st * kStageBytes;
    const unsigned char *src = Kb + (ok ? off : 0);
#pragma unroll
    for (int i = 0; i < kLRB / 16 / 4; ++i) {
      const int c = sub + 4 * i;
      cp_async16(S + (c >> 3) * kKRegion + l_sw(row, c & 7), src + c * 16, ok);
    }
  };

  // softmax state of head tid (threads 0-63): reference max (log2 domain) and
  // the sum of the weights taken against it
  float m_ref = -INFINITY, l_sum = 0.f;
  bool failed = false;
  uint32_t ph_s = 0, ph_o = 0;
  constexpr uint32_t kIdescS = l_idesc(128, kLT, false, false);
  constexpr uint32_t kIdescO = l_idesc(128, kLHalf, false, true);

  // the unit's partial: (max, sum) of each head, and O (row h: head h
  // channels 0-255; row 64 + h: head h channels 256-511); every MMA is
  // complete first
  auto flush = [&](int unit) {
    if (tid == 0) l_commit(bar_o);
    if (!l_mbar_wait(bar_o, ph_o)) failed = true;
    ph_o ^= 1u;
    l_fence_after();
    const int first = (unit * p.tiles_per_group) / tpc;
    const int piece = blockIdx.x - first;
    const size_t units = static_cast<size_t>(a.batch) * a.n_kv_heads;
    float *ml = a.part + (static_cast<size_t>(unit) * p.max_pieces + piece) * G * 2;
    float *po = a.part + units * p.max_pieces * G * 2 + (static_cast<size_t>(unit) * p.max_pieces + piece) * G * kLDV;
    if (tid < G) {
      ml[tid * 2] = m_ref;
      ml[tid * 2 + 1] = l_sum;
    }
    // Each warp moves its 32 rows 32 columns at a time through a swizzled
    // 4 KB block of shared memory, so that the global stores are whole
    // 128-byte row segments (8 lanes per row, 4 rows per instruction).
    unsigned char *stg = smem + kOffStaging + warp * 4096;
#pragma unroll 1
    for (int c0 = 0; c0 < kLHalf; c0 += 32) {
      float v[32];
      l_ld32(tmem_o + lane_base + c0, v);  // warp-collective: lane = row 32 warp + lane
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4 *>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
            make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int r = 4 * k + (lane >> 3), cj = lane & 7;
        const int row = warp * 32 + r, head = row & 63, half = row >> 6;
        const float4 x = *reinterpret_cast<const float4 *>(stg + r * 128 + ((cj ^ (r & 7)) << 4));
        if (head < G) *reinterpret_cast<float4 *>(po + static_cast<size_t>(head) * kLDV + half * kLHalf + c0 + 4 * cj) = x;
      }
      __syncwarp();
    }
  };

  int cur_unit = t_begin / p.tiles_per_group;
  bool first_of_unit = true;
  load_q(cur_unit);
  issue_tile(t_begin, 0);
  cp_async_commit();
  issue_tile(t_begin + 1, 1);
  cp_async_commit();
  int st = 0;
  for (int t = t_begin; t < t_end; ++t) {
    // (a) tile t (and the queries) landed; visible to the tensor cores
    cp_async_wait<1>();
    l_fence_async();
    l_fence_before();
    failed = __syncthreads_or(failed);
    if (failed) break;
    const int unit = t / p.tiles_per_group;
    if (unit != cur_unit) {  // the range enters the next group
      flush(cur_unit);
      l_fence_before();
      __syncthreads();  // O is read and every MMA reading the old queries is complete
      load_q(unit);
      cp_async_commit();
      cp_async_wait<0>();
      l_fence_async();
      m_ref = -INFINITY;
      l_sum = 0.f;
      first_of_unit = true;
      cur_unit = unit;
      failed = __syncthreads_or(failed);
      if (failed) break;
    }
    unsigned char *S = ring + st * kStageBytes;
    // (b) MMA 1: S = Q . K^T over 36 k-steps
    if (tid == 0) {
      l_fence_after();
      const uint32_t qbase = smem_addr(Qs), kbase = smem_addr(S);
#pragma unroll
      for (int r = 0; r < kLRegions; ++r)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          l_mma(tmem_s, l_desc(qbase + r * kQRegion + kk * 32, 16, 1024), l_desc(kbase + r * kKRegion + kk * 32, 16, 1024),
                kIdescS, (r | kk) ? 1u : 0u);
      l_commit(bar_s);
    }
    // (c) MMA 1 done, and with it every earlier MMA: the stage of tile t - 1
    //     and the P buffer are free
    if (!l_mbar_wait(bar_s, ph_s)) failed = true;
    ph_s ^= 1u;
    l_fence_after();
    // (d) the gather of tile t + 2 into the stage tile t - 1 used
    {
      int st2 = st + 2;
      if (st2 >= kLStages) st2 -= kLStages;
      issue_tile(t + 2, st2);
      cp_async_commit();
    }
    // (e) softmax of head tid over the tile's 32 tokens; P row tid
    bool need_rescale = false;
    if (warp < 2) {  // warp-uniform: TMEM lanes 0-63 belong to warps 0 and 1
      float s[32];
      l_ld32(tmem_s + lane_base, s);
      const uint32_t vm = mask[st];
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        s[j] = ((vm >> j) & 1u) ? s[j] * a.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, s[j]);
      }
      float alpha = 1.f;
      if (tmax > m_ref + kRescaleAt) {  // also the first finite max (m_ref = -inf)
        alpha = m_ref == -INFINITY ? 0.f : l_ex2(m_ref - tmax);
        need_rescale = m_ref != -INFINITY;
        m_ref = tmax;
        l_sum *= alpha;
      }
      alpha_s[tid] = alpha;
      const bool live = tid < G && m_ref != -INFINITY;
      uint32_t hi[16], lo[16];
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float p0 = live ? l_ex2(s[j] - m_ref) : 0.f;  // masked: exp2(-inf) = 0
        const float p1 = live ? l_ex2(s[j + 1] - m_ref) : 0.f;
        sum += p0 + p1;
        const uint32_t h0 = f32_to_bf16_rne(p0), h1 = f32_to_bf16_rne(p1);
        const float r0 = p0 - __uint_as_float(h0 << 16), r1 = p1 - __uint_as_float(h1 << 16);
        hi[j / 2] = h0 | (h1 << 16);
        lo[j / 2] = static_cast<uint32_t>(f32_to_bf16_rne(r0)) | (static_cast<uint32_t>(f32_to_bf16_rne(r1)) << 16);
      }
      l_sum += sum;
      unsigned char *prow = Pb + kQRegion;  // rows 0-63 of the P region
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        *reinterpret_cast<uint4 *>(prow + l_sw(tid, c)) = make_uint4(hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
        *reinterpret_cast<uint4 *>(prow + l_sw(tid, 4 + c)) =
            make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
      }
    }
    l_fence_async();
    l_fence_before();
    const int rescale = __syncthreads_or(need_rescale && !first_of_unit);
    failed = __syncthreads_or(failed);
    if (failed) break;
    // (f) rare: a head's max grew by more than kRescaleAt; scale its O rows
    if (rescale) {
      l_fence_after();
      const float al = alpha_s[tid & 63];
#pragma unroll 1
      for (int c0 = 0; c0 < kLHalf; c0 += 32) {
        float v[32];
        l_ld32(tmem_o + lane_base + c0, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= al;
        l_st32(tmem_o + lane_base + c0, v);
      }
      l_fence_before();
      __syncthreads();
    }
    // (g) MMA 2: O += P . V for both channel halves (hi and lo parts as four
    //     k-steps of 16: hi tokens 0-15, 16-31, lo tokens 0-15, 16-31)
    if (tid == 0) {
      l_fence_after();
      const uint32_t pbase = smem_addr(Pb), vbase = smem_addr(S);
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t ad = pbase + (c == 0 ? kQRegion : 0) + kk * 32;
          const uint32_t bd = vbase + (4 * c) * kKRegion + (kk & 1) * 16 * 128;
          l_mma(tmem_o, l_desc(ad, 16, 1024), l_desc(bd, kKRegion, 1024), kIdescO,
                (first_of_unit && c == 0 && kk == 0) ? 0u : 1u);
        }
    }
    first_of_unit = false;
    if (++st == kLStages) st = 0;
  }
  if (!failed) flush(cur_unit);
  cp_async_wait<0>();
  l_fence_before();
  failed = __syncthreads_or(failed);
  if (failed && tid == 0 && a.err) atomicOr(a.err, kErrAttnWait);
  if (warp == 0) {
    l_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kLCols) : "memory");
  }
}

}  // namespace

bool attn_mla_tc_supported(const AttnArgs &a) {
  const int G = a.n_kv_heads > 0 ? a.n_q_heads / a.n_kv_heads : 0;
  return a.v_is_k_prefix && a.dtype == 1 && a.d_qk == kLD && a.d_v == kLDV && !a.paged && G >= 4 && G <= kLHeads &&
         (G & (G - 1)) == 0;
}

int attn_mla_tc_tokens_per_tile() { return kLT; }

cudaError_t launch_attention_mla_tc(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kLSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  return launch_pdl(attn_mla_tc_kernel, dim3(p.grid), dim3(kLThreads), static_cast<size_t>(kLSmem), st, a, p);
}

}  // namespace tls
