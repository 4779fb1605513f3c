// tls_attn_tc.cu -- stage 5 (exact attention over the selected tokens) on the
// 5th-generation tensor cores: tcgen05.mma with operands in shared memory and
// accumulators in tensor memory (TMEM).  GQA, bf16, d = 128, G <= 8.
//
// One CTA (one warpgroup, 128 threads) per SM walks a contiguous range of
// (unit, 128-token tile) work, like the CUDA-core kernel.  Per tile:
//   gather   every thread stages rows of K and V with 16-byte cp.async into a
//            3-stage ring (rows of the next-but-one tile are requested as soon
//            as the stage they reuse is free).  A token row is two 128-byte
//            lines (channels 0-63 and 64-127), each in its own region with the
//            16-byte chunks XOR-swizzled by (token & 7): the canonical
//            128B-swizzle layout.  The same bytes are the K-major A operand of
//            S = K Q^T (M = tokens) and the MN-major A operand of O^T = V^T P^T
//            (M = channels).  Masked tokens are zero-filled.
//            (Row gathers through TMA tile::gather4 were measured about 2x
//            slower than these 16-byte copies on the decode workload.)
//   MMA 1    S[128 tok x 16] = K[128 x 128] . Q^T[128 x 16] (heads padded to 16)
//            into TMEM columns 0-15; one thread issues 8 MMAs (K = 16 each).
//   softmax  thread t reads token t's scores (tcgen05.ld), scales by tau log2 e,
//            online max/sum over the tile (warp shuffles + shared memory);
//            the running O^T in TMEM is rescaled by exp2(m_old - m_new) when the
//            max grows (thread t = channel t).
//   MMA 2    O^T[128 ch x 16] += V^T[128 ch x 128 tok] . P^T[128 tok x 16] into
//            TMEM columns 16-31.  P is split into bf16 hi + lo parts (rows 0-7
//            and 8-15 of P^T), so the product keeps ~16 bits of P.
// Completion of each MMA batch is signalled by tcgen05.commit on an mbarrier;
// every wait is bounded (on expiry the kernel records an error and stops).
// When the range leaves a unit, thread t writes channel t of the unit's partial
// (max, sum, o); the log-sum-exp merge kernel of tls_attn.cu combines them.
#include <algorithm>

#include "tls_device.cuh"
#include "tls_internal.h"

namespace tls {
namespace {

constexpr int kTcThreads = 128;
constexpr int kTcTile = 128;         // tokens per tile (MMA M of the score product)
constexpr int kTcStages = 3;
constexpr int kTcD = 128;            // channels (d_qk = d_v)
constexpr int kTcN = 16;             // MMA N: heads (hi rows 0-7, lo rows 8-15 for P)
constexpr int kRegion = kTcTile * 128;               // one 64-channel region of a tile: 16 KB
constexpr int kStageBytes = 4 * kRegion;             // K (2 regions) + V (2 regions)
constexpr int kOpBytes = 2 * kTcN * 128;             // Q^T or P^T: 2 regions x 16 rows x 128 B
constexpr int kOffBytes = kTcStages * kTcTile * 8;   // row byte offsets of the staged tiles (-1: masked)
constexpr int kMiscBytes = 256;                      // mbarriers, TMEM slot, reductions
constexpr int kTcSmem = kStageBytes * kTcStages + 2 * kOpBytes + kOffBytes + kMiscBytes + 1024 /*align*/;
static_assert(8 * 2 + 16 + 32 * 4 + 8 * 4 <= kMiscBytes, "misc block overflows");
static_assert(kTcSmem <= 227 * 1024, "shared memory budget");
constexpr uint32_t kTmemCols = 32;   // S: cols 0-15, O^T: cols 16-31
constexpr uint32_t kWaitLimit = 1u << 24;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      " .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity; false when it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (i > 32) __nanosleep(64);
  }
  return false;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: version 1).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor: kind::f16, bf16 x bf16 -> f32.
constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
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

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
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

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float *v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of element (row, col) in a 128B-swizzled region whose rows are
// 128 bytes (64 bf16): the 16-byte chunk index is XORed with (row & 7).
__device__ __forceinline__ uint32_t sw_off(int row, int col) {
  return row * 128 + ((((col >> 3) ^ row) & 7) << 4) + ((col & 7) << 1);
}

template <int G, bool PAGED>
__global__ void __launch_bounds__(kTcThreads, 1) attn_tc_kernel(AttnArgs a, AttnPlan p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char *stages = smem;                                    // [NS][K r0, K r1, V r0, V r1]
  unsigned char *qt = stages + kTcStages * kStageBytes;            // Q^T: 2 regions x 16 rows x 128 B
  unsigned char *pt = qt + kOpBytes;                               // P^T
  long long *off = reinterpret_cast<long long *>(pt + kOpBytes);   // [NS][128] row byte offsets (-1: masked)
  unsigned char *misc = reinterpret_cast<unsigned char *>(off) + kOffBytes;
  uint64_t *bar_s = reinterpret_cast<uint64_t *>(misc);            // MMA 1 done
  uint64_t *bar_o = bar_s + 1;                                     // MMA 2 done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_o + 1);
  float *red = reinterpret_cast<float *>(tmem_slot + 4);           // [4 warps][8]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t_begin = blockIdx.x * p.tiles_per_warp;
  const int t_end = min(t_begin + p.tiles_per_warp, p.total_tiles);
  if (t_begin >= t_end) return;  // whole CTA: nothing allocated yet

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // P^T and Q^T rows that are never written stay zero
  for (int i = tid; i < 2 * kOpBytes / 16; i += kTcThreads) reinterpret_cast<uint4 *>(qt)[i] = make_uint4(0, 0, 0, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dependency_wait();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s = tmem;        // columns 0-15
  const uint32_t tmem_o = tmem + 16;   // columns 16-31
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

  const unsigned char *Kb = static_cast<const unsigned char *>(a.K);
  const unsigned char *Vb = PAGED ? Kb : static_cast<const unsigned char *>(a.V);
  const long long v_delta = PAGED ? static_cast<long long>(a.block_size) * kTcD * 2 : 0;
  const int Gt = a.n_q_heads / a.n_kv_heads;
  constexpr uint32_t kIdescS = idesc_bf16(kTcTile, kTcN, false, false);
  constexpr uint32_t kIdescO = idesc_bf16(kTcD, kTcN, true, false);

  // Token index of this thread's row of tile t (-1: none), loaded ahead of use.
  auto load_tok = [&](int t) -> int {
    if (t >= t_end) return -1;
    const int unit = t / p.tiles_per_group, tile = t % p.tiles_per_group;
    const int j = tile * kTcTile + tid;
    return j < a.k_t ? a.token_idx[static_cast<size_t>(unit) * a.k_t + j] : -1;
  };
  // Byte offset of this thread's K row of tile t (-1: masked).
  auto off_of = [&](int t, int tok) -> long long {
    if (t >= t_end || tok < 0 || tok >= a.max_ctx) return -1;
    const int group = t / p.tiles_per_group;
    if constexpr (PAGED) {
      const int slot = a.slot_of_block[static_cast<size_t>(group) * a.n_blocks_max + tok / a.block_size];
      if (slot < 0 || slot >= a.n_slots) return -1;
      return ((static_cast<long long>(group) * a.n_slots + slot) * 2 * a.block_size + tok % a.block_size) * (kTcD * 2);
    } else {
      return (static_cast<long long>(group) * a.max_ctx + tok) * (kTcD * 2);
    }
  };
  // All threads: the 128 rows of tile t into stage st (one commit group, always).
  auto issue_rows = [&](int t, int st) {
    if (t < t_end) {
      unsigned char *S = stages + st * kStageBytes;
      // 128 rows x 16 chunks; lanes 0-15 take one row, 16-31 the next (contiguous 256 B each)
#pragma unroll 4
      for (int i = 0; i < kTcTile * 16 / kTcThreads; ++i) {
        const int idx = i * kTcThreads + tid;
        const int row = idx >> 4, c = idx & 15;
        const long long o = off[st * kTcTile + row];
        const bool ok = o >= 0;
        const long long ob = ok ? o : 0;
        const uint32_t d = (c >> 3) * kRegion + row * 128 + ((((c & 7) ^ row) & 7) << 4);
        cp_async16(S + d, Kb + ob + (c << 4), ok);
        cp_async16(S + 2 * kRegion + d, Vb + ob + v_delta + (c << 4), ok);
      }
    }
    cp_async_commit();
  };

  // prologue: tiles t_begin .. t_begin + NS - 2
#pragma unroll
  for (int s = 0; s < kTcStages - 1; ++s) off[s * kTcTile + tid] = off_of(t_begin + s, load_tok(t_begin + s));
  __syncthreads();
#pragma unroll
  for (int s = 0; s < kTcStages - 1; ++s) issue_rows(t_begin + s, s);

  float m[G], l[G];  // running max (log2 units, uniform) and own-token sum
  int cur_unit = -1, first_of_unit = 1;
  uint32_t ph_s = 0, ph_o = 0;
  bool o_pending = false, failed = false;

  auto wait_o = [&]() {
    if (o_pending) {
      if (!mbar_wait(bar_o, ph_o)) failed = true;
      ph_o ^= 1;
      o_pending = false;
      tc_fence_after();
    }
  };

  auto flush = [&](int unit) {
    wait_o();
    // sum of the own-token probabilities over the CTA
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float s = warp_sum(l[h]);
      if (lane == 0) red[warp * 8 + h] = s;
    }
    float ov[16];
    tmem_ld16(tmem_o + lane_base, ov);  // thread t = channel t
    failed = __syncthreads_or(failed);
    const int first = (unit * p.tiles_per_group) / p.tiles_per_warp;
    const int piece = blockIdx.x - first;
    const size_t units = static_cast<size_t>(a.batch) * a.n_kv_heads;
    float *ml = a.part + (static_cast<size_t>(unit) * p.max_pieces + piece) * G * 2;
    float *po = a.part + units * p.max_pieces * G * 2 + (static_cast<size_t>(unit) * p.max_pieces + piece) * G * kTcD;
#pragma unroll
    for (int h = 0; h < G; ++h)
      if (tid == h) {  // m[] indexed by a compile-time h stays in registers
        ml[h * 2] = m[h];
        ml[h * 2 + 1] = red[h] + red[8 + h] + red[16 + h] + red[24 + h];
      }
#pragma unroll
    for (int h = 0; h < G; ++h) po[h * kTcD + tid] = ov[h] + ov[8 + h];
    __syncthreads();
  };

  for (int t = t_begin; t < t_end && !failed; ++t) {
    const int st = (t - t_begin) % kTcStages;
    unsigned char *S = stages + st * kStageBytes;
    const int nxt = t + kTcStages - 1, nst = (nxt - t_begin) % kTcStages;
    const int tok_next = load_tok(nxt);
    // (a) the previous O^T product is complete (its stage is free); this tile's rows have landed
    wait_o();
    off[nst * kTcTile + tid] = off_of(nxt, tok_next);
    cp_async_wait<kTcStages - 2>();
    fence_async_smem();
    failed = __syncthreads_or(failed);
    if (failed) break;
    issue_rows(nxt, nst);  // rows of tile t + NS - 1 stream in while this tile computes
    const int unit = t / p.tiles_per_group;
    if (unit != cur_unit) {
      if (cur_unit >= 0) flush(cur_unit);
      // Q^T rows 0..G-1: raw bf16 q of the group's heads
      const int b = unit / a.n_kv_heads, g = unit % a.n_kv_heads;
      const uint16_t *q = static_cast<const uint16_t *>(a.q) + (static_cast<size_t>(b) * a.n_q_heads + g * Gt) * kTcD;
      for (int i = tid; i < G * kTcD; i += kTcThreads) {
        const int h = i / kTcD, ch = i % kTcD;
        *reinterpret_cast<uint16_t *>(qt + (ch >> 6) * (kTcN * 128) + sw_off(h, ch & 63)) = q[i];
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
      }
      cur_unit = unit;
      first_of_unit = 1;
      fence_async_smem();
      __syncthreads();
    }
    // (b) S = K Q^T
    if (tid == 0) {
      tc_fence_after();
      const uint32_t kbase = smem_u32(S), qbase = smem_u32(qt);
#pragma unroll
      for (int kk = 0; kk < kTcD / 16; ++kk) {
        const uint32_t ko = (kk >> 2) * kRegion + (kk & 3) * 32;
        const uint32_t qo = (kk >> 2) * (kTcN * 128) + (kk & 3) * 32;
        mma_bf16(tmem_s, sw128_desc(kbase + ko, 16, 1024), sw128_desc(qbase + qo, 16, 1024), kIdescS, kk > 0);
      }
      mma_commit(bar_s);
    }
    // (c) scores of own token
    if (!mbar_wait(bar_s, ph_s)) failed = true;
    ph_s ^= 1;
    tc_fence_after();
    float sv[16];
    tmem_ld16(tmem_s + lane_base, sv);
    const bool valid = off[st * kTcTile + tid] >= 0;
    // (d) tile max per head
#pragma unroll
    for (int h = 0; h < G; ++h) {
      sv[h] = valid ? sv[h] * a.scale_log2 : -INFINITY;
      const float wm = warp_max(sv[h]);
      if (lane == 0) red[warp * 8 + h] = wm;
    }
    failed = __syncthreads_or(failed);  // every wait so far succeeded everywhere, or nobody goes on
    if (failed) break;
    bool grow = false;  // uniform: every thread sees the same maxima
    float pr[G], al[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float tm = fmaxf(fmaxf(red[h], red[8 + h]), fmaxf(red[16 + h], red[24 + h]));
      const float mn = fmaxf(m[h], tm);
      al[h] = 1.f;
      pr[h] = 0.f;
      if (mn != -INFINITY) {
        al[h] = ex2f(m[h] - mn);
        pr[h] = ex2f(sv[h] - mn);
      }
      grow |= (mn != m[h]);
      l[h] = l[h] * al[h] + pr[h];
      m[h] = mn;
    }
    // (e) rescale the running O^T (complete: waited at (a)) when the max grew
    if (grow && !first_of_unit) {
      float ov[16];
      tmem_ld16(tmem_o + lane_base, ov);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        ov[h] *= al[h];
        ov[8 + h] *= al[h];
      }
      tmem_st16(tmem_o + lane_base, ov);
    }
    // (f) P^T: row h = hi part, row 8 + h = lo part, column = own token
    {
      unsigned char *pr0 = pt + (tid >> 6) * (kTcN * 128);
      const int col = tid & 63;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const uint16_t hi = f32_to_bf16_rne(pr[h]);
        const float rest = pr[h] - __uint_as_float(static_cast<uint32_t>(hi) << 16);
        *reinterpret_cast<uint16_t *>(pr0 + sw_off(h, col)) = hi;
        *reinterpret_cast<uint16_t *>(pr0 + sw_off(8 + h, col)) = f32_to_bf16_rne(rest);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // (g) O^T += V^T P^T
    if (tid == 0) {
      tc_fence_after();
      const uint32_t vbase = smem_u32(S + 2 * kRegion), pbase = smem_u32(pt);
#pragma unroll
      for (int kk = 0; kk < kTcTile / 16; ++kk) {
        const uint32_t vo = kk * 16 * 128;
        const uint32_t po_ = (kk >> 2) * (kTcN * 128) + (kk & 3) * 32;
        mma_bf16(tmem_o, sw128_desc(vbase + vo, kRegion, 1024), sw128_desc(pbase + po_, 16, 1024), kIdescO,
                 (first_of_unit && kk == 0) ? 0u : 1u);
      }
      mma_commit(bar_o);
    }
    o_pending = true;
    first_of_unit = 0;
  }
  if (cur_unit >= 0 && !failed) flush(cur_unit);
  if (!failed) wait_o();
  cp_async_wait<0>();
  if (failed && tid == 0 && a.err) atomicOr(a.err, kErrAttnWait);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

bool attn_tc_supported(const AttnArgs &a) {
  const int G = a.n_q_heads / a.n_kv_heads;
  return a.dtype == 1 && !a.v_is_k_prefix && a.d_qk == kTcD && a.d_v == kTcD && (G == 1 || G == 2 || G == 4 || G == 8);
}

bool attn_tc_plan(const AttnArgs &a, AttnPlan *p) {
  if (!attn_tc_supported(a)) return false;
  const int G = a.n_q_heads / a.n_kv_heads;
  p->warps_per_cta = kTcThreads / 32;
  p->tokens_per_tile = kTcTile;
  p->head_chunk = G;
  p->n_head_chunks = 1;
  const long long units = static_cast<long long>(a.batch) * a.n_kv_heads;
  p->tiles_per_group = (a.k_t + kTcTile - 1) / kTcTile;
  const long long total = units * p->tiles_per_group;
  if (total <= 0 || total > (1LL << 30)) return false;
  p->total_tiles = static_cast<int>(total);
  const int sms = a.num_sms > 0 ? a.num_sms : 148;
  p->grid = static_cast<int>(std::min<long long>(sms, total));
  p->tiles_per_warp = static_cast<int>((total + p->grid - 1) / p->grid);  // tiles per CTA
  p->max_pieces = (p->tiles_per_group + p->tiles_per_warp - 1) / p->tiles_per_warp + 1;
  p->part_floats = static_cast<size_t>(units) * p->max_pieces * G * (2 + a.d_v);
  return true;
}

template <int G, bool PAGED>
static cudaError_t run_tc(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<G, PAGED>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  return launch_pdl(attn_tc_kernel<G, PAGED>, dim3(p.grid), dim3(kTcThreads), kTcSmem, st, a, p);
}

cudaError_t launch_attention_tc(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  const int G = a.n_q_heads / a.n_kv_heads;
  switch (G) {
    case 1: return a.paged ? run_tc<1, true>(a, p, st) : run_tc<1, false>(a, p, st);
    case 2: return a.paged ? run_tc<2, true>(a, p, st) : run_tc<2, false>(a, p, st);
    case 4: return a.paged ? run_tc<4, true>(a, p, st) : run_tc<4, false>(a, p, st);
    case 8: return a.paged ? run_tc<8, true>(a, p, st) : run_tc<8, false>(a, p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace tls
