// tls_attn.cu -- stage 5 of the AsyncTLS decode step: exact softmax attention
// over the gathered K/V rows of the selected tokens (gist.science (es) section
// 2.A.2: the final attention runs at token precision on the K_t kept tokens).
//
// Design (B200):
//  * Work = (unit, tile): a unit is one KV group (all G heads of a GQA group, or
//    a chunk of HG heads of a latent group); a tile is 32 selected tokens.  The
//    flattened tile space is cut into equal contiguous ranges, one per warp of a
//    persistent grid (one CTA per SM), so every warp streams the same number of
//    gathered rows and never waits on another warp.
//  * Each warp runs its own NS-stage cp.async pipeline: row offsets of the
//    tile's tokens go to shared memory, then the warp gathers the 32 K rows
//    (and V rows) as 16-byte async copies (zero-fill for masked tokens) into a
//    private stage buffer.  K rows are stored with their 16-byte chunks XOR-
//    swizzled by (row & 7) so that lane r reading row r is conflict-free.
//  * QK: lane r owns token r of the tile and dots its K row with the group's
//    queries (fp32 in shared memory, pre-scaled by tau * log2 e, broadcast
//    reads), packed fp32x2 FMA.  Online softmax per head with a warp max.
//  * PV: lane owns d_v / 32 output channels for every head of the unit; the
//    per-token probabilities are broadcast from shared memory.
//  * When a warp's range leaves a unit it writes its partial (max, sum, o) for
//    that unit; a merge kernel combines the partials of each head by
//    log-sum-exp and writes out / lse.
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "tls_device.cuh"
#include "tls_internal.h"

namespace tls {
namespace {

constexpr int kTT = 16;  // tokens per tile (two lanes per token in QK)

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <typename E, int D, int DV, int HG, bool VPREFIX, int NS>
struct AttnLayout {
  static constexpr int kElt = E::kBytes;
  static constexpr int RB = D * kElt;                     // K row bytes
  static constexpr int KCH = RB / 16;                     // 16-byte chunks per K row
  static constexpr int VB = VPREFIX ? 0 : DV * kElt;      // V row bytes (0: V inside the K row)
  static constexpr int VCH = VB / 16;
  static constexpr int CPL = DV / 32;                     // output channels per lane
  static constexpr int kStageBytes = kTT * (RB + VB);
  static constexpr int kWarpBytes = NS * kStageBytes + HG * D * 4 + kTT * HG * 4 + NS * kTT * 8;
  static constexpr int kMaxSmem = 227 * 1024;
  static constexpr int W = (kMaxSmem / kWarpBytes) < 16 ? (kMaxSmem / kWarpBytes) : 16;  // warps per CTA
  static constexpr int kSmem = W * kWarpBytes;
  static_assert(KCH % 8 == 0, "the row swizzle permutes groups of 8 chunks (rows of a multiple of 128 bytes)");
  static_assert((kTT * KCH) % 32 == 0, "issue loop covers whole warps");
  static_assert(DV % 64 == 0, "d_v must be a multiple of 64");
  static_assert(W >= 1, "one warp's buffers must fit in shared memory");
};

// One CTA per SM; every warp streams its own contiguous range of (unit, tile)
// work.  Two lanes share a token: lane l handles token l & 15 and the half
// (l >> 4) of its channels in QK.
template <typename E, int D, int DV, int HG, bool VPREFIX, bool PAGED, int NS>
__global__ void __launch_bounds__(AttnLayout<E, D, DV, HG, VPREFIX, NS>::W * 32, 1)
    attn_split_kernel(AttnArgs a, AttnPlan p) {
  using L = AttnLayout<E, D, DV, HG, VPREFIX, NS>;
  using S = typename E::storage;
  constexpr int EPC = E::kEPC;
  constexpr int CPL = L::CPL;
  constexpr int HALF = L::KCH / 2;  // QK chunks per lane
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tr = lane & 15, hf = lane >> 4;
  unsigned char *wbase = smem + warp * L::kWarpBytes;
  float *Qs = reinterpret_cast<float *>(wbase + NS * L::kStageBytes);  // [HG][D]
  float *Ps = Qs + HG * D;                                             // [kTT][HG]
  long long *Off = reinterpret_cast<long long *>(Ps + kTT * HG);       // [NS][kTT] byte offsets

  grid_dependency_wait();
  const int gw = blockIdx.x * L::W + warp;
  const int t_begin = gw * p.tiles_per_warp;
  const int t_end = min(t_begin + p.tiles_per_warp, p.total_tiles);
  if (t_begin >= t_end) return;

  const unsigned char *Kb = static_cast<const unsigned char *>(a.K);
  const unsigned char *Vb = (VPREFIX || PAGED) ? Kb : static_cast<const unsigned char *>(a.V);
  const long long v_delta = PAGED ? static_cast<long long>(a.block_size) * L::RB : 0;
  const int Gt = a.n_q_heads / a.n_kv_heads;

  // Gather the rows of tile t into stage st (always commits one group).
  auto issue = [&](int t, int st) {
    if (t < t_end) {
      const int unit = t / p.tiles_per_group, tile = t % p.tiles_per_group;
      const int group = unit / p.n_head_chunks;
      if (lane < kTT) {
        const int j = tile * kTT + lane;
        long long off = -1;
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
        Off[st * kTT + lane] = off;
      }
      __syncwarp();
      unsigned char *Ks = wbase + st * L::kStageBytes;
      unsigned char *Vs = Ks + kTT * L::RB;
#pragma unroll
      for (int i = 0; i < kTT * L::KCH / 32; ++i) {
        const int idx = i * 32 + lane;
        const int row = idx / L::KCH, c = idx % L::KCH;
        const long long o = Off[st * kTT + row];
        const bool ok = o >= 0;
        const long long ob = ok ? o : 0;
        cp_async16(Ks + row * L::RB + ((c ^ (row & 7)) << 4), Kb + ob + (c << 4), ok);
        if constexpr (!VPREFIX) {
          // GQA: V rows have the same chunk count as K rows
          cp_async16(Vs + row * L::VB + (c << 4), Vb + ob + v_delta + (c << 4), ok);
        }
      }
    }
    cp_async_commit();
  };

  float2 acc[HG][CPL / 2];
  float m[HG], l[HG];
  int cur_unit = -1;

  auto reset = [&]() {
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
#pragma unroll
      for (int c = 0; c < CPL / 2; ++c) acc[h][c] = make_float2(0.f, 0.f);
    }
  };

  auto flush = [&](int unit) {
    const int first = (unit * p.tiles_per_group) / p.tiles_per_warp;
    const int piece = gw - first;
    const size_t units = static_cast<size_t>(a.batch) * a.n_kv_heads * p.n_head_chunks;
    float *ml = a.part + (static_cast<size_t>(unit) * p.max_pieces + piece) * HG * 2;
    float *po = a.part + units * p.max_pieces * HG * 2 + (static_cast<size_t>(unit) * p.max_pieces + piece) * HG * DV;
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      const float lt = warp_sum(l[h]);
      if (lane == 0) { ml[h * 2] = m[h]; ml[h * 2 + 1] = lt; }
      float2 *dst = reinterpret_cast<float2 *>(po + h * DV + lane * CPL);
#pragma unroll
      for (int c = 0; c < CPL / 2; ++c) dst[c] = acc[h][c];
    }
  };

  auto load_q = [&](int unit) {
    const int group = unit / p.n_head_chunks, hc = unit % p.n_head_chunks;
    const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
    const size_t q0 = (static_cast<size_t>(b) * a.n_q_heads + g * Gt + hc * HG) * D;
    for (int i = lane; i < HG * D; i += 32) Qs[i] = load_elem<E>(a.q, q0 + i) * a.scale_log2;
    __syncwarp();
  };

#pragma unroll
  for (int s = 0; s < NS - 1; ++s) issue(t_begin + s, s);

  for (int t = t_begin; t < t_end; ++t) {
    const int st = (t - t_begin) % NS;
    issue(t + NS - 1, (t + NS - 1 - t_begin) % NS);
    cp_async_wait<NS - 1>();
    __syncwarp();
    const int unit = t / p.tiles_per_group;
    if (unit != cur_unit) {
      if (cur_unit >= 0) flush(cur_unit);
      reset();
      load_q(unit);
      cur_unit = unit;
    }
    const unsigned char *Ks = wbase + st * L::kStageBytes;
    const bool valid = Off[st * kTT + tr] >= 0;

    // ---- scores: token tr, channel half hf
    float2 s2[HG];
#pragma unroll
    for (int h = 0; h < HG; ++h) s2[h] = make_float2(0.f, 0.f);
    const unsigned char *krow = Ks + tr * L::RB;
#pragma unroll 4
    for (int jj = 0; jj < HALF; ++jj) {
      const int j = hf * HALF + jj;
      const uint4 kc = *reinterpret_cast<const uint4 *>(krow + ((j ^ (tr & 7)) << 4));
      float kf[EPC];
      chunk_to_f32<E>(kc, kf);
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float4 *qp = reinterpret_cast<const float4 *>(Qs + h * D + j * EPC);
#pragma unroll
        for (int e = 0; e < EPC / 4; ++e) {
          const float4 qv = qp[e];
          ffma2(s2[h], make_float2(kf[4 * e], kf[4 * e + 1]), make_float2(qv.x, qv.y));
          ffma2(s2[h], make_float2(kf[4 * e + 2], kf[4 * e + 3]), make_float2(qv.z, qv.w));
        }
      }
    }
    // ---- online softmax (log2 domain); both lanes of a token hold its score
#pragma unroll
    for (int h = 0; h < HG; ++h) {
      float sc = s2[h].x + s2[h].y;
      sc += __shfl_xor_sync(0xffffffffu, sc, 16);
      sc = valid ? sc : -INFINITY;
      float tm = sc;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, o));
      const float mn = fmaxf(m[h], tm);
      float alpha = 1.f, pr = 0.f;
      if (mn != -INFINITY) {
        alpha = ex2(m[h] - mn);
        pr = ex2(sc - mn);
      }
      l[h] = l[h] * alpha + (hf == 0 ? pr : 0.f);
#pragma unroll
      for (int c = 0; c < CPL / 2; ++c) {
        acc[h][c].x *= alpha;
        acc[h][c].y *= alpha;
      }
      m[h] = mn;
      if (hf == 0) Ps[tr * HG + h] = pr;
    }
    __syncwarp();
    // ---- o += p v: lane owns channels [lane*CPL, lane*CPL + CPL)
    const unsigned char *Vs = VPREFIX ? Ks : Ks + kTT * L::RB;
#pragma unroll 4
    for (int r = 0; r < kTT; ++r) {
      float pv[HG];
      if constexpr (HG % 4 == 0) {
#pragma unroll
        for (int h = 0; h < HG; h += 4) {
          const float4 p4 = *reinterpret_cast<const float4 *>(Ps + r * HG + h);
          pv[h] = p4.x; pv[h + 1] = p4.y; pv[h + 2] = p4.z; pv[h + 3] = p4.w;
        }
      } else {
#pragma unroll
        for (int h = 0; h < HG; ++h) pv[h] = Ps[r * HG + h];
      }
      float vf[CPL];
      if constexpr (VPREFIX) {
#pragma unroll
        for (int q = 0; q < CPL / EPC; ++q) {
          const int c = lane * (CPL / EPC) + q;
          const uint4 vc = *reinterpret_cast<const uint4 *>(Vs + r * L::RB + ((c ^ (r & 7)) << 4));
          chunk_to_f32<E>(vc, vf + q * EPC);
        }
      } else {
        const unsigned char *vr = Vs + r * L::VB + lane * CPL * L::kElt;
        if constexpr (CPL * L::kElt == 16) {
          chunk_to_f32<E>(*reinterpret_cast<const uint4 *>(vr), vf);
        } else if constexpr (CPL * L::kElt == 8) {
          const uint2 w = *reinterpret_cast<const uint2 *>(vr);
          if constexpr (sizeof(S) == 2) {
            vf[0] = bf16_lo(w.x); vf[1] = bf16_hi(w.x); vf[2] = bf16_lo(w.y); vf[3] = bf16_hi(w.y);
          } else {
            vf[0] = __uint_as_float(w.x); vf[1] = __uint_as_float(w.y);
          }
        } else {
          static_assert(CPL * L::kElt == 4, "unsupported V slice");
          const uint32_t w = *reinterpret_cast<const uint32_t *>(vr);
          vf[0] = bf16_lo(w); vf[1] = bf16_hi(w);
        }
      }
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float2 pp = make_float2(pv[h], pv[h]);
#pragma unroll
        for (int c = 0; c < CPL / 2; ++c) ffma2(acc[h][c], make_float2(vf[2 * c], vf[2 * c + 1]), pp);
      }
    }
    __syncwarp();
  }
  if (cur_unit >= 0) flush(cur_unit);
  cp_async_wait<0>();
}

// Log-sum-exp merge of the pieces of one (unit, head, 32-channel slice); one
// warp each, one channel per lane.  The pieces' (max, sum) are read by the
// lanes in parallel, 32 pieces at a time; their partial outputs are then read
// as independent coalesced loads.
template <int DV, int HG>
__global__ void __launch_bounds__(128) attn_merge_kernel(AttnArgs a, AttnPlan p) {
  constexpr int NSL = DV / 32;
  grid_dependency_wait();
  const int lane = threadIdx.x & 31;
  const int w = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int n_units = a.batch * a.n_kv_heads * p.n_head_chunks;
  if (w >= n_units * HG * NSL) return;
  const int unit = w / (HG * NSL), rem = w % (HG * NSL);
  const int hh = rem / NSL, sl = rem % NSL;
  const int group = unit / p.n_head_chunks, hc = unit % p.n_head_chunks;
  const int b = group / a.n_kv_heads, g = group % a.n_kv_heads;
  const int Gt = a.n_q_heads / a.n_kv_heads;
  const int head = g * Gt + hc * HG + hh;
  const int first = (unit * p.tiles_per_group) / p.tiles_per_warp;
  const int last = ((unit + 1) * p.tiles_per_group - 1) / p.tiles_per_warp;
  const int n_pieces = last - first + 1;
  const int ch = sl * 32 + lane;
  const float *ml = a.part + static_cast<size_t>(unit) * p.max_pieces * HG * 2;
  const float *po = a.part + static_cast<size_t>(n_units) * p.max_pieces * HG * 2 +
                    static_cast<size_t>(unit) * p.max_pieces * HG * DV + hh * DV + ch;
  float M = -INFINITY, Lsum = 0.f, o = 0.f;
  for (int q0 = 0; q0 < n_pieces; q0 += 32) {
    // all loads of the chunk first (none depends on another): one round trip
    const int nq = min(32, n_pieces - q0);
    float v[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = k < nq ? po[static_cast<size_t>(q0 + k) * HG * DV] : 0.f;
    const int q = q0 + lane;
    const float mq = q < n_pieces ? ml[(q * HG + hh) * 2] : -INFINITY;
    const float lq = q < n_pieces ? ml[(q * HG + hh) * 2 + 1] : 0.f;
    const float Mn = fmaxf(M, warp_max(mq));
    const bool any = Mn != -INFINITY;  // false: no token of the unit so far
    const float scale_old = any ? ex2(M - Mn) : 1.f;
    const float wq = any ? ex2(mq - Mn) : 0.f;
    Lsum = Lsum * scale_old + warp_sum(wq * lq);
    o *= scale_old;
#pragma unroll
    for (int k = 0; k < 32; ++k) o = fmaf(__shfl_sync(0xffffffffu, wq, k), v[k], o);
    M = Mn;
  }
  const float res = Lsum > 0.f ? o / Lsum : 0.f;
  const size_t ob = (static_cast<size_t>(b) * a.n_q_heads + head) * DV + ch;
  if (a.out_dtype == 1) static_cast<uint16_t *>(a.out)[ob] = f32_to_bf16_rne(res);
  else static_cast<float *>(a.out)[ob] = res;
  if (a.lse && sl == 0 && lane == 0)
    a.lse[static_cast<size_t>(b) * a.n_q_heads + head] =
        (M == -INFINITY || Lsum <= 0.f) ? -INFINITY : (M + log2f(Lsum)) * 0.69314718055994531f;
}

template <typename E, int D, int DV, int HG, bool VPREFIX, bool PAGED, int NS>
cudaError_t run_attention(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  using L = AttnLayout<E, D, DV, HG, VPREFIX, NS>;
  auto kern = attn_split_kernel<E, D, DV, HG, VPREFIX, PAGED, NS>;
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

template <int DV, int HG>
cudaError_t run_merge(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  const int n_warps = a.batch * a.n_kv_heads * p.n_head_chunks * HG * (DV / 32);
  return launch_pdl(attn_merge_kernel<DV, HG>, dim3((n_warps + 3) / 4), dim3(128), 0, st, a, p);
}

// Kernel-set selection.  Returns false for shapes outside the compiled set.
struct Variant {
  int warps, head_chunk;
};

constexpr int kStages = 2;

template <typename E, int D, int DV, int HG, bool VPREFIX>
constexpr int warps_of() {
  return AttnLayout<E, D, DV, HG, VPREFIX, kStages>::W;
}

template <typename E, int D>
int gqa_warps(int G) {
  switch (G) {
    case 1: return warps_of<E, D, D, 1, false>();
    case 2: return warps_of<E, D, D, 2, false>();
    case 4: return warps_of<E, D, D, 4, false>();
    default: return warps_of<E, D, D, 8, false>();
  }
}

bool pick_variant(const AttnArgs &a, Variant *v) {
  const int G = a.n_q_heads / a.n_kv_heads;
  if (a.v_is_k_prefix) {
    if (a.dtype != 1 || a.d_qk != 576 || a.d_v != 512 || a.paged) return false;
    if (G % 4 != 0 || G > 128) return false;
    *v = {warps_of<BF16, 576, 512, 4, true>(), 4};
    return true;
  }
  if (a.d_qk != a.d_v || (a.d_qk != 64 && a.d_qk != 128)) return false;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16 && G != 32 && G != 64) return false;
  const int hc = G < 8 ? G : 8;  // larger groups run as units of 8 heads
  int w;
  if (a.dtype == 1) w = a.d_qk == 128 ? gqa_warps<BF16, 128>(hc) : gqa_warps<BF16, 64>(hc);
  else w = a.d_qk == 128 ? gqa_warps<F32, 128>(hc) : gqa_warps<F32, 64>(hc);
  *v = {w, hc};
  return true;
}

template <typename E, int D, bool PAGED>
cudaError_t dispatch_gqa(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  switch (p.head_chunk) {
    case 1: return run_attention<E, D, D, 1, false, PAGED, kStages>(a, p, st);
    case 2: return run_attention<E, D, D, 2, false, PAGED, kStages>(a, p, st);
    case 4: return run_attention<E, D, D, 4, false, PAGED, kStages>(a, p, st);
    case 8: return run_attention<E, D, D, 8, false, PAGED, kStages>(a, p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

// Kernel choice.  bf16 GQA shapes run the warp-MMA kernel (tls_attn_mma.cu)
// and latent shapes with up to 64 heads per group the tcgen05 latent kernel
// (tls_attn_mla_tc.cu) by default.  TLS_ATTN_IMPL=cuda_core selects this
// file's CUDA-core kernel for both, TLS_ATTN_IMPL=tensor_core the tcgen05
// kernel for bf16 GQA (d = 128), TLS_ATTN_IMPL=warp_mma the warp-MMA latent
// kernel (tls_attn_mla.cu; 16, 32 or 64 heads).  The variable is read once
// per process.  fp32 shapes and other latent head counts always run the
// CUDA-core kernel.
enum ImplChoice { kImplDefault = 0, kImplCudaCore = 1, kImplTcgen05 = 2, kImplWarpMma = 3 };
static int impl_choice() {
  static int choice = -1;
  if (choice < 0) {
    const char *e = getenv("TLS_ATTN_IMPL");
    if (e && strcmp(e, "tensor_core") == 0) choice = kImplTcgen05;
    else if (e && strcmp(e, "cuda_core") == 0) choice = kImplCudaCore;
    else if (e && strcmp(e, "warp_mma") == 0) choice = kImplWarpMma;
    else choice = kImplDefault;
  }
  return choice;
}

bool attn_plan(const AttnArgs &a, AttnPlan *p) {
  const int choice = impl_choice();
  if (choice == kImplTcgen05 && attn_tc_supported(a)) {
    p->impl = 1;
    return attn_tc_plan(a, p);
  }
  const bool mla_tc = (choice == kImplDefault || choice == kImplTcgen05) && attn_mla_tc_supported(a);
  if (mla_tc || (choice == kImplWarpMma && attn_mla_supported(a))) {
    // latent attention on the tensor cores: a unit is a whole group (all G
    // heads), a piece is one CTA's contiguous range of tiles
    const int G = a.n_q_heads / a.n_kv_heads;
    const int tt = mla_tc ? attn_mla_tc_tokens_per_tile() : 16;
    p->impl = mla_tc ? 5 : 3;
    p->warps_per_cta = mla_tc ? 4 : 8;
    p->tokens_per_tile = tt;
    p->head_chunk = G;
    p->n_head_chunks = 1;
    const long long units = static_cast<long long>(a.batch) * a.n_kv_heads;
    p->tiles_per_group = (a.k_t + tt - 1) / tt;
    const long long total = units * p->tiles_per_group;
    if (total <= 0 || total > (1LL << 30)) return false;
    p->total_tiles = static_cast<int>(total);
    const int sms = a.num_sms > 0 ? a.num_sms : 148;
    const long long g0 = std::min<long long>(sms, total);
    p->tiles_per_warp = static_cast<int>((total + g0 - 1) / g0);
    p->grid = static_cast<int>((total + p->tiles_per_warp - 1) / p->tiles_per_warp);
    p->max_pieces = (p->tiles_per_group + p->tiles_per_warp - 1) / p->tiles_per_warp + 1;
    p->part_floats = static_cast<size_t>(units) * p->max_pieces * G * (2 + a.d_v);
    return true;
  }
  const bool mma = choice == kImplDefault && attn_mma_supported(a);
  p->impl = mma ? 2 : 0;
  Variant v;
  if (!pick_variant(a, &v)) return false;
  if (mma) {
    v.warps = attn_mma_warps(a);
    v.head_chunk = attn_mma_head_chunk(a);
  }
  const int G = a.n_q_heads / a.n_kv_heads;
  p->warps_per_cta = v.warps;
  p->tokens_per_tile = kTT;
  p->head_chunk = v.head_chunk;
  p->n_head_chunks = G / v.head_chunk;
  const long long units = static_cast<long long>(a.batch) * a.n_kv_heads * p->n_head_chunks;
  p->tiles_per_group = (a.k_t + kTT - 1) / kTT;
  const long long total = units * p->tiles_per_group;
  if (total <= 0 || total > (1LL << 30)) return false;
  p->total_tiles = static_cast<int>(total);
  const int sms = a.num_sms > 0 ? a.num_sms : 148;
  p->grid = static_cast<int>(std::min<long long>(sms, (total + v.warps - 1) / v.warps));
  const long long nw = static_cast<long long>(p->grid) * v.warps;
  p->tiles_per_warp = static_cast<int>((total + nw - 1) / nw);
  p->max_pieces = (p->tiles_per_group + p->tiles_per_warp - 1) / p->tiles_per_warp + 1;
  p->part_floats = static_cast<size_t>(units) * p->max_pieces * p->head_chunk * (2 + a.d_v);
  return true;
}

static cudaError_t launch_split(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  if (p.impl == 1) return launch_attention_tc(a, p, st);
  if (p.impl == 2) return launch_attention_mma(a, p, st);
  if (p.impl == 3) return launch_attention_mla(a, p, st);
  if (p.impl == 5) return launch_attention_mla_tc(a, p, st);
  if (a.v_is_k_prefix) return run_attention<BF16, 576, 512, 4, true, false, kStages>(a, p, st);
  if (a.dtype == 1) {
    if (a.d_qk == 128) return a.paged ? dispatch_gqa<BF16, 128, true>(a, p, st) : dispatch_gqa<BF16, 128, false>(a, p, st);
    return a.paged ? dispatch_gqa<BF16, 64, true>(a, p, st) : dispatch_gqa<BF16, 64, false>(a, p, st);
  }
  if (a.d_qk == 128) return a.paged ? dispatch_gqa<F32, 128, true>(a, p, st) : dispatch_gqa<F32, 128, false>(a, p, st);
  return a.paged ? dispatch_gqa<F32, 64, true>(a, p, st) : dispatch_gqa<F32, 64, false>(a, p, st);
}

cudaError_t launch_attention_merge(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  if (a.v_is_k_prefix) {
    if (p.impl == 3 || p.impl == 5) {
      switch (p.head_chunk) {
        case 1: return run_merge<512, 1>(a, p, st);
        case 2: return run_merge<512, 2>(a, p, st);
        case 4: return run_merge<512, 4>(a, p, st);
        case 8: return run_merge<512, 8>(a, p, st);
        case 16: return run_merge<512, 16>(a, p, st);
        case 32: return run_merge<512, 32>(a, p, st);
        case 64: return run_merge<512, 64>(a, p, st);
      }
      return cudaErrorInvalidValue;
    }
    return run_merge<512, 4>(a, p, st);
  }
  const int dv = a.d_v;
  switch (p.head_chunk) {
    case 1: return dv == 128 ? run_merge<128, 1>(a, p, st) : run_merge<64, 1>(a, p, st);
    case 2: return dv == 128 ? run_merge<128, 2>(a, p, st) : run_merge<64, 2>(a, p, st);
    case 4: return dv == 128 ? run_merge<128, 4>(a, p, st) : run_merge<64, 4>(a, p, st);
    case 8: return dv == 128 ? run_merge<128, 8>(a, p, st) : run_merge<64, 8>(a, p, st);
    case 16: return dv == 128 ? run_merge<128, 16>(a, p, st) : run_merge<64, 16>(a, p, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attention(const AttnArgs &a, const AttnPlan &p, cudaStream_t st) {
  cudaError_t e = launch_split(a, p, st);
  if (e != cudaSuccess) return e;
  return launch_attention_merge(a, p, st);
}

}  // namespace tls
