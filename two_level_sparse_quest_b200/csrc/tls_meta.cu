// tls_meta.cu -- set-up kernels: per-block channel max/min summary and the
// label-channel slab (AsyncTLS block summary "Max/Min der Keys", gist.science
// (de) section 2.A "Stufe 1"; label channels, (es) section 2.A.2).
//
// build_meta: one thread owns one 16-byte chunk of channels of one block and
// walks the block's valid tokens; a warp reads 512 contiguous bytes per token
// step.  The max / min of stored values is itself a stored value, so the
// summary is exact in the storage type.
// build_slab: one thread per (token, label channel); coalesced slab writes.
#include "tls_device.cuh"
#include "tls_internal.h"

namespace tls {
namespace {

template <typename E>
__global__ void __launch_bounds__(256) build_meta_kernel(MetaArgs a) {
  grid_dependency_wait();
  constexpr int EPC = E::kEPC;
  const int chunks = a.d / EPC;  // 16-byte chunks per key row
  const int group = blockIdx.y;  // b * H_kv + g
  const int b = group / a.n_kv_heads;
  const int seq = min(max(a.seq_lens[b], 0), a.max_ctx);
  const long long item = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int blk = static_cast<int>(item / chunks), c = static_cast<int>(item % chunks);
  if (blk >= a.n_blocks_max) return;
  const int t0 = blk * a.block_size, t1 = min(t0 + a.block_size, seq);
  if (t0 >= t1) return;  // no valid token: left untouched
  using S = typename E::storage;
  const S *K = static_cast<const S *>(a.K) + (static_cast<size_t>(group) * a.max_ctx) * a.d + c * EPC;
  float hi[EPC], lo[EPC];
#pragma unroll
  for (int e = 0; e < EPC; ++e) { hi[e] = -INFINITY; lo[e] = INFINITY; }
  for (int t = t0; t < t1; ++t) {
    uint4 v = ld_stream16(K + static_cast<size_t>(t) * a.d);
    float f[EPC];
    chunk_to_f32<E>(v, f);
#pragma unroll
    for (int e = 0; e < EPC; ++e) { hi[e] = fmaxf(hi[e], f[e]); lo[e] = fminf(lo[e], f[e]); }
  }
  S *m = static_cast<S *>(a.meta) + ((static_cast<size_t>(group) * a.n_blocks_max + blk) * 2) * a.d + c * EPC;
  S ho[EPC], lw[EPC];
#pragma unroll
  for (int e = 0; e < EPC; ++e) {
    if constexpr (sizeof(S) == 2) {
      ho[e] = static_cast<S>(__float_as_uint(hi[e]) >> 16);  // exact: the value came from a bf16
      lw[e] = static_cast<S>(__float_as_uint(lo[e]) >> 16);
    } else {
      ho[e] = hi[e];
      lw[e] = lo[e];
    }
  }
  *reinterpret_cast<uint4 *>(m) = *reinterpret_cast<const uint4 *>(ho);
  *reinterpret_cast<uint4 *>(m + a.d) = *reinterpret_cast<const uint4 *>(lw);
}

template <typename E>
__global__ void __launch_bounds__(256) build_slab_kernel(MetaArgs a) {
  grid_dependency_wait();
  using S = typename E::storage;
  const int group = blockIdx.y;
  const int b = group / a.n_kv_heads;
  const int seq = min(max(a.seq_lens[b], 0), a.max_ctx);
  const long long item = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int t = static_cast<int>(item / a.n_label), c = static_cast<int>(item % a.n_label);
  if (t >= seq) return;
  const int ch = a.label_idx[c];
  const S *K = static_cast<const S *>(a.K) + (static_cast<size_t>(group) * a.max_ctx + t) * a.d;
  S v = (ch >= 0 && ch < a.d) ? K[ch] : S(0);
  static_cast<S *>(a.slab)[(static_cast<size_t>(group) * a.max_ctx + t) * a.n_label + c] = v;
}

// int8 label slab, step 1: per (group, label channel) the largest |K| over the
// valid tokens, read off the block summary (max(|max|, |min|) of each valid
// block is the block's largest |K|: exact), then scale = that / 127 (IEEE
// division).  One CTA per group; thread i takes channel i % r.
__global__ void __launch_bounds__(256) label_scales_kernel(MetaArgs a, float *scales) {
  grid_dependency_wait();
  __shared__ uint32_t amax[64];  // non-negative floats order like their bit patterns
  const int group = blockIdx.x, r = a.n_label;
  const int seq = min(max(a.seq_lens[group / a.n_kv_heads], 0), a.max_ctx);
  const int nb = (seq + a.block_size - 1) / a.block_size;
  if (threadIdx.x < r) amax[threadIdx.x] = 0u;
  __syncthreads();
  const int c = threadIdx.x % r, lanes = blockDim.x / r;
  const int ch = a.label_idx[c];
  if (static_cast<int>(threadIdx.x) < lanes * r && ch >= 0 && ch < a.d) {
    const uint16_t *m = static_cast<const uint16_t *>(a.meta) + static_cast<size_t>(group) * a.n_blocks_max * 2 * a.d;
    float best = 0.f;
    for (int blk = threadIdx.x / r; blk < nb; blk += lanes) {
      const uint16_t *row = m + static_cast<size_t>(blk) * 2 * a.d;
      best = fmaxf(best, fmaxf(fabsf(bf16_lo(row[ch])), fabsf(bf16_lo(row[a.d + ch]))));
    }
    atomicMax(&amax[c], __float_as_uint(best));
  }
  __syncthreads();
  if (threadIdx.x < r) scales[static_cast<size_t>(group) * r + threadIdx.x] = __fdiv_rn(__uint_as_float(amax[threadIdx.x]), 127.0f);
}

// int8 label slab, step 2: code = round-half-even(K / scale) clamped to
// [-127, 127] (0 where the scale is 0), decided in fp32; rows t < seq only.
__global__ void __launch_bounds__(256) build_slab_q8_kernel(MetaArgs a, const float *scales) {
  grid_dependency_wait();
  const int group = blockIdx.y;
  const int seq = min(max(a.seq_lens[group / a.n_kv_heads], 0), a.max_ctx);
  const long long item = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int t = static_cast<int>(item / a.n_label), c = static_cast<int>(item % a.n_label);
  if (t >= seq) return;
  const int ch = a.label_idx[c];
  const float scale = scales[static_cast<size_t>(group) * a.n_label + c];
  int code = 0;
  if (scale > 0.f && ch >= 0 && ch < a.d) {
    const uint16_t v = static_cast<const uint16_t *>(a.K)[(static_cast<size_t>(group) * a.max_ctx + t) * a.d + ch];
    code = min(max(__float2int_rn(__fdiv_rn(bf16_lo(v), scale)), -127), 127);
  }
  static_cast<int8_t *>(a.slab)[(static_cast<size_t>(group) * a.max_ctx + t) * a.n_label + c] = static_cast<int8_t>(code);
}

// Append update: CTA (j, group) rebuilds the j-th block touched by the rows
// [old, new) of the group's sequence from the block's valid rows (max / min
// over the stored values: exact, so the result equals a rebuild at the new
// length) and writes the slab rows of the appended tokens in that block.
template <typename E>
__global__ void __launch_bounds__(128) append_tokens_kernel(AppendArgs a) {
  grid_dependency_wait();
  using S = typename E::storage;
  constexpr int EPC = E::kEPC;
  const MetaArgs &m = a.m;
  const int group = blockIdx.y;
  const int b = group / m.n_kv_heads;
  const int old_len = a.old_lens[b], new_len = a.new_lens[b];
  if (old_len < 0 || new_len < old_len || new_len > m.max_ctx || new_len - old_len > a.max_append) {
    if (blockIdx.x == 0 && threadIdx.x == 0 && a.err) atomicOr(a.err, kErrAppendRange);
    return;
  }
  if (new_len == old_len) return;
  const int bs = m.block_size;
  const int blk = old_len / bs + static_cast<int>(blockIdx.x);
  const int t0 = blk * bs;
  if (t0 >= new_len) return;
  const int t1 = min(t0 + bs, new_len);
  const S *K = static_cast<const S *>(m.K) + static_cast<size_t>(group) * m.max_ctx * m.d;
  // block summary: one thread per 16-byte chunk of the channels
  const int chunks = m.d / EPC;
  S *mo = static_cast<S *>(m.meta) + ((static_cast<size_t>(group) * m.n_blocks_max + blk) * 2) * m.d;
  for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
    float hi[EPC], lo[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) {
      hi[e] = -INFINITY;
      lo[e] = INFINITY;
    }
    for (int t = t0; t < t1; ++t) {
      uint4 v = ld_stream16(K + static_cast<size_t>(t) * m.d + c * EPC);
      float f[EPC];
      chunk_to_f32<E>(v, f);
#pragma unroll
      for (int e = 0; e < EPC; ++e) {
        hi[e] = fmaxf(hi[e], f[e]);
        lo[e] = fminf(lo[e], f[e]);
      }
    }
    S ho[EPC], lw[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) {
      if constexpr (sizeof(S) == 2) {
        ho[e] = static_cast<S>(__float_as_uint(hi[e]) >> 16);  // exact: the value came from a bf16
        lw[e] = static_cast<S>(__float_as_uint(lo[e]) >> 16);
      } else {
        ho[e] = hi[e];
        lw[e] = lo[e];
      }
    }
    *reinterpret_cast<uint4 *>(mo + c * EPC) = *reinterpret_cast<const uint4 *>(ho);
    *reinterpret_cast<uint4 *>(mo + m.d + c * EPC) = *reinterpret_cast<const uint4 *>(lw);
  }
  // label slab rows of the appended tokens in this block
  if (m.slab) {
    const int s0 = max(t0, old_len);
    S *slab = static_cast<S *>(m.slab) + static_cast<size_t>(group) * m.max_ctx * m.n_label;
    for (int i = threadIdx.x; i < (t1 - s0) * m.n_label; i += blockDim.x) {
      const int t = s0 + i / m.n_label, c = i % m.n_label;
      const int ch = m.label_idx[c];
      slab[static_cast<size_t>(t) * m.n_label + c] = (ch >= 0 && ch < m.d) ? K[static_cast<size_t>(t) * m.d + ch] : S(0);
    }
  }
}

}  // namespace

cudaError_t launch_append_tokens(const AppendArgs &a, cudaStream_t st) {
  const int nblk = (a.max_append + a.m.block_size - 1) / a.m.block_size + 1;  // blocks one range can touch
  dim3 grid(static_cast<unsigned>(nblk), a.m.batch * a.m.n_kv_heads);
  if (a.m.dtype == 1) return launch_pdl(append_tokens_kernel<BF16>, grid, dim3(128), 0, st, a);
  return launch_pdl(append_tokens_kernel<F32>, grid, dim3(128), 0, st, a);
}

cudaError_t launch_build_meta(const MetaArgs &a, cudaStream_t st) {
  const int epc = a.dtype == 1 ? BF16::kEPC : F32::kEPC;
  const long long items = static_cast<long long>(a.n_blocks_max) * (a.d / epc);
  dim3 grid(static_cast<unsigned>((items + 255) / 256), a.batch * a.n_kv_heads);
  if (a.dtype == 1) return launch_pdl(build_meta_kernel<BF16>, grid, dim3(256), 0, st, a);
  return launch_pdl(build_meta_kernel<F32>, grid, dim3(256), 0, st, a);
}

cudaError_t launch_build_slab(const MetaArgs &a, cudaStream_t st) {
  const long long items = static_cast<long long>(a.max_ctx) * a.n_label;
  dim3 grid(static_cast<unsigned>((items + 255) / 256), a.batch * a.n_kv_heads);
  if (a.dtype == 1) return launch_pdl(build_slab_kernel<BF16>, grid, dim3(256), 0, st, a);
  return launch_pdl(build_slab_kernel<F32>, grid, dim3(256), 0, st, a);
}

cudaError_t launch_label_scales(const MetaArgs &a, float *scales, cudaStream_t st) {
  if (a.dtype != 1 || a.n_label > 64 || 256 % a.n_label) return cudaErrorInvalidValue;
  return launch_pdl(label_scales_kernel, dim3(a.batch * a.n_kv_heads), dim3(256), 0, st, a, scales);
}

cudaError_t launch_build_slab_q8(const MetaArgs &a, const float *scales, cudaStream_t st) {
  if (a.dtype != 1) return cudaErrorInvalidValue;
  const long long items = static_cast<long long>(a.max_ctx) * a.n_label;
  dim3 grid(static_cast<unsigned>((items + 255) / 256), a.batch * a.n_kv_heads);
  return launch_pdl(build_slab_q8_kernel, grid, dim3(256), 0, st, a, scales);
}

}  // namespace tls
