// tls_offload.cu -- the incremental block transfer of the AsyncTLS offload
// engine (gist.science (de) section 2.B: asynchronous prefetch that exploits
// temporal locality, and "Inkrementelle Block-Uebertragung": only the
// difference between consecutive block selections crosses PCIe; (es) section
// 2.B "Transferencia Incremental").
//
// The full KV cache stays in pinned host memory, one block per contiguous
// range ([2][bs][d]: K rows then V rows).  The GPU holds a slot cache with a
// per-group slot table.  prefetch_diff_kernel (one CTA per group) evicts the
// resident blocks that neither the previous nor the next selection holds,
// assigns free slots (lowest first) to the blocks of the next selection that
// are not resident and writes a copy list; copy_blocks_kernel then reads each listed block from host memory
// over PCIe with 16-byte loads and writes it into its slot.  Both run on the
// caller's copy stream, so the transfer overlaps the attention of the current
// step on the compute stream.
#include "tls_device.cuh"
#include "tls_internal.h"

namespace tls {
namespace {

constexpr int kDiffThreads = 512;
constexpr int kMaxBitmapWords = 16384 / 32;
constexpr int kMaxSlots = 4096;

__global__ void fill_neg1_kernel(int32_t *p, size_t n) {
  grid_dependency_wait();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    p[i] = -1;
}

__global__ void __launch_bounds__(kDiffThreads) prefetch_diff_kernel(OffloadArgs a) {
  __shared__ uint32_t keep[kMaxBitmapWords];
  __shared__ int16_t free_list[kMaxSlots];
  __shared__ int sh[33];
  grid_dependency_wait();
  const int group = blockIdx.x;
  const int nbm = a.n_blocks_max;
  int32_t *sob = a.slot_of_block + static_cast<size_t>(group) * nbm;
  int32_t *bos = a.block_of_slot + static_cast<size_t>(group) * a.n_slots;
  const int32_t *next = a.next_block_idx + static_cast<size_t>(group) * a.k_b;
  for (int i = threadIdx.x; i < (nbm + 31) / 32; i += kDiffThreads) keep[i] = 0;
  __syncthreads();
  // blocks to keep resident: the previous selection (still being attended) and the next one
  for (int i = threadIdx.x; i < a.k_b; i += kDiffThreads) {
    const int bn = next[i];
    if (bn >= 0 && bn < nbm) atomicOr(&keep[bn >> 5], 1u << (bn & 31));
    if (a.prev_block_idx) {
      const int bp = a.prev_block_idx[static_cast<size_t>(group) * a.k_b + i];
      if (bp >= 0 && bp < nbm) atomicOr(&keep[bp >> 5], 1u << (bp & 31));
    }
  }
  __syncthreads();
  // 1. evict every other resident block (no transfer, the slot becomes free)
  for (int s = threadIdx.x; s < a.n_slots; s += kDiffThreads) {
    const int blk = bos[s];
    if (blk >= 0 && (blk >= nbm || !(keep[blk >> 5] & (1u << (blk & 31))))) {
      if (blk < nbm) sob[blk] = -1;
      bos[s] = -1;
    }
  }
  __syncthreads();
  // 2. free slots in ascending order (each thread scans a contiguous segment)
  int n_free;
  {
    const int E = (a.n_slots + kDiffThreads - 1) / kDiffThreads;
    const int s0 = min(static_cast<int>(threadIdx.x) * E, a.n_slots), s1 = min(s0 + E, a.n_slots);
    int cnt = 0;
    for (int s = s0; s < s1; ++s) cnt += (bos[s] < 0);
    int pos = block_excl_scan<kDiffThreads>(cnt, sh, n_free);
    for (int s = s0; s < s1; ++s)
      if (bos[s] < 0) free_list[pos++] = static_cast<int16_t>(s);
  }
  __syncthreads();
  // 3. blocks of the next selection that are not resident, in list order, get
  //    the free slots in ascending order
  const int E = (a.k_b + kDiffThreads - 1) / kDiffThreads;
  const int i0 = min(static_cast<int>(threadIdx.x) * E, a.k_b), i1 = min(i0 + E, a.k_b);
  int cnt = 0;
  for (int i = i0; i < i1; ++i) {
    const int blk = next[i];
    cnt += (blk >= 0 && blk < nbm && sob[blk] < 0);
  }
  int n_need;
  int pos = block_excl_scan<kDiffThreads>(cnt, sh, n_need);
  int32_t *jobs = a.jobs + static_cast<size_t>(group) * a.k_b * 2;
  for (int i = i0; i < i1; ++i) {
    const int blk = next[i];
    if (blk >= 0 && blk < nbm && sob[blk] < 0) {
      if (pos < n_free) {
        jobs[pos * 2] = blk;
        jobs[pos * 2 + 1] = free_list[pos];
      }
      ++pos;
    }
  }
  __syncthreads();
  // 4. commit the table updates (separate pass: step 3 read the table)
  const int n_new = min(n_need, n_free);
  for (int q = threadIdx.x; q < n_new; q += kDiffThreads) {
    const int blk = jobs[q * 2], slot = jobs[q * 2 + 1];
    sob[blk] = slot;
    bos[slot] = blk;
  }
  if (threadIdx.x == 0) a.n_new[group] = n_new;
}

// One CTA per (job, group); a job is one block of 2 * bs * d elements.
__global__ void __launch_bounds__(256) copy_blocks_kernel(OffloadArgs a, int block_bytes) {
  grid_dependency_wait();
  const int group = blockIdx.y, q = blockIdx.x;
  if (q >= a.n_new[group]) return;
  const int32_t *jobs = a.jobs + static_cast<size_t>(group) * a.k_b * 2;
  const int blk = jobs[q * 2], slot = jobs[q * 2 + 1];
  const unsigned char *src = static_cast<const unsigned char *>(a.host_kv) +
                             (static_cast<size_t>(group) * a.n_blocks_max + blk) * block_bytes;
  unsigned char *dst = static_cast<unsigned char *>(a.cache) + (static_cast<size_t>(group) * a.n_slots + slot) * block_bytes;
  const int n16 = block_bytes / 16;
  constexpr int U = 4;
  for (int base = threadIdx.x; base < n16; base += 256 * U) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * 256;
      if (i < n16) v[u] = *reinterpret_cast<const uint4 *>(src + static_cast<size_t>(i) * 16);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * 256;
      if (i < n16) *reinterpret_cast<uint4 *>(dst + static_cast<size_t>(i) * 16) = v[u];
    }
  }
}

}  // namespace

cudaError_t launch_offload_reset(const OffloadArgs &a, cudaStream_t st) {
  const size_t groups = static_cast<size_t>(a.batch) * a.n_kv_heads;
  cudaError_t e = launch_pdl(fill_neg1_kernel, dim3(256), dim3(256), 0, st, a.slot_of_block, groups * a.n_blocks_max);
  if (e != cudaSuccess) return e;
  return launch_pdl(fill_neg1_kernel, dim3(64), dim3(256), 0, st, a.block_of_slot, groups * a.n_slots);
}

cudaError_t launch_prefetch_diff(const OffloadArgs &a, cudaStream_t st) {
  const int groups = a.batch * a.n_kv_heads;
  cudaError_t e = launch_pdl(prefetch_diff_kernel, dim3(groups), dim3(kDiffThreads), 0, st, a);
  if (e != cudaSuccess) return e;
  const int block_bytes = 2 * a.block_size * a.d * (a.dtype == 1 ? 2 : 4);
  return launch_pdl(copy_blocks_kernel, dim3(a.k_b, groups), dim3(256), 0, st, a, block_bytes);
}

}  // namespace tls
