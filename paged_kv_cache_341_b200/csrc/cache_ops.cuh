// Cache-maintenance kernels of one decode step (bit copies, HBM-bound).
//
// append_kernel: the new token's K/V row goes into its slot -- the write of a
//   token into the next position of its block ("PagedAttention Explained:
//   Managing KV Cache Efficiently", section "Implementing a Simplified Paged KV
//   Cache").  A cache row [Hkv][D] is contiguous and flat row index == slot, so
//   one CTA copies one row with 16-byte vector loads/stores.
// copy_kernel: copy-on-write of a shared block before a sequence writes into
//   it (krapton.com "How Paged Attention Works", step 4; agentechip.com "Shared
//   Prefix Caching").  A block is block_size contiguous rows; CTAs split each
//   block into 16 KB slices so even a handful of pairs spreads over many SMs.
#ifndef PAGEDATTN_CACHE_OPS_CUH
#define PAGEDATTN_CACHE_OPS_CUH

#include <cstdint>

#include "ptx.cuh"

namespace pa {

__global__ void __launch_bounds__(256) append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                                     const int64_t* __restrict__ slots, uint4* k_cache,
                                                     uint4* v_cache, int64_t num_slots, int row_vecs) {
  allow_dependent_launch();   // a following planner reads only the lengths: it may start now
  const int t = blockIdx.x;
  const int64_t slot = slots[t];
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (threadIdx.x == 0) set_device_error(DEVERR_BAD_SLOT);
    return;
  }
  const uint4* src = (blockIdx.y ? v_new : k_new) + static_cast<int64_t>(t) * row_vecs;
  uint4* dst = (blockIdx.y ? v_cache : k_cache) + slot * row_vecs;
  for (int i = threadIdx.x; i < row_vecs; i += blockDim.x) dst[i] = src[i];
}

constexpr int kCopySliceVecs = 1024;   // 16 KB per CTA slice

__global__ void __launch_bounds__(256) copy_kernel(uint4* k_cache, uint4* v_cache, const int32_t* __restrict__ pairs,
                                                   int num_blocks, int block_vecs) {
  const int pi = blockIdx.x;
  const int src = pairs[2 * pi];
  const int dst = pairs[2 * pi + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) set_device_error(DEVERR_BAD_PAIR);
    return;
  }
  uint4* cache = blockIdx.y ? v_cache : k_cache;
  const uint4* s = cache + static_cast<int64_t>(src) * block_vecs;
  uint4* d = cache + static_cast<int64_t>(dst) * block_vecs;
  const int begin = blockIdx.z * kCopySliceVecs;
  const int end = min(block_vecs, begin + kCopySliceVecs);
  for (int i = begin + threadIdx.x; i < end; i += blockDim.x) d[i] = s[i];
}

// Block-table maintenance between steps: write the entries a host reservation
// changed (a fresh block at a block boundary, or the copy of a shared block)
// into the device tables, instead of re-sending whole tables.  updates[i] =
// (row, column, block id); rows/columns outside the table are skipped and set
// the device error word.  The same launch copies the step's lengths into the
// device lengths (lens[i] = new_lens[i], i < num_lens) when lens is non-null.
__global__ void __launch_bounds__(256) table_update_kernel(int32_t* tables, int num_rows, int stride,
                                                           const int32_t* __restrict__ updates, int n,
                                                           int32_t* lens, const int32_t* __restrict__ new_lens,
                                                           int num_lens) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (lens != nullptr && i < num_lens) lens[i] = new_lens[i];
  if (i >= n) return;
  const int row = updates[3 * i], col = updates[3 * i + 1], val = updates[3 * i + 2];
  if (row < 0 || row >= num_rows || col < 0 || col >= stride) {
    set_device_error(DEVERR_BAD_SLOT);
    return;
  }
  tables[static_cast<int64_t>(row) * stride + col] = val;
}

// Read-bandwidth ceiling: every byte of a buffer read once with streaming
// (evict-first) 16-byte loads, four in flight per thread, XOR-folded so the
// loads cannot be dropped.  No writes apart from one word per warp.  The
// decode kernel's achieved bandwidth is compared against this as the
// practical ceiling of a read-only stream on the GPU at hand.
__global__ void __launch_bounds__(512, 4) read_stream_kernel(const uint4* __restrict__ p, int64_t n, uint32_t* sink) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  for (; i + 3 * stride < n; i += 4 * stride) {
    const uint4 a = __ldcs(p + i), b = __ldcs(p + i + stride), c = __ldcs(p + i + 2 * stride),
                d = __ldcs(p + i + 3 * stride);
    acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w ^ c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^ d.z ^ d.w;
  }
  for (; i < n; i += stride) {
    const uint4 a = __ldcs(p + i);
    acc ^= a.x ^ a.y ^ a.z ^ a.w;
  }
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

}  // namespace pa

#endif
