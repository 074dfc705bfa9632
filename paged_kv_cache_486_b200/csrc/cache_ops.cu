// Cache write (reshape_and_cache) and copy-on-write block copy (copy_blocks).
//
// Both are byte moves bound by launch latency (a decode step writes one token
// per sequence) or by HBM bandwidth (block copies).  Each thread moves 16-byte
// vectors; the copy kernel keeps several 16-byte loads in flight per thread
// before it stores them.
#include <cuda_runtime.h>

#include <cstdint>

#include "cache_ops.h"
#include "decode_common.cuh"

namespace pa {

// "KV Cache and PagedAttention: Why Your LLM Server Slows Down" / "What is the
// KV cache?": each new token's K and V are stored for reuse.  Token t's rows
// go to slot s = slot_mapping[t]: block s / bs, offset s % bs, in a cache laid
// out [num_blocks, Hkv, bs, D].  Slot -1 skips the token.
__global__ void reshape_and_cache_kernel(const uint4* __restrict__ key,
                                         const uint4* __restrict__ value, uint4* k_cache,
                                         uint4* v_cache, const int64_t* __restrict__ slots,
                                         int64_t total_chunks, int32_t row_chunks,
                                         int32_t num_kv_heads, int32_t block_size,
                                         int64_t num_slots, int32_t* dev_error) {
  // a decode launched to overlap its prologue with this kernel may start now; it
  // waits for this grid before it reads the cache
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int32_t token_chunks = row_chunks * num_kv_heads;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total_chunks;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / token_chunks;
    const int32_t r = static_cast<int32_t>(i - t * token_chunks);
    const int64_t slot = slots[t];
    if (slot < 0 || slot >= num_slots) {
      if (slot != -1 && r == 0) report(dev_error, PA_DEVERR_BAD_SLOT);
      continue;
    }
    const int32_t h = r / row_chunks;
    const int32_t c = r - h * row_chunks;
    const int64_t block = slot / block_size;
    const int64_t off = slot - block * block_size;
    const int64_t dst = ((block * num_kv_heads + h) * block_size + off) * row_chunks + c;
    const uint4 kv = key[i];
    const uint4 vv = value[i];
    k_cache[dst] = kv;
    v_cache[dst] = vv;
  }
}

// "KV Cache and PagedAttention: Why Your LLM Server Slows Down" / "How
// PagedAttention solves this": shared pages are copied before a write.  One CTA
// per (pair, layer, key-or-value) copies one whole block.
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(256) copy_blocks_kernel(const __grid_constant__ LayerPtrs ptrs,
                                                          const int32_t* __restrict__ pairs,
                                                          int32_t num_blocks, int64_t block_chunks,
                                                          int32_t* dev_error) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int32_t pair = blockIdx.x;
  const int32_t layer = blockIdx.y >> 1;
  const bool is_v = blockIdx.y & 1;
  const int32_t src = pairs[2 * pair];
  const int32_t dst = pairs[2 * pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) report(dev_error, PA_DEVERR_BAD_BLOCK);
    return;
  }
  uint4* base = static_cast<uint4*>(is_v ? ptrs.v[layer] : ptrs.k[layer]);
  const uint4* s = base + src * block_chunks;
  uint4* d = base + dst * block_chunks;
  const int64_t step = static_cast<int64_t>(blockDim.x) * kCopyUnroll;
  for (int64_t i0 = threadIdx.x; i0 < block_chunks; i0 += step) {
    uint4 buf[kCopyUnroll];
#pragma unroll
    for (int k = 0; k < kCopyUnroll; ++k) {
      const int64_t i = i0 + static_cast<int64_t>(k) * blockDim.x;
      if (i < block_chunks) buf[k] = s[i];
    }
#pragma unroll
    for (int k = 0; k < kCopyUnroll; ++k) {
      const int64_t i = i0 + static_cast<int64_t>(k) * blockDim.x;
      if (i < block_chunks) d[i] = buf[k];
    }
  }
}

// Block copy between two pools (device <-> pinned host memory, or device <->
// device): block pairs[i].to of the destination becomes a copy of block
// pairs[i].from of the source, for every layer, key and value.  Several 16-byte
// loads are kept in flight per thread so that reads across the host link
// (which cannot be posted like writes) overlap.
__global__ void __launch_bounds__(256) swap_blocks_kernel(const __grid_constant__ LayerPtrs dst,
                                                          const __grid_constant__ LayerPtrs src,
                                                          const int32_t* __restrict__ pairs,
                                                          int32_t src_blocks, int32_t dst_blocks,
                                                          int64_t block_chunks,
                                                          int32_t* dev_error) {
  const int32_t pair = blockIdx.x;
  const int32_t layer = blockIdx.y >> 1;
  const bool is_v = blockIdx.y & 1;
  const int32_t from = pairs[2 * pair];
  const int32_t to = pairs[2 * pair + 1];
  if (from < 0 || from >= src_blocks || to < 0 || to >= dst_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) report(dev_error, PA_DEVERR_BAD_BLOCK);
    return;
  }
  const uint4* s = static_cast<const uint4*>(is_v ? src.v[layer] : src.k[layer]) + from * block_chunks;
  uint4* d = static_cast<uint4*>(is_v ? dst.v[layer] : dst.k[layer]) + to * block_chunks;
  constexpr int kUnroll = 8;
  const int64_t step = static_cast<int64_t>(blockDim.x) * kUnroll;
  for (int64_t i0 = threadIdx.x; i0 < block_chunks; i0 += step) {
    uint4 buf[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int64_t i = i0 + static_cast<int64_t>(k) * blockDim.x;
      if (i < block_chunks) buf[k] = s[i];
    }
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int64_t i = i0 + static_cast<int64_t>(k) * blockDim.x;
      if (i < block_chunks) d[i] = buf[k];
    }
  }
}

cudaError_t launch_swap_blocks(const LayerPtrs& dst, const LayerPtrs& src, int32_t num_layers,
                               const int32_t* pairs, int32_t n_pairs, int32_t src_blocks,
                               int32_t dst_blocks, int64_t block_bytes, int32_t* dev_error,
                               cudaStream_t stream) {
  if (n_pairs == 0) return cudaSuccess;
  dim3 grid(n_pairs, 2 * num_layers);
  swap_blocks_kernel<<<grid, 256, 0, stream>>>(dst, src, pairs, src_blocks, dst_blocks,
                                               block_bytes / 16, dev_error);
  return cudaGetLastError();
}

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                     void* v_cache, const int64_t* slots, int32_t n_tokens,
                                     int32_t num_kv_heads, int32_t row_bytes, int32_t block_size,
                                     int32_t num_blocks, int32_t* dev_error, int sm_count,
                                     cudaStream_t stream) {
  const int32_t row_chunks = row_bytes / 16;
  const int64_t total = static_cast<int64_t>(n_tokens) * num_kv_heads * row_chunks;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int blocks = static_cast<int>(want < int64_t(sm_count) * 16 ? want : int64_t(sm_count) * 16);
  reshape_and_cache_kernel<<<blocks, threads, 0, stream>>>(
      static_cast<const uint4*>(key), static_cast<const uint4*>(value),
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), slots, total, row_chunks,
      num_kv_heads, block_size, static_cast<int64_t>(num_blocks) * block_size, dev_error);
  return cudaGetLastError();
}

cudaError_t launch_copy_blocks(const LayerPtrs& ptrs, int32_t num_layers, const int32_t* pairs,
                               int32_t n_pairs, int32_t num_blocks, int64_t block_bytes,
                               int32_t* dev_error, cudaStream_t stream) {
  if (n_pairs == 0 || num_layers == 0) return cudaSuccess;
  dim3 grid(n_pairs, 2 * num_layers);
  copy_blocks_kernel<<<grid, 256, 0, stream>>>(ptrs, pairs, num_blocks, block_bytes / 16,
                                               dev_error);
  return cudaGetLastError();
}

}  // namespace pa
