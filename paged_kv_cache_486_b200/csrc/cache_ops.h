// Launchers for the cache write and block copy kernels (internal).
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

namespace pa {

constexpr int kMaxLayers = 128;

struct LayerPtrs {
  void* k[kMaxLayers];
  void* v[kMaxLayers];
};

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                     void* v_cache, const int64_t* slots, int32_t n_tokens,
                                     int32_t num_kv_heads, int32_t row_bytes, int32_t block_size,
                                     int32_t num_blocks, int32_t* dev_error, int sm_count,
                                     cudaStream_t stream);

cudaError_t launch_copy_blocks(const LayerPtrs& ptrs, int32_t num_layers, const int32_t* pairs,
                               int32_t n_pairs, int32_t num_blocks, int64_t block_bytes,
                               int32_t* dev_error, cudaStream_t stream);

cudaError_t launch_swap_blocks(const LayerPtrs& dst, const LayerPtrs& src, int32_t num_layers,
                               const int32_t* pairs, int32_t n_pairs, int32_t src_blocks,
                               int32_t dst_blocks, int64_t block_bytes, int32_t* dev_error,
                               cudaStream_t stream);

}  // namespace pa
