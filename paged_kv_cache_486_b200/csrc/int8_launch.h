// Launchers for the INT8 cache kernels (internal).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_common.cuh"

namespace pa {

struct Int8WriteArgs {
  const void* key;
  const void* value;
  int8_t* k_codes;
  int8_t* v_codes;
  float* k_scales;
  float* v_scales;
  const int64_t* slots;
  int32_t n_tokens, num_kv_heads, head_dim, block_size, num_blocks;
  int32_t* dev_error;
};

// head_dim 64 or 128, block_size a multiple of 16; key / value in `dtype`.
cudaError_t launch_reshape_and_cache_int8(const Int8WriteArgs& a, pa_dtype dtype,
                                          cudaStream_t stream);

// Tensor maps of an INT8 cache (see decode_int8.cu): k_lo / k_hi view the key
// codes as rows of 128 bytes grouped by 4 tokens (k_hi starts 2 rows later).
// Value tiles are contiguous and need no map.
struct Int8Maps {
  CUtensorMap k_lo, k_hi;
};

// fp16 / bf16 queries, head_dim 128, group <= 8, block_size a multiple of 16.
// a.k_cache / a.v_cache are the code pools, a.k_scales / a.v_scales the scales.
cudaError_t launch_decode_int8(const DecodeArgs& a, pa_dtype dtype, const Int8Maps& maps,
                               int num_ctas, bool overlap, cudaStream_t stream);
int decode_int8_workers_per_cta();

}  // namespace pa
