// Launcher of the paged prefill kernel (internal).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_common.cuh"

namespace pa {

struct PrefillArgs {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start;  // [batch + 1]
  const void* k_cache;         // pools (the tcgen05 kernel loads partial groups itself)
  const void* v_cache;
  int32_t* dev_error;
  int32_t batch, num_q_heads, num_kv_heads, group, head_dim, block_size;
  int32_t num_blocks, max_blocks, max_q;
  int32_t total_q;             // rows of q and out
  int32_t three_d;             // tile maps are {64, rows, head_dim / 64}
  float scale_log2;
};

// P . V keeps P as a head + tail pair only where one 16-bit value is too coarse.
template <typename T> struct PrefillPSplit { static constexpr bool value = true; };
template <> struct PrefillPSplit<__half> { static constexpr bool value = false; };

// mma.sync kernel: fp16 / bf16, head_dim 64 or 128, 64 % group == 0, block_size
// a multiple of 16.
cudaError_t launch_prefill(const PrefillArgs& a, pa_dtype dtype, const CUtensorMap& kmap,
                           const CUtensorMap& vmap, cudaStream_t stream);

// tcgen05 kernel: head_dim 128, 128 % group == 0, scale > 0, q 16-byte aligned;
// qmap is the {head_dim, num_q_heads, total_q} map of q with a {64, group, 128 /
// group} box, kmap2d / vmap2d are {head_dim, rows} maps of the pools with a
// {64, 16} box, all with the 128-byte swizzle.
cudaError_t launch_prefill_tc5(const PrefillArgs& a, pa_dtype dtype, const CUtensorMap& qmap,
                               const CUtensorMap& kmap2d, const CUtensorMap& vmap2d,
                               cudaStream_t stream);

}  // namespace pa
