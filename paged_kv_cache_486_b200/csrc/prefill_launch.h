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
  int32_t tiles;               // work items of 256 query rows per (sequence, kv head)
                               // (tcgen05 kernels)
  uint64_t* sched;             // NULL or {next item, CTAs done}, zero between calls (tcgen05)
  int32_t pair_block;          // (one-SM tcgen05 kernel) items go longest first within
                               // blocks of this many (sequence, kv head) pairs
  float scale_log2;
};

// P . V keeps P as a head + tail pair only where one 16-bit value is too coarse.
template <typename T> struct PrefillPSplit { static constexpr bool value = true; };
template <> struct PrefillPSplit<__half> { static constexpr bool value = false; };

// mma.sync kernel: fp16 / bf16, head_dim 64 or 128, 64 % group == 0, block_size
// a multiple of 16.
cudaError_t launch_prefill(const PrefillArgs& a, pa_dtype dtype, const CUtensorMap& kmap,
                           const CUtensorMap& vmap, cudaStream_t stream);

// tcgen05 kernel (persistent, one CTA per SM): head_dim 128, 128 % group == 0,
// scale > 0, q and out 16-byte aligned; qmap is the {head_dim, num_q_heads,
// total_q} map of q with a {64, group, 128 / group} box, kmap2d the {head_dim,
// rows} map of the key pool with a {64, 16} box, vmap3d the {64, rows, 2} map of
// the value pool with a {64, 16, 2} box, all with the 128-byte swizzle.
cudaError_t launch_prefill_tc5(PrefillArgs a, pa_dtype dtype, const CUtensorMap& qmap,
                               const CUtensorMap& kmap2d, const CUtensorMap& vmap3d,
                               cudaStream_t stream);

// The same on pairs of SMs (cta_group::2, clusters of two CTAs, 256-row items):
// the shapes of launch_prefill_tc5, omap the map of out like qmap; kmap2d / vmap2d the {head_dim, rows} maps of
// the key / value pools with a {64, 16} box (each CTA loads half of every tile).
cudaError_t launch_prefill_pair(PrefillArgs a, pa_dtype dtype, const CUtensorMap& qmap,
                                const CUtensorMap& kmap2d, const CUtensorMap& vmap2d,
                                const CUtensorMap& omap, cudaStream_t stream);

}  // namespace pa
