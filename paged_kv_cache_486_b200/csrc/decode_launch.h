// Launchers for the decode kernels (internal).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "decode_common.cuh"

namespace pa {

// CUDA-core path: every dtype, head_dim 64 or 128, any group size.
// overlap: launch with programmatic stream serialisation, so the prologue (which
// reads only context_lens, block_tables and q) runs while the preceding kernel
// finishes; the kernel waits for that kernel before touching anything else.
cudaError_t launch_decode_simt(const DecodeArgs& a, pa_dtype dtype, bool overlap,
                               cudaStream_t stream);

// Tensor-core path: fp16 / bf16, head_dim 64 or 128, group <= 8, block_size a
// multiple of 16.  kmap / vmap describe the key / value pools (see
// make_tile_map in api.cu): three_d = maps {64, rows, head_dim / 64}, else
// {head_dim, rows}.
cudaError_t launch_decode_tc(const DecodeArgs& a, pa_dtype dtype, const CUtensorMap& kmap,
                             const CUtensorMap& vmap, bool three_d, int num_ctas, bool overlap,
                             cudaStream_t stream);
int decode_tc_workers_per_cta();
size_t decode_tc_smem_bytes(int head_dim, int batch);

}  // namespace pa
