// INT8 cache records and the launchers of the INT8 kernels (internal).
//
// An INT8 cache is two pools per layer, keys and values, each
// [num_blocks, num_kv_heads, block_size / 16] records of kRecordBytes: one
// record per 16-token group of a (block, kv head), laid out as the decode
// kernel wants it in shared memory, so that one bulk copy moves it.
//  key record:   16 lines of 128 code bytes, then the 16 key scales (fp32).
//                Line L holds group token key_token(L); the 16-byte chunk c of
//                its codes (head_dim 16c .. 16c+15) sits at chunk position
//                c ^ (L mod 8) of the line, so eight lines read at one chunk
//                hit eight different bank groups.
//  value record: 128 rows of 16 code bytes (row d = head_dim d of tokens 0..15
//                of the group, in token order), then the 16 value scales.
// Codes are signed bytes; an element reads back as code * scale.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_common.cuh"

namespace pa {
namespace i8 {

constexpr int kGroup = 16;                           // tokens per record
constexpr int kDim = 128;                            // head_dim
constexpr int kCodeBytes = kGroup * kDim;            // 2048
constexpr int kRecordBytes = kCodeBytes + kGroup * 4;  // codes + fp32 scales

// Line of group token t in a key record: t = 4i + 2h + e lies on line 2i + e + 8h.
__host__ __device__ inline int key_line(int t) { return ((t >> 2) << 1) + (t & 1) + ((t & 2) << 2); }
// Token on line L (the inverse of key_line).
__host__ __device__ inline int key_token(int L) {
  return (((L & 7) >> 1) << 2) + (L & 1) + ((L >> 3) << 1);
}
// Byte of code d of the token on line L.
__host__ __device__ inline int key_byte(int L, int d) {
  return L * kDim + ((((d >> 4) ^ (L & 7))) << 4) + (d & 15);
}

}  // namespace i8

struct Int8WriteArgs {
  const void* key;
  const void* value;
  uint8_t* k_pool;
  uint8_t* v_pool;
  const int64_t* slots;
  int32_t n_tokens, num_kv_heads, block_size, num_blocks;
  int32_t* dev_error;
};

// head_dim 128, block_size a multiple of 16; key / value in `dtype`.
cudaError_t launch_reshape_and_cache_int8(const Int8WriteArgs& a, pa_dtype dtype,
                                          cudaStream_t stream);

// fp16 / bf16 queries, head_dim 128, group <= 8, block_size a multiple of 16.
// a.k_cache / a.v_cache are the key / value record pools.
cudaError_t launch_decode_int8(const DecodeArgs& a, pa_dtype dtype, int num_ctas, bool overlap,
                               cudaStream_t stream);
int decode_int8_workers_per_cta();

}  // namespace pa
