// Cache write into an INT8 KV cache.
//
// "KV Cache for intermediates..." / "The four solutions", KV-cache quantisation:
// store K and V in 8 bits (about half the bytes of fp16).  Scheme (this
// library's; the pages fix none): per (token, kv head), symmetric over
// head_dim, every step in IEEE fp32 so the integer decisions are reproducible:
//   amax = max_d |x_d|,  scale = amax / 127,
//   code_d = round-to-nearest-even(x_d / scale) clamped to [-127, 127]
// (a zero row has scale 0 and zero codes).  Key codes [NB, Hkv, bs, D], value
// codes transposed in groups of 16 tokens [NB, Hkv, bs / 16, D, 16] (one group
// is a contiguous D x 16 tile, and a decode lane's 4 value bytes are 4
// consecutive tokens), fp32 scales [NB, Hkv, bs] for each.
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_common.cuh"
#include "int8_launch.h"

namespace pa {

template <typename T, int D>
__global__ void __launch_bounds__(256) reshape_and_cache_int8_kernel(
    const T* __restrict__ key, const T* __restrict__ value, int8_t* k_codes, int8_t* v_codes,
    float* k_scales, float* v_scales, const int64_t* __restrict__ slots, int64_t items,
    int32_t num_kv_heads, int32_t block_size, int64_t num_slots, int32_t* dev_error) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t item = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (item >= items) return;
  const int64_t t = item / num_kv_heads;
  const int h = static_cast<int>(item - t * num_kv_heads);
  const int64_t slot = slots[t];
  if (slot < 0 || slot >= num_slots) {
    if (slot != -1 && lane == 0 && h == 0) report(dev_error, PA_DEVERR_BAD_SLOT);
    return;
  }
  const int64_t blk = slot / block_size, off = slot - blk * block_size;
  const int64_t tile = blk * num_kv_heads + h;
#pragma unroll
  for (int kind = 0; kind < 2; ++kind) {
    const T* src = (kind ? value : key) + (t * num_kv_heads + h) * D + lane * PER;
    float x[PER];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      x[i] = Num<T>::to_f(src[i]);
      amax = fmaxf(amax, fabsf(x[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float scale = __fdiv_rn(amax, 127.0f);
    uint32_t packed = 0;
    int8_t c[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      int v = 0;
      if (scale > 0.f) v = max(-127, min(127, __float2int_rn(__fdiv_rn(x[i], scale))));
      c[i] = static_cast<int8_t>(v);
      packed |= (static_cast<uint32_t>(v) & 0xffu) << (8 * i);
    }
    if (kind == 0) {
      int8_t* dst = k_codes + (tile * block_size + off) * D + lane * PER;
      if constexpr (PER == 4) {
        *reinterpret_cast<uint32_t*>(dst) = packed;
      } else {
#pragma unroll
        for (int i = 0; i < PER; ++i) dst[i] = c[i];
      }
      if (lane == 0) k_scales[tile * block_size + off] = scale;
    } else {
#pragma unroll
      for (int i = 0; i < PER; ++i)
        v_codes[((tile * (block_size / 16) + off / 16) * D + lane * PER + i) * 16 + off % 16] = c[i];
      if (lane == 0) v_scales[tile * block_size + off] = scale;
    }
  }
}

template <typename T, int D>
static cudaError_t launch_t(const Int8WriteArgs& a, cudaStream_t stream) {
  const int64_t items = static_cast<int64_t>(a.n_tokens) * a.num_kv_heads;
  const int64_t threads = items * 32;
  const int blocks = static_cast<int>((threads + 255) / 256);
  reshape_and_cache_int8_kernel<T, D><<<blocks, 256, 0, stream>>>(
      static_cast<const T*>(a.key), static_cast<const T*>(a.value), a.k_codes, a.v_codes,
      a.k_scales, a.v_scales, a.slots, items, a.num_kv_heads, a.block_size,
      static_cast<int64_t>(a.num_blocks) * a.block_size, a.dev_error);
  return cudaGetLastError();
}

cudaError_t launch_reshape_and_cache_int8(const Int8WriteArgs& a, pa_dtype dtype,
                                          cudaStream_t stream) {
  if (a.n_tokens == 0) return cudaSuccess;
  if (a.head_dim == 128) {
    if (dtype == PA_F16) return launch_t<__half, 128>(a, stream);
    if (dtype == PA_BF16) return launch_t<__nv_bfloat16, 128>(a, stream);
    return launch_t<float, 128>(a, stream);
  }
  if (dtype == PA_F16) return launch_t<__half, 64>(a, stream);
  if (dtype == PA_BF16) return launch_t<__nv_bfloat16, 64>(a, stream);
  return launch_t<float, 64>(a, stream);
}

}  // namespace pa
