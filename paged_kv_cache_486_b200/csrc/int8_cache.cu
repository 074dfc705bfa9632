// Cache write into an INT8 cache (records described in int8_launch.h).
//
// "KV Cache for intermediates..." / "The four solutions", KV-cache quantisation:
// store K and V in 8 bits (about half the bytes of fp16).  Scheme (this
// library's; the pages fix none): per (token, kv head), symmetric over
// head_dim, every step in IEEE fp32 so the integer decisions are reproducible:
//   amax = max_d |x_d|,  scale = amax / 127,
//   code_d = round-to-nearest-even(x_d / scale) clamped to [-127, 127]
// (a zero row has scale 0 and zero codes).
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_common.cuh"
#include "int8_launch.h"

namespace pa {

// One warp per (token, kv head); lane l quantises head_dim 4l .. 4l+3.
template <typename T>
__global__ void __launch_bounds__(256) reshape_and_cache_int8_kernel(
    const T* __restrict__ key, const T* __restrict__ value, uint8_t* k_pool, uint8_t* v_pool,
    const int64_t* __restrict__ slots, int64_t items, int32_t num_kv_heads, int32_t block_size,
    int64_t num_slots, int32_t* dev_error) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int D = i8::kDim, PER = D / 32;
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
  const int64_t blk = slot / block_size;
  const int off = static_cast<int>(slot - blk * block_size);
  const int64_t rec = (blk * num_kv_heads + h) * (block_size / i8::kGroup) + off / i8::kGroup;
  const int gt = off % i8::kGroup;  // token within the record's group
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
    int c[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      c[i] = 0;
      if (scale > 0.f) c[i] = max(-127, min(127, __float2int_rn(__fdiv_rn(x[i], scale))));
      // stored offset-binary: the byte code + 128 (code XOR 0x80)
      packed |= ((static_cast<uint32_t>(c[i]) & 0xffu) ^ 0x80u) << (8 * i);
    }
    uint8_t* r = (kind ? v_pool : k_pool) + rec * i8::kRecordBytes;
    if (kind == 0) {
      // 4 consecutive codes stay inside one 16-byte chunk: one 32-bit store
      *reinterpret_cast<uint32_t*>(r + i8::key_byte(i8::key_line(gt), lane * PER)) = packed;
    } else {
#pragma unroll
      for (int i = 0; i < PER; ++i)
        r[(lane * PER + i) * i8::kGroup + gt] = static_cast<uint8_t>((c[i] & 0xff) ^ 0x80);
    }
    if (lane == 0) reinterpret_cast<float*>(r + i8::kCodeBytes)[gt] = scale;
  }
}

template <typename T>
static cudaError_t launch_t(const Int8WriteArgs& a, cudaStream_t stream) {
  const int64_t items = static_cast<int64_t>(a.n_tokens) * a.num_kv_heads;
  const int blocks = static_cast<int>((items * 32 + 255) / 256);
  reshape_and_cache_int8_kernel<T><<<blocks, 256, 0, stream>>>(
      static_cast<const T*>(a.key), static_cast<const T*>(a.value), a.k_pool, a.v_pool, a.slots,
      items, a.num_kv_heads, a.block_size, static_cast<int64_t>(a.num_blocks) * a.block_size,
      a.dev_error);
  return cudaGetLastError();
}

cudaError_t launch_reshape_and_cache_int8(const Int8WriteArgs& a, pa_dtype dtype,
                                          cudaStream_t stream) {
  if (a.n_tokens == 0) return cudaSuccess;
  if (dtype == PA_F16) return launch_t<__half>(a, stream);
  if (dtype == PA_BF16) return launch_t<__nv_bfloat16>(a, stream);
  return launch_t<float>(a, stream);
}

}  // namespace pa
