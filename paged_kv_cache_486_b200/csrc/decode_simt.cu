// Paged decode attention on CUDA cores (every dtype and head grouping).
//
// Each warp is one worker of the even split described in decode_common.cuh.
// Within a segment the warp walks the sequence's blocks through its block-table
// row; for each token the 32 lanes hold head_dim / 32 elements of the key and
// value rows (coalesced), reduce the dot products of up to 8 query heads with
// shuffles and keep an online softmax per head in fp32.  Query heads beyond 8
// per KV head are done in further passes over the same blocks.
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_common.cuh"
#include "decode_launch.h"

namespace pa {

constexpr int kSimtWarps = 8;

template <typename T, int D>
__global__ void __launch_bounds__(kSimtWarps * 32) decode_simt_kernel(DecodeArgs a) {
  extern __shared__ int32_t simt_smem[];
  int32_t* cum = simt_smem;
  int32_t* ctx_s = simt_smem + a.batch + 1;
  prefetch_tables(a);
  scan_context(a, cum, ctx_s);
  wait_prior_grid();  // the cache, the output and the workspace are touched only after this
  zero_empty_rows<T>(a, ctx_s);

  const int B = a.batch, Hkv = a.num_kv_heads, G = a.group, Hq = a.num_q_heads;
  const Split sp = make_split(static_cast<int64_t>(Hkv) * cum[B], a.workers);
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kSimtWarps + (threadIdx.x >> 5);
  if (w >= sp.W) return;

  constexpr int PER = D / 32;
  const T* q = static_cast<const T*>(a.q);
  const T* kc = static_cast<const T*>(a.k_cache);
  const T* vc = static_cast<const T*>(a.v_cache);
  T* out = static_cast<T*>(a.out);
  const int bs = a.block_size;
  const int piece_floats = G * (D + 2);

  // the worker's static range first, then tail chunks while any are left
  for (int64_t r = w;;) {
    UnitCursor c;
    cursor_seek(c, sp.start(r), sp.end(r), cum, B, Hkv);
    bool first_seg = true;
    while (c.u < c.u_end) {
      const int b = c.b, kvh = c.kvh, j0 = c.j;
      const int64_t left = c.u_end - c.u;
      const int seg = static_cast<int>(left < c.nblk - c.j ? left : c.nblk - c.j);
      const int j1 = j0 + seg;
      const bool complete = j0 == 0 && j1 == c.nblk;
      const int slot = first_seg ? 0 : 1;
      const int ctx = ctx_s[b];
      for (int hg = 0; hg < G; hg += 8) {
        const int nh = G - hg < 8 ? G - hg : 8;
        float qv[8][PER], o[8][PER], m[8], l[8];
#pragma unroll
        for (int hh = 0; hh < 8; ++hh) {
          m[hh] = -INFINITY;
          l[hh] = 0.f;
#pragma unroll
          for (int i = 0; i < PER; ++i) {
            o[hh][i] = 0.f;
            qv[hh][i] = hh < nh ? Num<T>::to_f(q[(static_cast<int64_t>(b) * Hq + kvh * G + hg + hh) *
                                                      D + lane + 32 * i])
                                : 0.f;
          }
        }
        for (int j = j0; j < j1; ++j) {
          const int32_t phys = a.block_tables[static_cast<int64_t>(b) * a.max_blocks + j];
          if (phys < 0 || phys >= a.num_blocks) {
            if (lane == 0) report(a.dev_error, PA_DEVERR_BAD_BLOCK);
            continue;
          }
          const int rem = ctx - j * bs;
          const int ntok = rem < bs ? rem : bs;
          const int64_t tile = ((static_cast<int64_t>(phys) * Hkv + kvh) * bs) * D;
          for (int t = 0; t < ntok; ++t) {
            float kr[PER], vr[PER];
#pragma unroll
            for (int i = 0; i < PER; ++i) {
              kr[i] = Num<T>::to_f(kc[tile + t * D + lane + 32 * i]);
              vr[i] = Num<T>::to_f(vc[tile + t * D + lane + 32 * i]);
            }
            float s[8];
#pragma unroll
            for (int hh = 0; hh < 8; ++hh) {
              float acc = 0.f;
#pragma unroll
              for (int i = 0; i < PER; ++i) acc = fmaf(qv[hh][i], kr[i], acc);
              s[hh] = acc;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
              for (int hh = 0; hh < 8; ++hh) s[hh] += __shfl_xor_sync(0xffffffffu, s[hh], off);
            }
#pragma unroll
            for (int hh = 0; hh < 8; ++hh) {
              const float t2 = s[hh] * a.scale_log2;
              const float mn = fmaxf(m[hh], t2);
              const float alpha = exp2f(m[hh] - mn);
              const float p = exp2f(t2 - mn);
              l[hh] = l[hh] * alpha + p;
#pragma unroll
              for (int i = 0; i < PER; ++i) o[hh][i] = fmaf(o[hh][i], alpha, p * vr[i]);
              m[hh] = mn;
            }
          }
        }
        if (complete) {
#pragma unroll
          for (int hh = 0; hh < 8; ++hh) {
            if (hh < nh) {
              const float inv = 1.f / l[hh];
              T* orow = out + (static_cast<int64_t>(b) * Hq + kvh * G + hg + hh) * D;
#pragma unroll
              for (int i = 0; i < PER; ++i) orow[lane + 32 * i] = Num<T>::from_f(o[hh][i] * inv);
            }
          }
        } else {
          float* piece = a.ws_pieces + (r * 2 + slot) * piece_floats;
#pragma unroll
          for (int hh = 0; hh < 8; ++hh) {
            if (hh < nh) {
              if (lane == 0) {
                piece[hg + hh] = m[hh];
                piece[G + hg + hh] = l[hh];
              }
#pragma unroll
              for (int i = 0; i < PER; ++i)
                piece[2 * G + (hg + hh) * D + lane + 32 * i] = o[hh][i];
            }
          }
        }
      }
      if (!complete) piece_done<T, D>(a, cum, b, kvh, sp, lane);
      first_seg = false;
      c.u += seg - 1;
      c.j = j1 - 1;
      cursor_next(c, cum, Hkv);
    }
    if (sp.NC == 0) break;
    const int64_t chunk = claim_chunk(a, lane);
    if (chunk >= sp.NC) break;
    r = sp.W + chunk;
  }
  worker_finished(a, sp.W, lane);
}

template <typename T, int D>
static cudaError_t launch_simt_t(const DecodeArgs& a, bool overlap, cudaStream_t stream) {
  const int ctas = (a.workers + kSimtWarps - 1) / kSimtWarps;
  const size_t smem = sizeof(int32_t) * (2 * a.batch + 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(kSimtWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = overlap ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_simt_kernel<T, D>, a);
}

cudaError_t launch_decode_simt(const DecodeArgs& a, pa_dtype dtype, bool overlap,
                               cudaStream_t stream) {
  if (a.head_dim == 64) {
    if (dtype == PA_F32) return launch_simt_t<float, 64>(a, overlap, stream);
    if (dtype == PA_F16) return launch_simt_t<__half, 64>(a, overlap, stream);
    return launch_simt_t<__nv_bfloat16, 64>(a, overlap, stream);
  }
  if (dtype == PA_F32) return launch_simt_t<float, 128>(a, overlap, stream);
  if (dtype == PA_F16) return launch_simt_t<__half, 128>(a, overlap, stream);
  return launch_simt_t<__nv_bfloat16, 128>(a, overlap, stream);
}

}  // namespace pa
