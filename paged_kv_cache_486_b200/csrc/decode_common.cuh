// Work split and shared device helpers for paged decode attention.
//
// The unit of work is one KV block of one (sequence b, kv head) pair.  Units
// are numbered b-major, then kv head, then logical block j:
//     u = Hkv * cum[b] + kvh * nblk[b] + j,   cum[b] = sum_{b' < b} nblk[b'],
// nblk[b] = ceil(ctx[b] / block_size).  Worker w (one warp) takes the units
// [start(w), start(w + 1)) with start(w) = floor(U * w / W), so every worker
// gets the same number of KV bytes to within one block.  A run of units of
// one (b, kv head) inside one worker is a "segment".  A segment that holds a
// whole (b, kv head) writes the output directly (single pass); otherwise it is
// a piece of a longer context that a log-sum-exp combine merges.  Only a
// worker's first and last segments can be pieces, so each worker owns two
// piece slots: slot 0 for the segment that contains start(w), slot 1 for its
// last segment.
//
// Piece layout (fp32): m[G], l[G], o[G][D] where, for the piece's tokens j,
//   m = max_j t_j, l = sum_j 2^(t_j - m), o = sum_j 2^(t_j - m) v_j,
//   t_j = (q . k_j) * scale * log2(e)   (scores in base-2 units).
#pragma once
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "pa.h"

namespace pa {

constexpr int kMaxBatch = 4096;
constexpr int kMaxWorkers = 2048;
constexpr int kPieceHeadBudget = 16384;  // workers x G kept in the workspace

struct DecodeArgs {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int32_t* dev_error;
  int32_t* ws_cum;      // [B + 1] written by CTA 0
  float* ws_pieces;     // [2 * max_workers][G * (D + 2)]
  int32_t batch, num_q_heads, num_kv_heads, group, head_dim, block_size;
  int32_t num_blocks, max_blocks;
  int32_t workers;      // workers launched (the split uses min(workers, U))
  float scale_log2;     // scale * log2(e)
};

__host__ __device__ inline int64_t split_start(int64_t w, int64_t U, int64_t W) {
  return (U * w) / W;
}

// The worker whose range holds unit u (requires W <= U so no range is empty).
__host__ __device__ inline int64_t split_worker_of(int64_t u, int64_t U, int64_t W) {
  return ((u + 1) * W - 1) / U;
}

__device__ inline void report(int32_t* dev_error, int32_t bits) {
  if (dev_error) atomicOr(dev_error, bits);
}

// Block-wide prologue: clamp context lengths, count blocks and scan them into
// cum[0..B] (shared memory); ctx_s[b] keeps the clamped length.  Uses every
// thread of the block and ends with __syncthreads().
__device__ inline void scan_context(const DecodeArgs& a, int32_t* cum, int32_t* ctx_s) {
  __shared__ int32_t warp_tot[32];
  const int B = a.batch;
  const int nt = blockDim.x;
  const int per = (B + nt - 1) / nt;
  const int lo = threadIdx.x * per;
  const int hi = min(B, lo + per);
  const int64_t cap = static_cast<int64_t>(a.max_blocks) * a.block_size;
  int32_t local = 0;
  for (int b = lo; b < hi; ++b) {
    int32_t c = a.context_lens[b];
    if (c < 0 || c > cap) {
      if (blockIdx.x == 0) report(a.dev_error, PA_DEVERR_BAD_CTX);
      c = c < 0 ? 0 : static_cast<int32_t>(cap);
    }
    ctx_s[b] = c;
    local += (c + a.block_size - 1) / a.block_size;
  }
  // exclusive scan of `local` across the block
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = (nt + 31) >> 5;
    int32_t v = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane < nw) warp_tot[lane] = v;  // inclusive totals per warp
  }
  __syncthreads();
  int32_t run = (warp ? warp_tot[warp - 1] : 0) + incl - local;
  for (int b = lo; b < hi; ++b) {
    cum[b] = run;
    run += (ctx_s[b] + a.block_size - 1) / a.block_size;
  }
  if (threadIdx.x == nt - 1) cum[B] = run;
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int b = threadIdx.x; b <= B; b += nt) a.ws_cum[b] = cum[b];
  }
}

// Largest b with Hkv * cum[b] <= u (cum is non-decreasing, cum[0] = 0).
__device__ inline int find_seq(const int32_t* cum, int B, int64_t u, int Hkv) {
  int lo = 0, hi = B;  // answer in [lo, hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (static_cast<int64_t>(Hkv) * cum[mid] <= u) lo = mid; else hi = mid;
  }
  return lo;
}

// Position of a worker inside the unit sequence.
struct UnitCursor {
  int64_t u, u_end;
  int b, kvh, j, nblk;
};

__device__ inline void cursor_seek(UnitCursor& c, int64_t u, int64_t u_end, const int32_t* cum,
                                   int B, int Hkv) {
  c.u = u;
  c.u_end = u_end;
  if (u >= u_end) return;
  c.b = find_seq(cum, B, u, Hkv);
  // skip sequences with no blocks (their cum does not advance)
  while (cum[c.b + 1] == cum[c.b]) ++c.b;
  c.nblk = cum[c.b + 1] - cum[c.b];
  const int64_t rem = u - static_cast<int64_t>(Hkv) * cum[c.b];
  c.kvh = static_cast<int>(rem / c.nblk);
  c.j = static_cast<int>(rem % c.nblk);
}

__device__ inline void cursor_next(UnitCursor& c, const int32_t* cum, int Hkv) {
  ++c.u;
  if (c.u >= c.u_end) return;
  if (++c.j == c.nblk) {
    c.j = 0;
    if (++c.kvh == Hkv) {
      c.kvh = 0;
      do {
        ++c.b;
      } while (cum[c.b + 1] == cum[c.b]);
      c.nblk = cum[c.b + 1] - cum[c.b];
    }
  }
}

// ------------------------------- dtypes ------------------------------------
template <typename T> struct Num;
template <> struct Num<float> {
  __device__ static float to_f(float x) { return x; }
  __device__ static float from_f(float x) { return x; }
};
template <> struct Num<__half> {
  __device__ static float to_f(__half x) { return __half2float(x); }
  __device__ static __half from_f(float x) { return __float2half_rn(x); }
};
template <> struct Num<__nv_bfloat16> {
  __device__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

}  // namespace pa
