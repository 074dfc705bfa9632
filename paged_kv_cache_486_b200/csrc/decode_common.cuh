// Work split and shared device helpers for paged decode attention.
//
// The unit of work is one KV block of one (sequence b, kv head) pair.  Units
// are numbered b-major, then kv head, then logical block j:
//     u = Hkv * cum[b] + kvh * nblk[b] + j,   cum[b] = sum_{b' < b} nblk[b'],
// nblk[b] = ceil(ctx[b] / block_size).  The units are cut into ranges:
//  * static ranges: the first Us units are split evenly over the W workers
//    (one warp each): range w = [floor(Us w / W), floor(Us (w + 1) / W));
//  * tail chunks: the last U - Us units (1/8 of them when there are at least
//    16 per worker) are cut into NC chunks of CH units that workers claim one
//    at a time, from a counter, when they run out of work.  An even split by
//    bytes is not an even split by time (memory latency differs from warp to
//    warp); the claimed tail evens out the finishing times.
// A run of units of one (b, kv head) inside one range is a "segment".  A
// segment that holds a whole (b, kv head) writes the output directly (single
// pass); otherwise it is a piece of a longer context: the worker stores the
// piece's (max, sum, unnormalised output) and the worker whose piece arrives
// last merges all of them with a log-sum-exp combine (piece_done below).  Only
// a range's first and last segments can be pieces, so each range owns two
// piece slots: slot 0 for the segment that contains the range's first unit,
// slot 1 for its last segment.
//
// Piece layout (fp32): m[G], l[G], o[G][D] where, for the piece's tokens j,
//   m = max_j t_j, l = sum_j 2^(t_j - m), o = sum_j 2^(t_j - m) v_j,
//   t_j = (q . k_j) * scale * log2(e)   (scores in base-2 units).
//
// Workspace words that must start at zero (the chunk counter, the finished-
// worker counter and one arrival count per (b, kv head)) are returned to zero
// by every call that completes, so a workspace zero-filled once stays usable.
#pragma once
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "pa.h"

namespace pa {

constexpr int kMaxBatch = 4096;
constexpr int kMaxWorkers = 2048;
constexpr int kPieceHeadBudget = 16384;  // workers x G kept in the workspace
constexpr int kMaxArrivals = 262144;     // batch x kv heads (arrival words)
constexpr int kMaxKvHeads = 4096;        // kv heads per layer

struct DecodeArgs {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int32_t* dev_error;
  uint32_t* ws_ctrl;      // [0] next tail chunk, [1] workers finished
  uint32_t* ws_arrivals;  // [B * Hkv] pieces arrived
  float* ws_pieces;       // [2 * max_ranges][G * (D + 2)]
  int32_t batch, num_q_heads, num_kv_heads, group, head_dim, block_size;
  int32_t num_blocks, max_blocks;
  int32_t workers;        // workers launched (the split uses at most this many)
  float scale_log2;       // scale * log2(e)
  int32_t test_expire;    // tests of the failure path: every worker's first tile wait
                          // counts as run out (PA_DECODE_TEST_WAIT_EXPIRY)
};

// Ranges of the unit sequence (see the header comment).  Every range is non-empty.
struct Split {
  int64_t U, Us, W, CH, NC;
  __host__ __device__ int64_t start(int64_t r) const {
    return r < W ? (Us * r) / W : Us + (r - W) * CH;
  }
  __host__ __device__ int64_t end(int64_t r) const {
    const int64_t e = r + 1 < W ? (Us * (r + 1)) / W : Us + (r + 1 - W) * CH;
    return e < U ? e : U;
  }
  __host__ __device__ int64_t range_of(int64_t u) const {
    return u < Us ? ((u + 1) * W - 1) / Us : W + (u - Us) / CH;
  }
};

// Maximum number of ranges for `workers` workers (piece slots are 2 per range).
__host__ __device__ inline int64_t max_ranges(int64_t workers) { return workers + workers / 2 + 1; }

__host__ __device__ inline Split make_split(int64_t U, int64_t workers) {
  Split s;
  s.U = U;
  const int64_t T = U >= 16 * workers ? U / 8 : 0;
  s.Us = U - T;
  s.W = workers < s.Us ? workers : s.Us;
  if (T > 0) {
    const int64_t cap = s.W / 2 > 1 ? s.W / 2 : 1;
    s.CH = (T + cap - 1) / cap;
    s.NC = (T + s.CH - 1) / s.CH;
  } else {
    s.CH = 1;
    s.NC = 0;
  }
  return s;
}

// Waits for the grid this launch depends on (a no-op unless the decode was
// launched to overlap its prologue with the preceding kernel).
__device__ inline void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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
}

// Each CTA pulls a slice of the block table into L2, so that the first block
// ids the workers read after the context scan are L2 hits.
__device__ inline void prefetch_tables(const DecodeArgs& a) {
  const int64_t bytes = static_cast<int64_t>(a.batch) * a.max_blocks * 4;
  const int64_t lines = (bytes + 127) / 128;
  const char* base = reinterpret_cast<const char*>(a.block_tables);
  for (int64_t l = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; l < lines;
       l += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(base + l * 128));
  }
}

// Rows of sequences with an empty context are zero; CTA (b mod grid) writes them.
template <typename T>
__device__ inline void zero_empty_rows(const DecodeArgs& a, const int32_t* ctx_s) {
  const int per_row = a.num_q_heads * a.head_dim;
  for (int b = blockIdx.x; b < a.batch; b += gridDim.x) {
    if (ctx_s[b] != 0) continue;
    T* o = static_cast<T*>(a.out) + static_cast<int64_t>(b) * per_row;
    for (int i = threadIdx.x; i < per_row; i += blockDim.x) o[i] = T(0.f);
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

// ------------------------- merging split contexts --------------------------
// A worker that has written a piece of (b, kv head) counts it on the pair's
// arrival word; the warp whose piece completes the set merges all pieces:
//   M = max_p m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p,
// then returns the word to zero for the next call.

// Claims the next tail chunk (whole warp; lane 0 touches the counter).
__device__ inline int64_t claim_chunk(const DecodeArgs& a, int lane) {
  uint32_t c = 0;
  if (lane == 0) c = atomicAdd(&a.ws_ctrl[0], 1u);
  return __shfl_sync(0xffffffffu, c, 0);
}

// Whole warp, once it has claimed its last chunk: the last of the W workers
// to finish returns both counters to zero.
__device__ inline void worker_finished(const DecodeArgs& a, int64_t W, int lane) {
  if (lane == 0) {
    const uint32_t n = atomicAdd(&a.ws_ctrl[1], 1u) + 1u;
    if (n == static_cast<uint32_t>(W)) {
      a.ws_ctrl[0] = 0u;
      a.ws_ctrl[1] = 0u;
    }
  }
}

__device__ inline float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ inline float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T> struct Num;

// Whole warp, after its piece of (b, kvh) is stored.  cum: block prefix sums.
// The merge keeps many loads in flight: pass 1 spreads the pieces over the
// lanes and finds each head's max and sum in one round of loads; pass 2 gives
// every lane the columns d = lane + 32k of a few heads and walks the pieces two
// at a time, each round issuing all of their loads for the lane at once.
template <typename T, int D>
__device__ inline void piece_done(const DecodeArgs& a, const int32_t* cum, int b, int kvh,
                                  const Split& sp, int lane) {
  constexpr int PER = D / 32;
  constexpr int HG = 16 / PER;  // heads merged per pass (16 accumulators per lane)
  constexpr int PQ = 2;         // pieces loaded per round in pass 2
  const int Hkv = a.num_kv_heads, G = a.group;
  const int nblk = cum[b + 1] - cum[b];
  const int64_t u0 = static_cast<int64_t>(Hkv) * cum[b] + static_cast<int64_t>(kvh) * nblk;
  const int64_t rf = sp.range_of(u0);
  const int64_t rl = sp.range_of(u0 + nblk - 1);
  __syncwarp();
  __threadfence();  // this warp's piece is visible before it is counted
  __syncwarp();
  uint32_t n = 0;
  if (lane == 0) n = atomicAdd(&a.ws_arrivals[static_cast<int64_t>(b) * Hkv + kvh], 1u) + 1u;
  n = __shfl_sync(0xffffffffu, n, 0);
  const int np = static_cast<int>(rl - rf + 1);
  if (n != static_cast<uint32_t>(np)) return;
  __threadfence();  // every other piece is visible to this warp
  // only the first piece can sit in slot 1 (its range started before u0)
  const int first_slot = sp.start(rf) >= u0 ? 0 : 1;
  const int64_t wf = rf;
  const int pf = G * (D + 2);
  const float* base = a.ws_pieces + (wf * 2 + first_slot) * pf;  // piece 0
  const float* rest = a.ws_pieces + (wf + 1) * 2 * pf;            // piece p >= 1: rest + 2 pf (p - 1)
  auto piece = [&](int p) { return p == 0 ? base : rest + static_cast<int64_t>(2 * pf) * (p - 1); };
  T* out = static_cast<T*>(a.out) + (static_cast<int64_t>(b) * a.num_q_heads + kvh * G) * D;
  for (int h0 = 0; h0 < G; h0 += HG) {
    const int nh = G - h0 < HG ? G - h0 : HG;
    float M[HG], L[HG], O[HG][PER];
#pragma unroll
    for (int hh = 0; hh < HG; ++hh) {
      M[hh] = -INFINITY;
      L[hh] = 0.f;
#pragma unroll
      for (int k = 0; k < PER; ++k) O[hh][k] = 0.f;
    }
    // pass 1: (max, sum) of every head; one round of loads when np <= 32
    for (int p0 = 0; p0 < np; p0 += 32) {
      const int p = p0 + lane;
      float pm[HG], pl[HG];
#pragma unroll
      for (int hh = 0; hh < HG; ++hh) {
        const bool on = p < np && hh < nh;
        pm[hh] = on ? __ldcg(piece(p) + h0 + hh) : -INFINITY;
        pl[hh] = on ? __ldcg(piece(p) + G + h0 + hh) : 0.f;
      }
#pragma unroll
      for (int hh = 0; hh < HG; ++hh) {
        const float mx = fmaxf(M[hh], warp_max(pm[hh]));
        const float part = pl[hh] == 0.f ? 0.f : pl[hh] * exp2f(pm[hh] - mx);
        L[hh] = L[hh] * exp2f(M[hh] - mx) + warp_sum(part);
        M[hh] = mx;
      }
    }
    // pass 2: weighted sum of the pieces' outputs, PQ pieces per round of loads
    for (int p0 = 0; p0 < np; p0 += PQ) {
      float e[PQ][HG], v[PQ][HG][PER];
#pragma unroll
      for (int q = 0; q < PQ; ++q) {
        const bool in = p0 + q < np;
        const float* pc = piece(in ? p0 + q : 0);
#pragma unroll
        for (int hh = 0; hh < HG; ++hh) {
          const bool on = in && hh < nh;
          e[q][hh] = on ? __ldcg(pc + h0 + hh) : -INFINITY;
#pragma unroll
          for (int k = 0; k < PER; ++k)
            v[q][hh][k] = on ? __ldcg(pc + 2 * G + (h0 + hh) * D + lane + 32 * k) : 0.f;
        }
      }
#pragma unroll
      for (int q = 0; q < PQ; ++q) {
#pragma unroll
        for (int hh = 0; hh < HG; ++hh) {
          const float wgt = exp2f(e[q][hh] - M[hh]);
#pragma unroll
          for (int k = 0; k < PER; ++k) O[hh][k] = fmaf(wgt, v[q][hh][k], O[hh][k]);
        }
      }
    }
#pragma unroll
    for (int hh = 0; hh < HG; ++hh) {
      if (hh < nh) {
        const float inv = 1.f / L[hh];
#pragma unroll
        for (int k = 0; k < PER; ++k)
          out[(h0 + hh) * D + lane + 32 * k] = Num<T>::from_f(O[hh][k] * inv);
      }
    }
  }
  if (lane == 0) a.ws_arrivals[static_cast<int64_t>(b) * Hkv + kvh] = 0u;
}

// ------------------------------- dtypes ------------------------------------
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
