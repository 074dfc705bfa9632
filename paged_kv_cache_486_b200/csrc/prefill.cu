// Paged prefill / chunked-prefill attention on tensor cores.
//
// "What is PagedAttention and what did it change in LLM serving" mentions the
// prompt phase served over the same paged cache; the pages print no formula.
// Reading: sequence b has n_b new tokens, the last n_b of its ctx_b cached
// tokens (their keys and values already written); new token i at position
// p = ctx_b - n_b + i attends causally to every token j <= p:
//   out[t, h] = sum_{j <= p} softmax_j(scale q[t, h] . K_b[j, g]) V_b[j, g],
// g = h / G.  n_b = ctx_b is a whole prompt, n_b < ctx_b a chunk on top of
// earlier context, n_b = 1 is decode.
//
// Shape of the work.  A CTA owns 64 query rows of one (sequence, kv head); a
// row is a (new token, head of the kv head's group) pair, row r = token r / G,
// head r mod G, so every 64-key K / V tile it loads serves all G heads.  Four
// warps own 16 rows each and run FlashAttention-style:
//   S[16 x 64] = Q[16 x D] . K_tile^T   (mma m16n8k16, K rows through ldmatrix)
//   online softmax per row in base-2 units (fp32),
//   O[16 x D] += P[16 x 64] . V_tile    (P straight from the S accumulators,
//                                        V through ldmatrix.trans)
// bf16 keeps P as a head + tail pair of bf16 values (two products), as decode
// does, so outputs that nearly cancel stay accurate.  Tiles are double
// buffered: thread 0 issues the next tile's TMA copies (one per 16-key group:
// a 16-row box of the pool, the same maps as decode) once all warps are done
// with the stage.  CTAs with later query tiles (more keys) are launched first.
//
// Roofline.  Tensor work: 4 * D * Hq * (sum over new tokens of keys attended)
// flops; K / V bytes: each (sequence, kv head)'s keys are read once from HBM
// and reused from L2 by its other query tiles.
#include "decode_tc.cuh"
#include "prefill_launch.h"

namespace pa {
namespace pf {

using tc::kFull;
constexpr int kBM = 64;      // query rows per CTA
constexpr int kBN = 64;      // keys per tile
constexpr int kGroupKeys = 16;
constexpr int kThreads = 128;

template <int D>
struct Geo {
  static constexpr int kGroupBytes = kGroupKeys * D * 2;   // one 16-key box
  static constexpr int kTileBytes = (kBN / kGroupKeys) * kGroupBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;       // K tile + V tile
  static constexpr int kSmem = 1024 + 2 * kStageBytes + 64;
};

// Byte address of 16-byte chunk c (0 .. D/8-1) of key kk (0 .. 63) of a tile:
// group kk / 16, column block c / 8 (64 columns), line kk mod 16, position
// (c mod 8) ^ (kk mod 8) (the 128-byte swizzle).
template <int D>
__device__ __forceinline__ uint32_t key_addr(uint32_t tile, int kk, int c) {
  return tile + (kk >> 4) * Geo<D>::kGroupBytes + (c >> 3) * (kGroupKeys * 128) +
         (kk & 15) * 128 + (((c & 7) ^ (kk & 7)) << 4);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2)
    prefill_kernel(const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, PrefillArgs a) {
  using Gm = Geo<D>;
  constexpr int KC = D / 16;   // k-steps of the first product
  constexpr int NT = D / 8;    // n-tiles of the second product
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t ring0 = (raw + 1023u) & ~1023u;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + (ring0 - raw) + 2 * Gm::kStageBytes);
  int32_t* loaded = reinterpret_cast<int32_t*>(bars + 2);  // per stage: bit k = group k loaded

  const int b = blockIdx.z, g = blockIdx.y;
  const int tile_q = gridDim.x - 1 - blockIdx.x;  // later query tiles first
  const int q0 = a.query_start[b];
  const int nq = a.query_start[b + 1] - q0;
  const int ctx = a.context_lens[b];
  const int G = a.group;
  if (nq <= 0) return;
  if (ctx < nq || ctx > a.max_blocks * a.block_size || nq > a.max_q || q0 < 0 ||
      q0 > a.total_q - nq) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && g == 0) report(a.dev_error, PA_DEVERR_BAD_CTX);
    return;
  }
  const int rows = nq * G;
  const int r0 = tile_q * kBM;
  if (r0 >= rows) return;
  const int past = ctx - nq;
  const int n_keys = past + (min(r0 + kBM, rows) - 1) / G + 1;  // keys any row of the CTA needs
  const int n_tiles = (n_keys + kBN - 1) / kBN;
  const int bs = a.block_size;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    tc::mbar_init(tc::smem_u32(&bars[0]), 1);
    tc::mbar_init(tc::smem_u32(&bars[1]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&kmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
  }
  __syncthreads();

  // Thread 0: the copies of key tile t into `stage` (groups past n_keys and
  // groups whose block id is out of range are not loaded).
  auto issue = [&](int t, int stage) {
    const uint32_t kt = ring0 + stage * Gm::kStageBytes;
    const uint32_t bar = tc::smem_u32(&bars[stage]);
    int ids[kBN / kGroupKeys];
    int mask = 0, n = 0;
    for (int k = 0; k < kBN / kGroupKeys; ++k) {
      const int key = t * kBN + k * kGroupKeys;
      ids[k] = -1;
      if (key >= n_keys) continue;
      const int id = __ldg(&a.block_tables[static_cast<int64_t>(b) * a.max_blocks + key / bs]);
      if (id < 0 || id >= a.num_blocks) {
        report(a.dev_error, PA_DEVERR_BAD_BLOCK);
        continue;
      }
      ids[k] = id;
      mask |= 1 << k;
      ++n;
    }
    loaded[stage] = mask;
    if (n == 0) {
      tc::mbar_arrive(bar);
      return;
    }
    tc::mbar_arrive_expect_tx(bar, n * 2 * Gm::kGroupBytes);
    for (int k = 0; k < kBN / kGroupKeys; ++k) {
      if (ids[k] < 0) continue;
      const int key = t * kBN + k * kGroupKeys;
      const int row = (ids[k] * a.num_kv_heads + g) * bs + key % bs;
      tc::tma_tile<D>(kt + k * Gm::kGroupBytes, &kmap, row, a.three_d != 0, bar);
      tc::tma_tile<D>(kt + Gm::kTileBytes + k * Gm::kGroupBytes, &vmap, row, a.three_d != 0, bar);
    }
  };
  if (tid == 0) {
    issue(0, 0);
    if (n_tiles > 1) issue(1, 1);
  }

  // ---- this warp's rows: lane (lg, lc) holds rows lg and lg + 8 ----
  const int lg = lane >> 2, lc = lane & 3;
  const int wr0 = r0 + warp * 16;
  int pos[2];           // position of each of the lane's rows (-1: no such row)
  const T* qrow[2];
  for (int i = 0; i < 2; ++i) {
    const int r = wr0 + lg + 8 * i;
    pos[i] = -1;
    qrow[i] = nullptr;
    if (r < rows) {
      const int tok = r / G, hh = r - tok * G;
      pos[i] = past + tok;
      qrow[i] = static_cast<const T*>(a.q) +
                (static_cast<int64_t>(q0 + tok) * a.num_q_heads + g * G + hh) * D;
    }
  }
  // Q as the A operand: a[ks] = {row lg: d 16ks+2lc,+1}, {row lg+8: same},
  //                             {row lg: d 16ks+8+2lc,+1}, {row lg+8: same}
  uint32_t qa[KC][4];
#pragma unroll
  for (int ks = 0; ks < KC; ++ks) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(qrow[i]);
      qa[ks][i] = qrow[i] ? __ldg(src + (16 * ks + 2 * lc) / 2) : 0u;
      qa[ks][2 + i] = qrow[i] ? __ldg(src + (16 * ks + 8 + 2 * lc) / 2) : 0u;
    }
  }
  float o[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  const int pos_min = pos[0] < 0 ? INT32_MAX : pos[0];  // row lg has the lane's smallest position

  bool timed_out = false;
  int t = 0;
  for (; t < n_tiles; ++t) {
    const int stage = t & 1;
    const uint32_t kt = ring0 + stage * Gm::kStageBytes, vt = kt + Gm::kTileBytes;
    const bool ok = tc::mbar_wait_bounded(tc::smem_u32(&bars[stage]), (t >> 1) & 1);
    if (__syncthreads_or(!ok)) {
      if (tid == 0) report(a.dev_error, PA_DEVERR_TIMEOUT);
      timed_out = true;
      break;
    }
    const int mask = loaded[stage];
    const int valid = min(kBN, n_keys - t * kBN);  // keys of this tile any row needs
    if (valid < kBN || mask != (1 << ((valid + kGroupKeys - 1) / kGroupKeys)) - 1) {
      // V rows that no row may use (past n_keys, or in a group not loaded) may
      // hold anything, even NaN: clear them before P . V
      for (int i = tid; i < kBN * (D / 8); i += kThreads) {
        const int kk = i / (D / 8), c = i - kk * (D / 8);
        if (kk >= valid || !((mask >> (kk >> 4)) & 1))
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(key_addr<D>(vt, kk, c)),
                       "r"(0u)
                       : "memory");
      }
      __syncthreads();
    }

    // ---- S = Q . K^T over the tile's 64 keys ----
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KC; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t r[4];
        const int kk = 16 * np + ((lane >> 4) & 1) * 8 + (lane & 7);
        tc::ldsm_x4(key_addr<D>(kt, kk, 2 * ks + ((lane >> 3) & 1)), r);
        const uint32_t b0[2] = {r[0], r[1]}, b1[2] = {r[2], r[3]};
        tc::mma16816<T>(s[2 * np], qa[ks], b0);
        tc::mma16816<T>(s[2 * np + 1], qa[ks], b1);
      }
    }
    // ---- mask, scale to base 2, online softmax ----
    const int key0 = t * kBN;
    const bool need_mask = key0 + kBN - 1 > pos_min || valid < kBN || mask != 0xf;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = s[n][e] * a.scale_log2;
        if (need_mask) {
          const int kk = 8 * n + 2 * lc + (e & 1);
          const int j = key0 + kk;
          if (j > pos[e >> 1] || !((mask >> (kk >> 4)) & 1)) v = -INFINITY;
        }
        s[n][e] = v;
      }
    }
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      mx[0] = fmaxf(mx[0], fmaxf(s[n][0], s[n][1]));
      mx[1] = fmaxf(mx[1], fmaxf(s[n][2], s[n][3]));
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(kFull, mx[i], 1));
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(kFull, mx[i], 2));
    }
    float mref[2], alpha[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float mn = fmaxf(m[i], mx[i]);
      alpha[i] = mn == -INFINITY ? 1.f : exp2f(m[i] - mn);  // m = -inf: nothing to rescale
      m[i] = mn;
      mref[i] = mn == -INFINITY ? 0.f : mn;
      l[i] *= alpha[i];
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      o[n][0] *= alpha[0];
      o[n][1] *= alpha[0];
      o[n][2] *= alpha[1];
      o[n][3] *= alpha[1];
    }
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      s[n][0] = exp2f(s[n][0] - mref[0]);
      s[n][1] = exp2f(s[n][1] - mref[0]);
      s[n][2] = exp2f(s[n][2] - mref[1]);
      s[n][3] = exp2f(s[n][3] - mref[1]);
      l[0] += s[n][0] + s[n][1];
      l[1] += s[n][2] + s[n][3];
    }
    // ---- O += P . V (P from the accumulators: keys 16kk .. 16kk+15) ----
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t ph[4], pt[4];
      tc::split2<T>(s[2 * kk][0], s[2 * kk][1], ph[0], pt[0]);
      tc::split2<T>(s[2 * kk][2], s[2 * kk][3], ph[1], pt[1]);
      tc::split2<T>(s[2 * kk + 1][0], s[2 * kk + 1][1], ph[2], pt[2]);
      tc::split2<T>(s[2 * kk + 1][2], s[2 * kk + 1][3], ph[3], pt[3]);
#pragma unroll
      for (int dp = 0; dp < NT / 2; ++dp) {
        uint32_t r[4];
        const int key = 16 * kk + ((lane >> 3) & 1) * 8 + (lane & 7);
        tc::ldsm_x4_trans(key_addr<D>(vt, key, 2 * dp + (lane >> 4)), r);
        const uint32_t b0[2] = {r[0], r[1]}, b1[2] = {r[2], r[3]};
        tc::mma16816<T>(o[2 * dp], ph, b0);
        tc::mma16816<T>(o[2 * dp + 1], ph, b1);
        if (PrefillPSplit<T>::value) {
          tc::mma16816<T>(o[2 * dp], pt, b0);
          tc::mma16816<T>(o[2 * dp + 1], pt, b1);
        }
      }
    }
    // every warp is done with this stage (and its generic writes are ordered
    // before the copies that refill it)
    tc::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0 && t + 2 < n_tiles) issue(t + 2, stage);
  }
  if (timed_out) {
    // let copies already in flight land before the CTA's shared memory goes away
    if (tid == 0) {
      for (int k = t; k < n_tiles && k < t + 2; ++k)
        tc::mbar_wait_bounded(tc::smem_u32(&bars[k & 1]), (k >> 1) & 1);
    }
    return;
  }
  // ---- normalise and store ----
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l[i] += __shfl_xor_sync(kFull, l[i], 1);
    l[i] += __shfl_xor_sync(kFull, l[i], 2);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    if (pos[i] < 0) continue;
    const int r = wr0 + lg + 8 * i;
    const int tok = r / G, hh = r - tok * G;
    T* dst = static_cast<T*>(a.out) +
             (static_cast<int64_t>(q0 + tok) * a.num_q_heads + g * G + hh) * D;
    const float inv = 1.f / l[i];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const uint32_t v = tc::pack2<T>(o[n][2 * i] * inv, o[n][2 * i + 1] * inv);
      *reinterpret_cast<uint32_t*>(dst + 8 * n + 2 * lc) = v;
    }
  }
}

template <typename T, int D>
static cudaError_t launch_t(const PrefillArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                            int tiles, cudaStream_t stream) {
  auto kern = prefill_kernel<T, D>;
  static bool raised[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !raised[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo<D>::kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) raised[dev] = true;
  }
  dim3 grid(tiles, a.num_kv_heads, a.batch);
  kern<<<grid, kThreads, Geo<D>::kSmem, stream>>>(kmap, vmap, a);
  return cudaGetLastError();
}

}  // namespace pf

cudaError_t launch_prefill(const PrefillArgs& a, pa_dtype dtype, const CUtensorMap& kmap,
                           const CUtensorMap& vmap, cudaStream_t stream) {
  const int64_t tiles = (static_cast<int64_t>(a.max_q) * a.group + pf::kBM - 1) / pf::kBM;
  if (a.head_dim == 128) {
    return dtype == PA_F16
               ? pf::launch_t<__half, 128>(a, kmap, vmap, static_cast<int>(tiles), stream)
               : pf::launch_t<__nv_bfloat16, 128>(a, kmap, vmap, static_cast<int>(tiles), stream);
  }
  return dtype == PA_F16
             ? pf::launch_t<__half, 64>(a, kmap, vmap, static_cast<int>(tiles), stream)
             : pf::launch_t<__nv_bfloat16, 64>(a, kmap, vmap, static_cast<int>(tiles), stream);
}

}  // namespace pa
