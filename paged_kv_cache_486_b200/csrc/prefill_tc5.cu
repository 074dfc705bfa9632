// Paged prefill on the 5th-generation tensor cores (tcgen05 / UMMA, TMEM).
//
// Same definition and row layout as prefill.cu (causal attention of each
// sequence's new tokens over its paged cache; a CTA owns rows = (new token,
// head of one kv head's group) pairs), head_dim 128, fp16 / bf16.
//
// Per CTA: 128 query rows and key tiles of 128 keys.
//   S = Q . K_tile^T   UMMA M=128 N=128, K=128 in 8 steps of 16 (Q and K from
//                      shared memory, 128-byte-swizzled K-major), fp32 in TMEM;
//   softmax            one thread per row reads its S row from TMEM (no
//                      shuffles), masks (causal), updates its running max
//                      lazily (rescale O only when the max moves by > 2^8),
//                      writes P as 16-bit values back to TMEM;
//   O += P . V_tile    UMMA with A = P from TMEM (K-major), B = V from shared
//                      memory (MN-major: head_dim contiguous), fp32 in TMEM.
// bf16 keeps P as a head + tail pair (two products), fp16 a single value.
// Warps: 0 loads K / V tiles (TMA, two stages), 1 allocates TMEM and issues
// every UMMA (one thread), 2..5 run the softmax and the epilogue (warp w reads
// TMEM lanes 32 (w mod 4) .. +31, which is its rows).  S is double buffered in
// TMEM, so the tensor core computes the next tile's scores while the softmax
// works on this one.  TMEM columns: S0 0..127, S1 128..255, P head 256..319,
// P tail 320..383, O 384..511.
//
// Shared memory (1024-byte aligned, every tile in 64-column blocks of rows of
// 128 bytes, 128-byte swizzle): Q 32 KB, K 2 x 32 KB, V 2 x 32 KB.  That keeps
// one CTA per SM, so the 512-column TMEM allocation never waits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_tc.cuh"
#include "prefill_launch.h"

namespace pa {
namespace t5 {

using tc::kFull;
constexpr int kRows = 128;   // query rows per CTA
constexpr int kKeys = 128;   // keys per tile
constexpr int kD = 128;
constexpr int kThreads = 192;
constexpr int kColBlock = kRows * 128;     // one 64-column block of 128 rows: 16 KB
constexpr int kTileBytes = 2 * kColBlock;  // 128 rows x 128 columns x 2 bytes
constexpr int kQOff = 0;
constexpr int kKOff = kTileBytes;                 // 2 stages
constexpr int kVOff = kKOff + 2 * kTileBytes;     // 2 stages
constexpr int kRing = kVOff + 2 * kTileBytes;     // 160 KB
constexpr int kSmem = 1024 + kRing + 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColP = 256, kColPT = 320, kColO = 384;
constexpr float kSlack = 8.f;

// ---- PTX wrappers ----
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  // start address >> 4 (bits 0..13), leading byte offset >> 4 (16..29), stride
  // byte offset >> 4 (32..45), version 1 (46..47), 128-byte swizzle (61..63)
  return static_cast<uint64_t>((addr >> 4) & 0x3fff) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3fff) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3fff) << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16 instruction descriptor: fp32 accumulator, A / B in fp16 (0) or
// bf16 (1), A K-major, B K-major (0) or MN-major (1), N = 128, M = 128.
__host__ __device__ constexpr uint32_t idesc(uint32_t ab_format, uint32_t b_major) {
  return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (b_major << 16) |
         ((kKeys >> 3) << 17) | ((kRows >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(id), "r"(accumulate), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t id,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b), "r"(id), "r"(accumulate), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(bar) : "memory");
}

__device__ __forceinline__ void fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive columns of this thread's lane, not yet waited for.
__device__ __forceinline__ void tmem_ld32_issue(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

// Waits for this thread's outstanding TMEM loads; the registers are operands so
// that no use of them is scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
        "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]),
        "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
        "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]),
        "+r"(r[31])
      :
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32_issue(taddr, r);
  tmem_ld_wait(r);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
        "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
        "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Byte offset of 16-byte chunk c (0..15) of row r in a tile (64-column blocks
// of 128 rows x 128 bytes, 128-byte swizzle).
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
  return (c >> 3) * kColBlock + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc5_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + kRing);
  // barriers: kv_full[2], kv_empty[2], s_full[2], p_full, o_done, q_ready, mma_final
  const uint32_t b_kv_full = tc::smem_u32(&bars[0]);
  const uint32_t b_kv_empty = tc::smem_u32(&bars[2]);
  const uint32_t b_s_full = tc::smem_u32(&bars[4]);
  const uint32_t b_p_full = tc::smem_u32(&bars[6]);
  const uint32_t b_o_done = tc::smem_u32(&bars[7]);
  const uint32_t b_q_ready = tc::smem_u32(&bars[8]);
  const uint32_t b_final = tc::smem_u32(&bars[9]);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(bars + 11);

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
  const int r0 = tile_q * kRows;
  if (r0 >= rows) return;
  const int past = ctx - nq;
  const int n_keys = past + (min(r0 + kRows, rows) - 1) / G + 1;
  const int n_tiles = (n_keys + kKeys - 1) / kKeys;
  const int bs = a.block_size;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kAB = PrefillPSplit<T>::value ? 1u : 0u;  // operand format: bf16 1, fp16 0
  constexpr uint32_t kIdS = idesc(kAB, 0), kIdO = idesc(kAB, 1);

  if (threadIdx.x == 0) {
    tc::mbar_init(b_kv_full, 1);
    tc::mbar_init(b_kv_full + 8, 1);
    tc::mbar_init(b_kv_empty, 1);
    tc::mbar_init(b_kv_empty + 8, 1);
    tc::mbar_init(b_s_full, 1);
    tc::mbar_init(b_s_full + 8, 1);
    tc::mbar_init(b_p_full, 4);
    tc::mbar_init(b_o_done, 1);
    tc::mbar_init(b_q_ready, 4);
    tc::mbar_init(b_final, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&kmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(tc::smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ============================ K / V producer ============================
    for (int t = 0; t < n_tiles && !*abort_flag; ++t) {
      const int stage = t & 1;
      if (t >= 2 && !__all_sync(kFull, tc::mbar_wait_bounded(b_kv_empty + 8 * stage,
                                                             ((t >> 1) - 1) & 1))) {
        if (lane == 0) {
          report(a.dev_error, PA_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      const uint32_t kt = base + kKOff + stage * kTileBytes;
      const uint32_t vt = base + kVOff + stage * kTileBytes;
      // 16-key groups: whole and in a valid block -> TMA; partial (the one
      // holding key n_keys - 1) -> loaded here with the rows past it zeroed;
      // past n_keys or in an invalid block -> V rows zeroed (P is 0 there).
      int tma_groups = 0;
      for (int k = 0; k < kKeys / 16; ++k) {
        const int key = t * kKeys + k * 16;
        bool tma = false;
        int id = -1;
        if (key < n_keys) {
          id = __ldg(&a.block_tables[static_cast<int64_t>(b) * a.max_blocks + key / bs]);
          if (id < 0 || id >= a.num_blocks) {
            if (lane == 0) report(a.dev_error, PA_DEVERR_BAD_BLOCK);
            id = -1;
          }
          tma = id >= 0 && key + 16 <= n_keys;
        }
        if (tma) {
          ++tma_groups;
          continue;
        }
        // this group by hand: 16 rows x 16 chunks per tensor, 32 lanes
        const int valid = id >= 0 ? n_keys - key : 0;  // rows of the group to load
        const T* ks = nullptr;
        const T* vs = nullptr;
        if (id >= 0) {
          const int64_t row0 =
              (static_cast<int64_t>(id) * a.num_kv_heads + g) * bs + (key % bs);
          ks = static_cast<const T*>(a.k_cache) + row0 * kD;
          vs = static_cast<const T*>(a.v_cache) + row0 * kD;
        }
        for (int i = lane; i < 16 * 16; i += 32) {
          const int rr = i >> 4, c = i & 15;
          uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
          if (rr < valid) {
            kv = __ldg(reinterpret_cast<const uint4*>(ks + rr * kD) + c);
            vv = __ldg(reinterpret_cast<const uint4*>(vs + rr * kD) + c);
          }
          const uint32_t off = tile_off(k * 16 + rr, c);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(kt + off), "r"(kv.x),
                       "r"(kv.y), "r"(kv.z), "r"(kv.w) : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(vt + off), "r"(vv.x),
                       "r"(vv.y), "r"(vv.z), "r"(vv.w) : "memory");
        }
      }
      // generic writes above are read by the tensor core (async proxy)
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        const uint32_t bar = b_kv_full + 8 * stage;
        if (tma_groups)
          tc::mbar_arrive_expect_tx(bar, tma_groups * 4 * (16 * 128));
        else
          tc::mbar_arrive(bar);
        for (int k = 0; k < kKeys / 16; ++k) {
          const int key = t * kKeys + k * 16;
          if (key >= n_keys || key + 16 > n_keys) continue;
          const int id = __ldg(&a.block_tables[static_cast<int64_t>(b) * a.max_blocks + key / bs]);
          if (id < 0 || id >= a.num_blocks) continue;
          const int row = (id * a.num_kv_heads + g) * bs + key % bs;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            asm volatile(
                "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                " [%0], [%1, {%2, %3}], [%4];" ::"r"(kt + h * kColBlock + k * 16 * 128),
                "l"(reinterpret_cast<uint64_t>(&kmap)), "r"(64 * h), "r"(row), "r"(bar)
                : "memory");
            asm volatile(
                "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                " [%0], [%1, {%2, %3}], [%4];" ::"r"(vt + h * kColBlock + k * 16 * 128),
                "l"(reinterpret_cast<uint64_t>(&vmap)), "r"(64 * h), "r"(row), "r"(bar)
                : "memory");
          }
        }
      }
    }
  } else if (warp == 1) {
    // ============================= UMMA issuer ==============================
    const bool leader = lane == 0;
    bool ok = __all_sync(kFull, tc::mbar_wait_bounded(b_q_ready, 0));
    const uint32_t q_s = base + kQOff;
    auto issue_s = [&](int t) {  // S[t & 1] = Q . K_t^T
      const uint32_t kt = base + kKOff + (t & 1) * kTileBytes;
      const uint32_t d = tmem + kColS + (t & 1) * kKeys;
#pragma unroll
      for (int s = 0; s < kD / 16; ++s) {
        const uint32_t off = (s >> 2) * kColBlock + (s & 3) * 32;
        mma_ss(d, smem_desc(q_s + off, 16, 1024), smem_desc(kt + off, 16, 1024), kIdS, s > 0);
      }
      commit(b_s_full + 8 * (t & 1));
    };
    if (ok && leader) fence_after();
    if (ok) {
      if (!__all_sync(kFull, tc::mbar_wait_bounded(b_kv_full, 0))) ok = false;
    }
    if (ok && leader) {
      fence_after();
      issue_s(0);
    }
    for (int t = 0; ok && t < n_tiles; ++t) {
      // the next tile's scores while the softmax works on this one
      if (t + 1 < n_tiles) {
        if (!__all_sync(kFull, tc::mbar_wait_bounded(b_kv_full + 8 * ((t + 1) & 1),
                                                     ((t + 1) >> 1) & 1))) {
          ok = false;
          break;
        }
        if (leader) {
          fence_after();
          issue_s(t + 1);
        }
      }
      // O += P_t . V_t once the softmax has written P_t
      if (!__all_sync(kFull, tc::mbar_wait_bounded(b_p_full, t & 1))) {
        ok = false;
        break;
      }
      if (leader) {
        fence_after();
        const uint32_t vt = base + kVOff + (t & 1) * kTileBytes;
#pragma unroll
        for (int s = 0; s < kKeys / 16; ++s) {
          const uint64_t bd = smem_desc(vt + s * 16 * 128, kColBlock, 1024);
          mma_ts(tmem + kColO, tmem + kColP + 8 * s, bd, kIdO, (t > 0 || s > 0) ? 1u : 0u);
          if (PrefillPSplit<T>::value) mma_ts(tmem + kColO, tmem + kColPT + 8 * s, bd, kIdO, 1u);
        }
        commit(b_kv_empty + 8 * (t & 1));  // K_t / V_t may be refilled
        commit(b_o_done);                  // O (and P) are free again
      }
    }
    if (!ok && lane == 0) {
      report(a.dev_error, PA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    // every UMMA this thread issued has completed before TMEM is released
    if (leader) commit(b_final);
    __syncwarp();
    tc::mbar_wait_bounded(b_final, 0);
  } else {
    // ======================= softmax and epilogue ===========================
    const int sw = warp - 2;                 // 0..3
    const int quarter = warp & 3;            // TMEM lanes 32 quarter .. +31
    const int r = 32 * quarter + lane;       // this thread's row of the CTA
    const int grow = r0 + r;
    const bool valid = grow < rows;
    const int tok = valid ? grow / G : 0;
    const int hh = valid ? grow - tok * G : 0;
    const int pos = valid ? past + tok : -1;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
    // Q row into shared memory (swizzled), zeros past the rows
    {
      const T* qr = static_cast<const T*>(a.q) +
                    (static_cast<int64_t>(q0 + tok) * a.num_q_heads + g * G + hh) * kD;
      for (int c = 0; c < 16; ++c) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (valid) v = __ldg(reinterpret_cast<const uint4*>(qr) + c);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                     ::"r"(base + kQOff + tile_off(r, c)), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                     : "memory");
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(b_q_ready);
    }
    (void)sw;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      if (!__all_sync(kFull, tc::mbar_wait_bounded(b_s_full + 8 * (t & 1), (t >> 1) & 1))) {
        ok = false;
        break;
      }
      fence_after();
      const uint32_t srow = trow + kColS + (t & 1) * kKeys;
      // pass 1: this row's maximum over the tile (masked)
      float mx = -INFINITY;
      uint32_t su[4][32];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_ld32_issue(srow + 32 * ch, su[ch]);
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_ld_wait(su[ch]);  // the first waits for all four
      float sv[4][32];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int j = t * kKeys + 32 * ch + i;
          float v = __uint_as_float(su[ch][i]) * a.scale_log2;
          if (j > pos) v = -INFINITY;
          sv[ch][i] = v;
          mx = fmaxf(mx, v);
        }
      }
      // P must not be overwritten before the previous P . V has read it
      if (t > 0 && !__all_sync(kFull, tc::mbar_wait_bounded(b_o_done, (t - 1) & 1))) {
        ok = false;
        break;
      }
      fence_after();
      // a row whose maximum rose by more than 2^kSlack takes it as its new
      // reference and rescales its row of O (after the previous P . V).  TMEM
      // loads and stores are warp-collective, so the warp does this together;
      // rows that keep their reference scale by 1.
      const bool moves = mx > m + kSlack;
      if (__any_sync(kFull, moves)) {
        const float mnew = moves ? mx : m;
        const float alpha = m == -INFINITY ? 0.f : exp2f(m - mnew);
        if (t > 0) {
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            float ov[32];
            tmem_ld32(trow + kColO + 32 * ch, ov);
            uint32_t ou[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) ou[i] = __float_as_uint(ov[i] * alpha);
            tmem_st32(trow + kColO + 32 * ch, ou);
          }
        }
        l *= alpha;
        m = mnew;
      }
      const float mref = m == -INFINITY ? 0.f : m;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t ph[16], pt[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = exp2f(sv[ch][2 * i] - mref);
          const float p1 = exp2f(sv[ch][2 * i + 1] - mref);
          l += p0 + p1;
          if (PrefillPSplit<T>::value)
            tc::split2<T>(p0, p1, ph[i], pt[i]);
          else
            ph[i] = pt[i] = tc::pack2<T>(p0, p1);
        }
        // 16 columns of packed pairs per 32 keys
        uint32_t buf[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          buf[i] = ph[i];
          buf[16 + i] = pt[i];
        }
        // head pairs -> P columns 16 ch .. +15, tail pairs -> P tail columns
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
            "%10, %11, %12, %13, %14, %15, %16};"
            ::"r"(trow + kColP + 16 * ch), "r"(buf[0]), "r"(buf[1]), "r"(buf[2]), "r"(buf[3]),
              "r"(buf[4]), "r"(buf[5]), "r"(buf[6]), "r"(buf[7]), "r"(buf[8]), "r"(buf[9]),
              "r"(buf[10]), "r"(buf[11]), "r"(buf[12]), "r"(buf[13]), "r"(buf[14]), "r"(buf[15])
            : "memory");
        if (PrefillPSplit<T>::value) {
          asm volatile(
              "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
              "%10, %11, %12, %13, %14, %15, %16};"
              ::"r"(trow + kColPT + 16 * ch), "r"(buf[16]), "r"(buf[17]), "r"(buf[18]),
                "r"(buf[19]), "r"(buf[20]), "r"(buf[21]), "r"(buf[22]), "r"(buf[23]),
                "r"(buf[24]), "r"(buf[25]), "r"(buf[26]), "r"(buf[27]), "r"(buf[28]),
                "r"(buf[29]), "r"(buf[30]), "r"(buf[31])
              : "memory");
        }
      }
      tmem_st_wait();
      fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(b_p_full);
    }
    // epilogue: O / l once the last P . V is done
    if (ok && __all_sync(kFull, tc::mbar_wait_bounded(b_o_done, (n_tiles - 1) & 1))) {
      fence_after();
      T* dst = static_cast<T*>(a.out) +
               (static_cast<int64_t>(q0 + tok) * a.num_q_heads + g * G + hh) * kD;
      const float inv = 1.f / l;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        float ov[32];
        tmem_ld32(trow + kColO + 32 * ch, ov);
        if (valid) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            reinterpret_cast<uint32_t*>(dst)[16 * ch + i] =
                tc::pack2<T>(ov[2 * i] * inv, ov[2 * i + 1] * inv);
        }
      }
    } else if (lane == 0) {
      report(a.dev_error, PA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
  }

  // every role is done: release TMEM (after the tensor core has finished)
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols) : "memory");
  }
}

template <typename T>
static cudaError_t launch_t(const PrefillArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                            int tiles, cudaStream_t stream) {
  auto kern = prefill_tc5_kernel<T>;
  static bool raised[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !raised[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) raised[dev] = true;
  }
  dim3 grid(tiles, a.num_kv_heads, a.batch);
  kern<<<grid, kThreads, kSmem, stream>>>(kmap, vmap, a);
  return cudaGetLastError();
}

}  // namespace t5

// 2-D maps {head_dim, rows} with a {64, 16} box, 128-byte swizzle: one 16-key
// group of one 64-column block per copy.
cudaError_t launch_prefill_tc5(const PrefillArgs& a, pa_dtype dtype, const CUtensorMap& kmap2d,
                               const CUtensorMap& vmap2d, cudaStream_t stream) {
  const int64_t tiles = (static_cast<int64_t>(a.max_q) * a.group + t5::kRows - 1) / t5::kRows;
  return dtype == PA_F16
             ? t5::launch_t<__half>(a, kmap2d, vmap2d, static_cast<int>(tiles), stream)
             : t5::launch_t<__nv_bfloat16>(a, kmap2d, vmap2d, static_cast<int>(tiles), stream);
}

}  // namespace pa
