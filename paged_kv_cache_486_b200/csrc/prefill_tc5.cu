// Paged prefill on the 5th-generation tensor cores (tcgen05 / UMMA, TMEM).
//
// Same definition and row layout as prefill.cu (causal attention of each
// sequence's new tokens over its paged cache; rows are (new token, head of one
// kv head's group) pairs of one sequence and kv head), head_dim 128, fp16 /
// bf16, scale > 0.
//
// A work item is 256 rows of one sequence and kv head, taken as two halves of
// 128 rows that share every key and value tile: each K / V tile of 128 keys is
// brought into shared memory once for both.  Each half runs on its own: its own
// issuing thread, its own four softmax warps, its output accumulator O_h and two
// score buffers in TMEM.  A half walks its keys in sub-tiles of 64:
//   S = Q_h . K_sub^T   UMMA M=128 N=64 (the half's last sub-tile: N rounded up
//                       to 16 past its keys), K=128 in 8 steps of 16, Q and K
//                       from shared memory (128-byte-swizzled, K-major), fp32 in
//                       TMEM, into the half's two score buffers in turn;
//   softmax             one thread per row reads its 64 scores from TMEM, masks
//                       (causal, diagonal sub-tiles only), keeps its running max
//                       lazily (O_h is rescaled only when the max rises by more
//                       than 2^8) and writes P as 16-bit values over its own
//                       score columns;
//   O_h += P . V_sub    UMMA M=128 N=128, K=64 in 4 steps, A = P from TMEM
//                       (K-major), B = V from shared memory (MN-major: head_dim
//                       contiguous), fp32 in TMEM.
// bf16 keeps P as a head + tail pair (two products), fp16 a single value.
// With two score buffers a half's next scores are computed while its softmax
// works on the current ones: a buffer takes new scores once the P . V that read
// its P two sub-tiles back has completed, so the softmax warps run from one
// sub-tile to the next without waiting for the tensor core.  The epilogue
// divides by the row sum and stores each row straight from registers (256
// contiguous bytes per row).
//
// Persistent when the caller gives a scheduling workspace: one CTA per SM takes
// items from a global counter.  The (sequence, kv head) pairs go in blocks whose
// keys and values fit in part of L2; within a block the longest items go first
// (so the kernel does not end on a long one) and the items reading the same keys
// and values run at about the same time, so those reach each SM from L2.  The K
// producer takes the items and passes them to the other roles through a
// four-slot ring in shared memory.  Without a workspace each CTA runs one item.
//
// Warps: 0 loads the K tiles (and takes the items), 2 the Q halves and the V
// tiles (TMA, each tensor with its own stages), 1 and 3 issue the S products of
// half 0 and half 1, 4 and 5 their P . V products (one thread each, so a P . V
// goes out as soon as its P is written, whatever the S side is doing; warp 1
// also allocates TMEM), 6 and 7 have no role, 8..11 run the softmax and
// epilogue of half 0, 12..15 of half 1 (warp w reads TMEM lanes
// 32 (w mod 4) .. +31, which are its rows).  TMEM columns: half h's score
// buffers at 128 h and 128 h + 64, O_0 256..383, O_1 384..511.
//
// Shared memory (1024-byte aligned, rows of 128 bytes with the 128-byte
// swizzle): Q 2 x 32 KB (one tile per half), K 3 x 32 KB, V 2 x 32 KB.  Q and K
// tiles are two 64-column blocks of 128 rows (the S product's K-major
// operands); a V tile is eight 16-key groups of two 64-column blocks of 16
// rows, so one 4 KB copy brings a group.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "decode_tc.cuh"
#include "prefill_launch.h"
#include "tc5_ptx.cuh"

namespace pa {
namespace t5 {

using tc::kFull;
constexpr int kRows = 128;   // query rows per half
constexpr int kKeys = 128;   // keys per K / V tile
constexpr int kSub = 64;     // keys per score sub-tile
constexpr int kD = 128;
constexpr int kThreads = 512;
constexpr int kKWarp = 0, kVWarp = 2;      // S issuers: warps 1, 3; P . V issuers: 4, 5
constexpr int kColBlock = kRows * 128;     // one 64-column block of 128 rows: 16 KB
constexpr int kTileBytes = 2 * kColBlock;  // 128 rows x 128 columns x 2 bytes
constexpr int kGroupBytes = 16 * 128;      // 16 rows of one 64-column block
constexpr int kKStages = 3;                // K tiles in flight
constexpr int kVStages = 2;                // V tiles in flight
constexpr int kQOff = 0;                   // Q of half 0, half 1
constexpr int kKOff = 2 * kTileBytes;
constexpr int kVOff = kKOff + kKStages * kTileBytes;
constexpr int kRing = kVOff + kVStages * kTileBytes;  // 224 KB
constexpr int kRingSlots = 4;              // items passed from the K producer to the others
constexpr int kItemReaders = 13;           // V / Q producer, four issuers, eight softmax warps
constexpr int kSmem = 1024 + kRing + 512;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 2 * kKeys;      // O_h at 256 + 128 h
constexpr float kSlack = 8.f;
constexpr long long kSpinLimit = 1ll << 31;  // clock cycles without progress
// Registers: the launch gives every thread kLaunchRegs; warpgroups 0 and 1 (the
// loaders and the issuers) give most of theirs up (setmaxnreg.dec), the two
// softmax warpgroups take them (setmaxnreg.inc).  The counts must add up to no
// more than the launch's total, or the increase would wait for good.
constexpr int kLaunchRegs = 128;
constexpr int kOtherRegs = 80;
constexpr int kSoftmaxRegs = 176;
static_assert(kThreads * kLaunchRegs <= 65536, "launch registers");
static_assert(256 * kOtherRegs + 256 * kSoftmaxRegs <= kThreads * kLaunchRegs, "register split");

// ---- PTX wrappers (the generic ones are in tc5_ptx.cuh) ----
// kind::f16 instruction descriptor: fp32 accumulator, A / B in fp16 (0) or
// bf16 (1), A K-major, B K-major (0) or MN-major (1), M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc(uint32_t ab_format, uint32_t b_major, uint32_t n) {
  return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (b_major << 16) | ((n >> 3) << 17) |
         ((kRows >> 4) << 24);
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t id,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b), "r"(id), "r"(accumulate)
      : "memory");
}

// UMMAs into d, back to back: step s reads A through a[s] (a shared-memory
// descriptor, or a TMEM address in ta[s]) and B through b[s]; the first
// accumulates into d when acc0 != 0, the others always.  The operands are
// computed before the first is issued: an issue waits for the tensor core to
// take the previous one, so work between them would leave it idle.
__device__ __forceinline__ void mma_ss8(uint32_t d, const uint64_t (&a)[8], const uint64_t (&b)[8],
                                        uint32_t id, uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %18, 0;\n\tsetp.ne.b32 q, %19, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %9, %17, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %10, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %11, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %12, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %13, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %6, %14, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %15, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %8, %16, %17, q;\n\t}"
      ::"r"(d), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(a[4]), "l"(a[5]), "l"(a[6]),
        "l"(a[7]), "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]),
        "l"(b[7]), "r"(id), "r"(acc0), "r"(1u)
      : "memory");
}

__device__ __forceinline__ void mma_ts4(uint32_t d, const uint32_t (&ta)[4], const uint64_t (&b)[4],
                                        uint32_t id, uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %10, 0;\n\tsetp.ne.b32 q, %11, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %5, %9, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %6, %9, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %7, %9, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %8, %9, q;\n\t}"
      ::"r"(d), "r"(ta[0]), "r"(ta[1]), "r"(ta[2]), "r"(ta[3]), "l"(b[0]), "l"(b[1]), "l"(b[2]),
        "l"(b[3]), "r"(id), "r"(acc0), "r"(1u)
      : "memory");
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// One 32-byte store (the address 32-byte aligned).
__device__ __forceinline__ void st_global8(void* p, uint32_t a0, uint32_t a1, uint32_t a2,
                                           uint32_t a3, uint32_t a4, uint32_t a5, uint32_t a6,
                                           uint32_t a7) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a0),
               "r"(a1), "r"(a2), "r"(a3), "r"(a4), "r"(a5), "r"(a6), "r"(a7)
               : "memory");
}

__device__ __forceinline__ void commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(bar) : "memory");
}

// Byte offset of 16-byte chunk c (0..15) of row r in a tile (64-column blocks
// of 128 rows x 128 bytes, 128-byte swizzle).
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
  return (c >> 3) * kColBlock + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// The same for row rr of 16-key group k of a V tile (groups of 4 KB: two
// 64-column blocks of 16 rows).
__device__ __forceinline__ uint32_t vtile_off(int k, int rr, int c) {
  return k * 2 * kGroupBytes + (c >> 3) * kGroupBytes + rr * 128 + (((c & 7) ^ (rr & 7)) << 4);
}

// One work item: rows r0[0] .. r0[0] + 255 of sequence b, kv head g.  Half h
// holds rows r0[h] .. +127 and reads n_keys_h[h] keys (0: the sequence has no
// rows there); the K / V tiles loaded are the larger half's.
struct Item {
  int b, g, q0, rows, past;
  int n_keys, n_tiles, n_last;  // keys, tiles and last tile's rows of the larger half
  int r0[2], n_keys_h[2];
};

// Item w.  The (sequence, kv head) pairs go in blocks of a.pair_block; within
// a block the items go by rank, rank x being each pair's pair of query tiles
// tiles - 1 - x (the latest, longest, first), pair by pair.  False when there
// is nothing to do (the sequence has fewer rows, no new tokens, or lengths
// outside the launch's bounds, which `rep` reports).
__device__ __forceinline__ bool item_at(const PrefillArgs& a, int64_t w, Item& it, bool rep) {
  const int64_t n_pairs = static_cast<int64_t>(a.num_kv_heads) * a.batch;
  const int64_t pb = a.pair_block;
  const int64_t blk = w / (pb * a.tiles);
  const int64_t local = w - blk * pb * a.tiles;
  const int64_t in_blk = min(pb, n_pairs - blk * pb);  // pairs in this block
  const int x = static_cast<int>(local / in_blk);
  const int64_t bg = blk * pb + (local - x * in_blk);
  it.g = static_cast<int>(bg % a.num_kv_heads);
  it.b = static_cast<int>(bg / a.num_kv_heads);
  const int tile_q = a.tiles - 1 - x;
  it.q0 = a.query_start[it.b];
  const int nq = a.query_start[it.b + 1] - it.q0;
  const int ctx = a.context_lens[it.b];
  if (nq <= 0) return false;
  if (ctx < nq || ctx > a.max_blocks * a.block_size || nq > a.max_q || it.q0 < 0 ||
      it.q0 > a.total_q - nq) {
    if (rep && tile_q == 0 && it.g == 0) report(a.dev_error, PA_DEVERR_BAD_CTX);
    return false;
  }
  it.rows = nq * a.group;
  const int r0 = tile_q * 2 * kRows;
  if (r0 >= it.rows) return false;
  it.past = ctx - nq;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    it.r0[h] = r0 + h * kRows;
    it.n_keys_h[h] = it.r0[h] < it.rows
                         ? it.past + (min(it.r0[h] + kRows, it.rows) - 1) / a.group + 1
                         : 0;
  }
  it.n_keys = it.n_keys_h[1] > 0 ? it.n_keys_h[1] : it.n_keys_h[0];
  it.n_tiles = (it.n_keys + kKeys - 1) / kKeys;
  // rows of the last tile rounded up to 16: the groups loaded
  it.n_last = ((it.n_keys - (it.n_tiles - 1) * kKeys) + 15) & ~15;
  return true;
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc5_kernel(const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + kRing);
  // barriers: k_full, k_empty (one per K stage each; a stage is free after a
  // commit per half), v_full, v_empty (the same for V), per half q_full,
  // q_empty (its Q tile may be reloaded), o_free (O_h read by the epilogue),
  // final (one per issuer: its UMMAs completed), per half and score buffer
  // s_full (scores written), p_full (P written), pv_done (the P . V that read it
  // completed), then the item ring
  constexpr int kB = 2 * (kKStages + kVStages);
  const uint32_t b_k_full = tc::smem_u32(&bars[0]);
  const uint32_t b_k_empty = tc::smem_u32(&bars[kKStages]);
  const uint32_t b_v_full = tc::smem_u32(&bars[2 * kKStages]);
  const uint32_t b_v_empty = tc::smem_u32(&bars[2 * kKStages + kVStages]);
  const uint32_t b_q_full = tc::smem_u32(&bars[kB]);
  const uint32_t b_q_empty = tc::smem_u32(&bars[kB + 2]);
  const uint32_t b_o_free = tc::smem_u32(&bars[kB + 4]);
  const uint32_t b_final = tc::smem_u32(&bars[kB + 6]);     // one per issuer
  const uint32_t b_s_full = tc::smem_u32(&bars[kB + 10]);   // [half][buffer]
  const uint32_t b_p_full = tc::smem_u32(&bars[kB + 14]);
  const uint32_t b_pv_done = tc::smem_u32(&bars[kB + 18]);
  const uint32_t b_item_full = tc::smem_u32(&bars[kB + 22]);
  const uint32_t b_item_empty = tc::smem_u32(&bars[kB + 22 + kRingSlots]);
  constexpr int kNB = kB + 22 + 2 * kRingSlots;  // barriers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNB);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(bars + kNB + 1);
  volatile int64_t* item_q = reinterpret_cast<volatile int64_t*>(bars + kNB + 2);  // the ring

  const int64_t n_items = static_cast<int64_t>(a.tiles) * a.num_kv_heads * a.batch;
  const int G = a.group;
  const int bs = a.block_size;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kAB = PrefillPSplit<T>::value ? 1u : 0u;  // operand format: bf16 1, fp16 0

  if (threadIdx.x == 0) {
    for (int i = 0; i < kKStages; ++i) {
      tc::mbar_init(b_k_full + 8 * i, 1);
      tc::mbar_init(b_k_empty + 8 * i, 2);
    }
    for (int i = 0; i < kVStages; ++i) {
      tc::mbar_init(b_v_full + 8 * i, 1);
      tc::mbar_init(b_v_empty + 8 * i, 2);
    }
    for (int h = 0; h < 2; ++h) {
      tc::mbar_init(b_q_full + 8 * h, 1);
      tc::mbar_init(b_q_empty + 8 * h, 1);
      tc::mbar_init(b_o_free + 8 * h, 4);
    }
    for (int i = 0; i < 4; ++i) tc::mbar_init(b_final + 8 * i, 1);
    for (int i = 0; i < 4; ++i) {
      tc::mbar_init(b_s_full + 8 * i, 1);
      tc::mbar_init(b_p_full + 8 * i, 4);
      tc::mbar_init(b_pv_done + 8 * i, 1);
    }
    for (int i = 0; i < kRingSlots; ++i) {
      tc::mbar_init(b_item_full + 8 * i, 1);
      tc::mbar_init(b_item_empty + 8 * i, kItemReaders);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&qmap)) : "memory");
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

  // The ring's item ig (its slot ig % kRingSlots): the item index, or -1 after
  // the last.  Blocking read for the roles that have nothing else to do.
  auto ring_read = [&](int ig) -> int64_t {
    const int slot = ig % kRingSlots;
    if (!wait_ok(b_item_full + 8 * slot, (ig / kRingSlots) & 1, abort_flag, a.dev_error))
      return -1;
    const int64_t w = item_q[slot];
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(b_item_empty + 8 * slot);
    return w;
  };

  if (warp < 8) {
    // the register split is made per warpgroup, ahead of each role's code
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
    if (warp == kKWarp || warp == kVWarp) {
      // ================ K producer; Q and V producer ==================
      const int which = warp == kKWarp ? 0 : 1;  // 0: keys, 1: values (and Q)
      const int n_st = which ? kVStages : kKStages;
      const uint32_t full0 = which ? b_v_full : b_k_full;
      const uint32_t empty0 = which ? b_v_empty : b_k_empty;
      const uint32_t ring = base + (which ? kVOff : kKOff);
      const T* src = static_cast<const T*>(which ? a.v_cache : a.k_cache);
      const CUtensorMap* map = which ? &vmap : &kmap;
      int tg = 0;            // tiles of this CTA so far
      int nq0 = 0, nq1 = 0;  // (Q) items of each half so far
      bool live = true;
      int64_t w_static = blockIdx.x;
      for (int ig = 0; live; ++ig) {
        Item it;
        int64_t w = -1;
        if (which == 0) {
          // take the next item that has work (reporting invalid lengths) and
          // pass it on; -1 after the last
          const int slot = ig % kRingSlots;
          if (ig >= kRingSlots && !wait_ok(b_item_empty + 8 * slot, ((ig / kRingSlots) - 1) & 1,
                                           abort_flag, a.dev_error))
            break;
          if (lane == 0) {
            for (;;) {
              if (a.sched) {
                w = atomicAdd(reinterpret_cast<unsigned long long*>(a.sched), 1ull);
              } else {
                w = w_static;
                w_static += gridDim.x;
              }
              if (w >= n_items) {
                w = -1;
                break;
              }
              if (item_at(a, w, it, true)) break;
            }
            item_q[slot] = w;
            tc::mbar_arrive(b_item_full + 8 * slot);
          }
          w = __shfl_sync(kFull, w, 0);
        } else {
          w = ring_read(ig);
        }
        if (w < 0) break;
        item_at(a, w, it, false);
        if (which == 1) {
          // Half h's Q: 128 / G consecutive tokens x the G heads of kv head g,
          // one {64, G, 128 / G} box per 64-column block (rows past the
          // sequence's tokens are other tokens or zeros; their rows are never
          // stored), loaded once the half's last S product of its previous
          // item has completed.
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            int& nq = h ? nq1 : nq0;
            if (!live || it.n_keys_h[h] == 0) continue;
            if (nq >= 1 && !wait_ok(b_q_empty + 8 * h, (nq - 1) & 1, abort_flag, a.dev_error)) {
              live = false;
              continue;
            }
            if (lane == 0) {
              const uint32_t qf = b_q_full + 8 * h;
              tc::mbar_arrive_expect_tx(qf, kTileBytes);
              const uint32_t qs = base + kQOff + h * kTileBytes;
              const int tok = it.q0 + it.r0[h] / G;
              tma_3d(qs, &qmap, 0, it.g * G, tok, qf);
              tma_3d(qs + kColBlock, &qmap, 64, it.g * G, tok, qf);
            }
            ++nq;
          }
          if (!live) break;
        }
        // Lane k (< 8) reads the block id of 16-key group k of the next tile
        // while this one is loaded; an id is checked where it is used.
        const int32_t* bt = a.block_tables + static_cast<int64_t>(it.b) * a.max_blocks;
        auto raw_id = [&](int t) {
          const int key = t * kKeys + 16 * (lane & 7);
          return (lane < 8 && key < it.n_keys) ? __ldg(&bt[key / bs]) : -1;
        };
        int id_next = raw_id(0);
        for (int t = 0; t < it.n_tiles; ++t, ++tg) {
          const int stage = tg % n_st;
          const int n_grp = t == it.n_tiles - 1 ? it.n_last / 16 : kKeys / 16;
          int id_mine = id_next;
          if (t + 1 < it.n_tiles) id_next = raw_id(t + 1);
          const int key_mine = t * kKeys + 16 * (lane & 7);
          if (lane < n_grp && key_mine < it.n_keys && (id_mine < 0 || id_mine >= a.num_blocks)) {
            if (which == 0) report(a.dev_error, PA_DEVERR_BAD_BLOCK);
            id_mine = -1;
          }
          // whole groups in a valid block go by tensor map; the group holding
          // key n_keys - 1 when it is partial, and groups of invalid blocks, by
          // hand with zeros in the rows that hold no key; groups past the
          // tile's last row are never read
          const uint32_t tma_mask =
              __ballot_sync(kFull, lane < n_grp && id_mine >= 0 && key_mine + 16 <= it.n_keys);
          const uint32_t hand_mask = __ballot_sync(kFull, lane < n_grp) & ~tma_mask;
          const int row_mine =
              (id_mine < 0 ? 0 : id_mine * a.num_kv_heads + it.g) * bs + key_mine % bs;
          const uint32_t full = full0 + 8 * stage;
          if (tg >= n_st &&
              !wait_ok(empty0 + 8 * stage, ((tg / n_st) - 1) & 1, abort_flag, a.dev_error)) {
            live = false;
            break;
          }
          const uint32_t dst = ring + stage * kTileBytes;
          if (hand_mask) {
            for (int k = 0; k < kKeys / 16; ++k) {
              if (!(hand_mask >> k & 1)) continue;
              const int id = __shfl_sync(kFull, id_mine, k);
              const int key = t * kKeys + 16 * k;
              const int valid = id >= 0 ? min(16, it.n_keys - key) : 0;
              const T* rows0 =
                  src + (static_cast<int64_t>(id < 0 ? 0 : id * a.num_kv_heads + it.g) * bs +
                         key % bs) * kD;
              for (int i = lane; i < 16 * 16; i += 32) {
                const int rr = i >> 4, c = i & 15;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (rr < valid) v = __ldg(reinterpret_cast<const uint4*>(rows0 + rr * kD) + c);
                st_shared4(dst + (which ? vtile_off(k, rr, c) : tile_off(16 * k + rr, c)), v);
              }
            }
            // generic writes above are read by the tensor core (async proxy)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          }
          __syncwarp();
          if (lane == 0) {
            if (tma_mask)
              tc::mbar_arrive_expect_tx(full, __popc(tma_mask) * 2 * kGroupBytes);
            else
              tc::mbar_arrive(full);
          }
          __syncwarp();
          if (tma_mask >> lane & 1) {
            if (which) {  // {64, 16, 2} box of the {64, rows, 2} map: the whole group
              tma_3d(dst + lane * 2 * kGroupBytes, map, 0, row_mine, 0, full);
            } else {      // {64, 16} boxes of the {128, rows} map, one per column block
              tma_2d(dst + lane * kGroupBytes, map, 0, row_mine, full);
              tma_2d(dst + kColBlock + lane * kGroupBytes, map, 64, row_mine, full);
            }
          }
        }
      }
    } else if (warp == 1 || warp == 3 || warp == 4 || warp == 5) {
      // ============================ UMMA issuers ============================
      // Per half, one thread issues the S products and another the P . V
      // products, each after a (suspending) wait for its inputs.  S(u) needs
      // the K tile, the half's Q for the item's first sub-tile, and its score
      // buffer (u's parity among the half's sub-tiles), which held P two
      // sub-tiles back: free once that P . V has completed.  P . V(u) needs
      // P(u) and the V tile, and for an item's first sub-tile O_h of the
      // previous item read out.  Waiting rather than polling keeps the issuers
      // off the issue slots their SM sub-partitions share with softmax warps.
      const bool s_side = warp == 1 || warp == 3;
      const int h = (warp == 1 || warp == 4) ? 0 : 1;
      if (lane == 0) {
        const uint32_t s_col = tmem + h * kKeys;  // buffer j at + 64 j
        const uint32_t o_col = tmem + kColO + h * kD;
        const uint32_t bar_s = b_s_full + 16 * h, bar_p = b_p_full + 16 * h;
        const uint32_t bar_pv = b_pv_done + 16 * h;
        int kt = 0;  // K / V tiles of the CTA before the current item
        int n = 0;   // the half's sub-tiles so far (this side's products)
        int nq = 0;  // the half's items so far
        bool ok = true;
        auto wait1 = [&](uint32_t bar, uint32_t parity) {
          if (!ok) return false;
          if (tc::mbar_try_wait(bar, parity)) return true;
          const long long t0 = clock64();
          for (uint32_t i = 0; i < (1u << 26); ++i) {
            if (tc::mbar_try_wait(bar, parity)) return true;
            if ((i & 15) == 15 && (*abort_flag || clock64() - t0 > kSpinLimit)) break;
          }
          ok = false;
          return false;
        };
        constexpr uint32_t kIdO = idesc(kAB, 1, kD);
        int n_keys = 0, n_sub = 0, other_tiles = 0;
        // S of sub-tile u of the current item
        auto issue_s = [&](int u) {
          const int kidx = kt + (u >> 1);
          const uint32_t j = n & 1;
          if (n >= 2) wait1(bar_pv + 8 * j, ((n >> 1) - 1) & 1);
          if (u == 0) wait1(b_q_full + 8 * h, nq & 1);
          wait1(b_k_full + 8 * (kidx % kKStages), (kidx / kKStages) & 1);
          if (!ok) return;
          fence_after();
          const bool last = u == n_sub - 1;
          const uint32_t nn = last ? ((n_keys - kSub * u) + 15) & ~15 : kSub;
          // step s: columns 16 s .. +15, 32 bytes apart in a 64-column block,
          // the second block 16 KB on; the sub-tile's keys are rows 64 (u & 1)
          // on (descriptor start addresses count 16 bytes)
          const uint64_t dq = smem_desc(base + kQOff + h * kTileBytes, 16, 1024);
          const uint64_t dk = smem_desc(base + kKOff + (kidx % kKStages) * kTileBytes +
                                            (u & 1) * kSub * 128, 16, 1024);
          uint64_t qa[8], kb[8];
#pragma unroll
          for (int s = 0; s < kD / 16; ++s) {
            const uint32_t off = ((s >> 2) * kColBlock + (s & 3) * 32) >> 4;
            qa[s] = dq + off;
            kb[s] = dk + off;
          }
          mma_ss8(s_col + kSub * j, qa, kb, idesc(kAB, 0, nn), 0u);
          commit(bar_s + 8 * j);
          if ((u & 1) || last) {  // the half's last S on this K tile
            const uint32_t ke = b_k_empty + 8 * (kidx % kKStages);
            commit(ke);
            if ((u >> 1) >= other_tiles) commit(ke);  // the other half does not read it
          }
          if (last) {
            commit(b_q_empty + 8 * h);  // the half's Q may be reloaded
            ++nq;
          }
          ++n;
        };
        // P . V of sub-tile u of the current item
        auto issue_pv = [&](int u) {
          const int kidx = kt + (u >> 1);
          const uint32_t j = n & 1;
          wait1(bar_p + 8 * j, (n >> 1) & 1);
          wait1(b_v_full + 8 * (kidx % kVStages), (kidx / kVStages) & 1);
          if (u == 0 && nq > 0) wait1(b_o_free + 8 * h, (nq - 1) & 1);
          if (!ok) return;
          fence_after();
          const uint32_t p = s_col + kSub * j;  // P head: the buffer's columns 0..31
          const bool last = u == n_sub - 1;
          const int steps = last ? (((n_keys - kSub * u) + 15) & ~15) / 16 : kSub / 16;
          // 16-key group 4 (u & 1) + s of the V tile: column blocks 2 KB apart
          // (N), 8-key core groups 1 KB apart (K)
          const uint64_t dv = smem_desc(base + kVOff + (kidx % kVStages) * kTileBytes +
                                            (u & 1) * 4 * 2 * kGroupBytes, kGroupBytes, 1024);
          if (steps == kSub / 16) {
            uint64_t vb[4];
            uint32_t pa4[4];
#pragma unroll
            for (int s = 0; s < 4; ++s) {
              vb[s] = dv + ((s * 2 * kGroupBytes) >> 4);
              pa4[s] = p + 8 * s;
            }
            mma_ts4(o_col, pa4, vb, kIdO, u > 0 ? 1u : 0u);
            if (PrefillPSplit<T>::value) {
#pragma unroll
              for (int s = 0; s < 4; ++s) pa4[s] = p + 32 + 8 * s;
              mma_ts4(o_col, pa4, vb, kIdO, 1u);
            }
          } else {
            for (int s = 0; s < steps; ++s) {
              const uint64_t bd = dv + ((s * 2 * kGroupBytes) >> 4);
              mma_ts(o_col, p + 8 * s, bd, kIdO, (u > 0 || s > 0) ? 1u : 0u);
              if (PrefillPSplit<T>::value) mma_ts(o_col, p + 32 + 8 * s, bd, kIdO, 1u);
            }
          }
          commit(bar_pv + 8 * j);  // O_h holds this item's P . V so far
          if ((u & 1) || last) {   // the half's last P . V on this V tile
            const uint32_t ve = b_v_empty + 8 * (kidx % kVStages);
            commit(ve);
            if ((u >> 1) >= other_tiles) commit(ve);
          }
          ++n;
          if (last) ++nq;
        };
        for (int ig = 0; ok; ++ig) {
          const int slot = ig % kRingSlots;
          if (!wait1(b_item_full + 8 * slot, (ig / kRingSlots) & 1)) break;
          const int64_t w = item_q[slot];
          tc::mbar_arrive(b_item_empty + 8 * slot);
          if (w < 0) break;
          Item it;
          item_at(a, w, it, false);
          n_keys = h ? it.n_keys_h[1] : it.n_keys_h[0];
          const int keys_other = h ? it.n_keys_h[0] : it.n_keys_h[1];
          n_sub = (n_keys + kSub - 1) / kSub;
          other_tiles = (keys_other + kKeys - 1) / kKeys;
          for (int u = 0; u < n_sub && ok; ++u) {
            if (s_side)
              issue_s(u);
            else
              issue_pv(u);
          }
          kt += it.n_tiles;
        }
        if (!ok) {
          if (!*abort_flag) report(a.dev_error, PA_DEVERR_TIMEOUT);
          *abort_flag = 1;
        }
        // every UMMA this thread issued has completed before TMEM is released
        const uint32_t fin = b_final + 8 * (s_side ? h : 2 + h);
        commit(fin);
        tc::mbar_wait_bounded(fin, 0);
      }
      __syncwarp();
    }
  } else {
    // ======================= softmax and epilogue ===========================
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // Warps 8..11 take half 0, 12..15 half 1; a half's four warps run the same
    // items and meet at mbarriers only (bounded waits, so a warp that stops
    // after an abort holds no one up for good).
    const int h = (warp - 8) >> 2;
    const int quarter = warp & 3;            // TMEM lanes 32 quarter .. +31
    const int r = 32 * quarter + lane;       // this thread's row of the half
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
    const uint32_t col_s = h * kKeys, col_o = kColO + h * kD;
    const uint32_t bar_s = b_s_full + 16 * h, bar_p = b_p_full + 16 * h;
    const uint32_t bar_pv = b_pv_done + 16 * h, bar_o = b_o_free + 8 * h;
    const float c = a.scale_log2;  // > 0
    int m = 0;                     // the half's sub-tiles so far
    bool ok = true;
    for (int ig = 0;; ++ig) {
      // every softmax warp reads the ring, so all eight see the same items
      const int64_t w = ring_read(ig);
      if (w < 0) break;
      Item it;
      item_at(a, w, it, false);
      const int n_keys = h ? it.n_keys_h[1] : it.n_keys_h[0];
      if (n_keys == 0) continue;
      const int n_sub = (n_keys + kSub - 1) / kSub;
      const int grow = (h ? it.r0[1] : it.r0[0]) + r;
      const int pos = grow < it.rows ? it.past + grow / G : -1;
      float mref = -INFINITY;  // running reference, scaled (log2) domain
      // the row sum in two pairs, accumulated with packed fp32 adds
      float2 la = make_float2(0.f, 0.f), lb = make_float2(0.f, 0.f);
      for (int u = 0; u < n_sub; ++u, ++m) {
        const uint32_t j = m & 1;
        if (ok) ok = wait_ok(bar_s + 8 * j, (m >> 1) & 1, abort_flag, a.dev_error);
        if (!ok) continue;
        fence_after();
        const uint32_t sp = trow + col_s + kSub * j;
        uint32_t su[2][32];
        tmem_ld32_issue(sp, su[0]);
        tmem_ld32_issue(sp + 32, su[1]);
        tmem_ld_wait(su[0]);  // waits for both
        tmem_ld_wait(su[1]);
        float sv[2][32];
#pragma unroll
        for (int ch = 0; ch < 2; ++ch)
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[ch][i] = __uint_as_float(su[ch][i]);
        // causal mask where the sub-tile reaches past some row's position (and
        // for rows past the sequence); columns past the sub-tile's N are
        // masked too
        const int key0 = kSub * u;
        if (__any_sync(kFull, key0 + kSub - 1 > pos)) {
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (key0 + 32 * ch + i > pos) sv[ch][i] = -INFINITY;
        }
        // P over this sub-tile's score columns (head pairs in columns 0..31,
        // tails in 32..63) against the reference -neg, x = s c - reference two
        // at a time (packed fp32 FMA); with kMax the sub-tile's raw maximum is
        // taken in the same pass.
        float x0 = -INFINITY, x1 = -INFINITY, x2 = -INFINITY, x3 = -INFINITY;
        auto exps = [&](float neg, auto kMax) {
          const float2 c2 = make_float2(c, c), n2 = make_float2(neg, neg);
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t ph[16], pt[16];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              if (decltype(kMax)::value && (i & 2) == 0) {
                x0 = fmax3(x0, sv[ch][2 * i], sv[ch][2 * i + 1]);
                x1 = fmax3(x1, sv[ch][2 * i + 2], sv[ch][2 * i + 3]);
                x2 = fmax3(x2, sv[ch][2 * i + 4], sv[ch][2 * i + 5]);
                x3 = fmax3(x3, sv[ch][2 * i + 6], sv[ch][2 * i + 7]);
              }
              const float2 xa = __ffma2_rn(make_float2(sv[ch][2 * i], sv[ch][2 * i + 1]), c2, n2);
              const float2 xb =
                  __ffma2_rn(make_float2(sv[ch][2 * i + 2], sv[ch][2 * i + 3]), c2, n2);
              const float p0 = ex2(xa.x), p1 = ex2(xa.y), p2 = ex2(xb.x), p3 = ex2(xb.y);
              la = __fadd2_rn(la, make_float2(p0, p1));
              lb = __fadd2_rn(lb, make_float2(p2, p3));
              if (PrefillPSplit<T>::value) {
                tc::split2<T>(p0, p1, ph[i], pt[i]);
                tc::split2<T>(p2, p3, ph[i + 1], pt[i + 1]);
              } else {
                ph[i] = tc::pack2<T>(p0, p1);
                ph[i + 1] = tc::pack2<T>(p2, p3);
              }
            }
            tmem_st16(sp + 16 * ch, ph);
            if (PrefillPSplit<T>::value) tmem_st16(sp + 32 + 16 * ch, pt);
          }
        };
        // Once every row of the warp has a reference, the exponentials are
        // taken against it while the maximum is found; they stand unless some
        // row's maximum rose by more than 2^kSlack (then the row sums are put
        // back and the sub-tile is done again below, as for a first sub-tile).
        // Either way the weights and sums are those of the plain order.
        // (16-bit P without a tail only: the head + tail form would spill.)
        bool done = false;
        if (!PrefillPSplit<T>::value && __all_sync(kFull, mref != -INFINITY)) {
          const float2 la0 = la, lb0 = lb;
          exps(-mref, std::true_type{});
          const float mr = fmax3(fmaxf(x0, x1), x2, x3);
          const float m2 = mr == -INFINITY ? -INFINITY : mr * c;
          if (!__any_sync(kFull, m2 > mref + kSlack)) {
            done = true;
          } else {
            la = la0;
            lb = lb0;
            tmem_st_wait();  // the stores above land before the ones that replace them
          }
        } else {
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              x0 = fmax3(x0, sv[ch][i], sv[ch][i + 1]);
              x1 = fmax3(x1, sv[ch][i + 2], sv[ch][i + 3]);
              x2 = fmax3(x2, sv[ch][i + 4], sv[ch][i + 5]);
              x3 = fmax3(x3, sv[ch][i + 6], sv[ch][i + 7]);
            }
        }
        if (!done) {
          const float mx_raw = fmax3(fmaxf(x0, x1), x2, x3);
          const float mx = mx_raw == -INFINITY ? -INFINITY : mx_raw * c;
          // a row whose maximum rose by more than 2^kSlack takes it as its new
          // reference and rescales its row of O_h once the half's previous
          // P . V has completed.  TMEM loads and stores are warp-collective, so
          // the warp does this together; rows that keep their reference scale
          // by 1.
          const bool moves = mx > mref + kSlack;
          if (__any_sync(kFull, moves)) {
            const float mnew = moves ? mx : mref;
            const float alpha = mref == -INFINITY ? 0.f : ex2(mref - mnew);
            if (u > 0) {
              const int mp = m - 1;
              ok = wait_ok(bar_pv + 8 * (mp & 1), (mp >> 1) & 1, abort_flag, a.dev_error);
              if (!ok) continue;
              fence_after();
#pragma unroll 1
              for (int ch = 0; ch < 4; ++ch) {
                uint32_t ou[32];
                tmem_ld32_issue(trow + col_o + 32 * ch, ou);
                tmem_ld_wait(ou);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  ou[i] = __float_as_uint(__uint_as_float(ou[i]) * alpha);
                tmem_st32(trow + col_o + 32 * ch, ou);
              }
            }
            la = __fmul2_rn(la, make_float2(alpha, alpha));
            lb = __fmul2_rn(lb, make_float2(alpha, alpha));
            mref = mnew;
          }
          exps(mref == -INFINITY ? 0.f : -mref, std::false_type{});
        }
        tmem_st_wait();
        fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar_p + 8 * j);
      }
      // epilogue: O_h / l once the item's last P . V is done, each row stored
      // from registers (rows past the sequence are not stored)
      if (ok) {
        const int mp = m - 1;
        ok = wait_ok(bar_pv + 8 * (mp & 1), (mp >> 1) & 1, abort_flag, a.dev_error);
      }
      if (ok) {
        fence_after();
        const float inv = 1.f / ((la.x + la.y) + (lb.x + lb.y));
        T* dst = nullptr;
        if (grow < it.rows) {
          const int tok = grow / G, hh = grow - tok * G;
          dst = static_cast<T*>(a.out) +
                (static_cast<int64_t>(it.q0 + tok) * a.num_q_heads + it.g * G + hh) * kD;
        }
        // rows are 256 bytes: 32-byte stores when out allows them, else 16-byte
        const bool wide = (reinterpret_cast<uintptr_t>(a.out) & 31) == 0;
#pragma unroll 1
        for (int ch = 0; ch < 4; ch += 2) {
          uint32_t ou[2][32];
          tmem_ld32_issue(trow + col_o + 32 * ch, ou[0]);
          tmem_ld32_issue(trow + col_o + 32 * ch + 32, ou[1]);
          tmem_ld_wait(ou[0]);  // waits for both
          tmem_ld_wait(ou[1]);
          if (dst) {
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = tc::pack2<T>(__uint_as_float(ou[c2][2 * i]) * inv,
                                     __uint_as_float(ou[c2][2 * i + 1]) * inv);
              T* d = dst + 32 * (ch + c2);  // 64 bytes
              if (wide) {
                st_global8(d, pk[0], pk[1], pk[2], pk[3], pk[4], pk[5], pk[6], pk[7]);
                st_global8(d + 16, pk[8], pk[9], pk[10], pk[11], pk[12], pk[13], pk[14], pk[15]);
              } else {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  reinterpret_cast<uint4*>(d)[k] =
                      make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
              }
            }
          }
        }
      }
      // O_h has been read: the next item's first P . V may overwrite it
      fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar_o);
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
  // the last CTA to finish returns the scheduling counter to zero (every
  // CTA's last take is behind it)
  if (a.sched && threadIdx.x == 0) {
    __threadfence();
    unsigned long long* done = reinterpret_cast<unsigned long long*>(a.sched + 1);
    if (atomicAdd(done, 1ull) == gridDim.x - 1) {
      a.sched[0] = 0;
      a.sched[1] = 0;
      __threadfence();
    }
  }
}

template <typename T>
static cudaError_t launch_t(const PrefillArgs& a, const CUtensorMap& qmap, const CUtensorMap& kmap,
                            const CUtensorMap& vmap, cudaStream_t stream) {
  auto kern = prefill_tc5_kernel<T>;
  static bool raised[64] = {};
  static int sms[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int n_sm = dev >= 0 && dev < 64 ? sms[dev] : 0;
  if (n_sm == 0) {
    e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) sms[dev] = n_sm;
  }
  if (dev < 0 || dev >= 64 || !raised[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) raised[dev] = true;
  }
  const int64_t n_items = static_cast<int64_t>(a.tiles) * a.num_kv_heads * a.batch;
  // persistent (one CTA per SM) with a scheduling counter, else one item per CTA
  const int64_t cap = a.sched ? n_sm : INT32_MAX;
  const int grid = static_cast<int>(n_items < cap ? n_items : cap);
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, kThreads, kSmem, stream>>>(qmap, kmap, vmap, a);
  return cudaGetLastError();
}

}  // namespace t5

cudaError_t launch_prefill_tc5(PrefillArgs a, pa_dtype dtype, const CUtensorMap& qmap,
                               const CUtensorMap& kmap2d, const CUtensorMap& vmap3d,
                               cudaStream_t stream) {
  // items of two 128-row halves per (sequence, kv head)
  a.tiles = static_cast<int>((static_cast<int64_t>(a.max_q) * a.group + 2 * t5::kRows - 1) /
                             (2 * t5::kRows));
  return dtype == PA_F16 ? t5::launch_t<__half>(a, qmap, kmap2d, vmap3d, stream)
                         : t5::launch_t<__nv_bfloat16>(a, qmap, kmap2d, vmap3d, stream);
}

}  // namespace pa
