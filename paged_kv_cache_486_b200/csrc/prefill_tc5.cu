// Paged prefill on the 5th-generation tensor cores (tcgen05 / UMMA, TMEM).
//
// Same definition and row layout as prefill.cu (causal attention of each
// sequence's new tokens over its paged cache; a work item is 128 rows = (new
// token, head of one kv head's group) pairs of one sequence and kv head),
// head_dim 128, fp16 / bf16, scale > 0.
//
// Persistent when the caller gives a scheduling workspace: one CTA per SM takes
// items from a global counter, and the next item's Q, K and V loads and first
// scores overlap this item's last tiles and its store.  Items go by (sequence,
// kv head), the latest (longest) query tile first: the tiles that read the same
// keys and values run on neighbouring SMs at the same time, so those reach
// each SM from L2 (the way one CTA per item with the tile index fastest is
// dispatched).  The K producer takes the items and passes them to the other roles
// through a four-slot ring in shared memory.  Without a workspace each CTA
// runs one item.
//
// Per item, key tiles of 128 keys:
//   S = Q . K_tile^T   UMMA M=128 N=128 (the last tile: N rounded up to 16
//                      past its keys), K=128 in 8 steps of 16, Q and K from
//                      shared memory (128-byte-swizzled, K-major), fp32 in TMEM;
//   softmax            one thread per row reads its S row from TMEM, masks
//                      (causal, diagonal tiles only), keeps its running max
//                      lazily (O is rescaled only when the max rises by more
//                      than 2^8) and writes P as 16-bit values over its own S
//                      columns;
//   O += P . V_tile    UMMA with A = P from TMEM (K-major), B = V from shared
//                      memory (MN-major: head_dim contiguous), fp32 in TMEM.
// bf16 keeps P as a head + tail pair (two products), fp16 a single value.
//
// Warps: 0 loads Q and the K tiles, 6 the V tiles (TMA, each tensor with its
// own stages), 1 allocates TMEM and issues every UMMA from one thread as soon
// as each product's inputs are ready, 2..5 run the softmax and the epilogue
// (warp w reads TMEM lanes 32 (w mod 4) .. +31, which are its rows).  S / P
// has three buffers in TMEM (columns 0, 128, 256), so the tensor core
// computes the next tiles' scores while the softmax works on this one; a
// buffer takes new scores only once the product that read its P has completed
// (products with different accumulators are not ordered by issue alone).  O is
// in 384..511; an item's first P . V waits until the softmax warps have read
// the previous item's O.
//
// Shared memory (1024-byte aligned, rows of 128 bytes with the 128-byte
// swizzle): Q 2 x 32 KB (an item's O is staged in its Q tile and written by
// TMA when the tile is whole, by coalesced stores when it is the ragged end of
// a sequence), K 3 x 32 KB, V 2 x 32 KB.  Q and K tiles are two 64-column
// blocks of 128 rows (the S product's K-major operands); a V tile is eight
// 16-key groups of two 64-column blocks of 16 rows, so one 4 KB copy brings a
// group (half the copies of two 2 KB boxes; the P . V operand is described
// group by group either way).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_tc.cuh"
#include "prefill_launch.h"
#include "tc5_ptx.cuh"

namespace pa {
namespace t5 {

using tc::kFull;
constexpr int kRows = 128;   // query rows per item
constexpr int kKeys = 128;   // keys per tile
constexpr int kD = 128;
constexpr int kThreads = 224;
constexpr int kVWarp = 6;                  // the V producer (warp 0 loads Q and K)
constexpr int kColBlock = kRows * 128;     // one 64-column block of 128 rows: 16 KB
constexpr int kTileBytes = 2 * kColBlock;  // 128 rows x 128 columns x 2 bytes
constexpr int kGroupBytes = 16 * 128;      // 16 rows of one 64-column block
constexpr int kKStages = 3;                // K tiles in flight
constexpr int kVStages = 2;                // V tiles in flight
constexpr int kQOff = 0;                   // two Q tiles
constexpr int kKOff = 2 * kTileBytes;
constexpr int kVOff = kKOff + kKStages * kTileBytes;
constexpr int kRing = kVOff + kVStages * kTileBytes;  // 224 KB
constexpr int kRingSlots = 4;              // items passed from the K producer to the others
constexpr int kItemReaders = 7;            // V producer, issuer (S and P . V), 4 softmax warps
constexpr int kSmem = 1024 + kRing + 512;
constexpr uint32_t kTmemCols = 512;
constexpr int kSBuf = 3;  // S / P buffers in TMEM
constexpr uint32_t kColS = 0, kColO = kSBuf * kKeys;
constexpr float kSlack = 8.f;
constexpr long long kSpinLimit = 1ll << 31;  // clock cycles without progress

// ---- PTX wrappers (the generic ones are in tc5_ptx.cuh) ----
// kind::f16 instruction descriptor: fp32 accumulator, A / B in fp16 (0) or
// bf16 (1), A K-major, B K-major (0) or MN-major (1), M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc(uint32_t ab_format, uint32_t b_major, uint32_t n) {
  return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (b_major << 16) | ((n >> 3) << 17) |
         ((kRows >> 4) << 24);
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

// One work item: 128 rows of sequence b, kv head g.
struct Item {
  int b, g, q0, r0, rows, past, n_keys, n_tiles, n_last;
};

// Item w: (sequence, kv head) w / tiles, its query tile tiles - 1 - w % tiles
// (latest first).  False when there is nothing to do (the sequence has fewer
// rows, no new tokens, or lengths outside the launch's bounds, which `rep`
// reports).
__device__ __forceinline__ bool item_at(const PrefillArgs& a, int64_t w, Item& it, bool rep) {
  const int64_t bg = w / a.tiles;
  const int x = static_cast<int>(w - bg * a.tiles);
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
  it.r0 = tile_q * kRows;
  if (it.r0 >= it.rows) return false;
  it.past = ctx - nq;
  it.n_keys = it.past + (min(it.r0 + kRows, it.rows) - 1) / a.group + 1;
  it.n_tiles = (it.n_keys + kKeys - 1) / kKeys;
  // keys of the last tile rounded up to 16: its S product's N, its P . V steps
  it.n_last = ((it.n_keys - (it.n_tiles - 1) * kKeys) + 15) & ~15;
  return true;
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc5_kernel(const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap,
                       const __grid_constant__ CUtensorMap omap, PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + kRing);
  // barriers: k_full, k_empty (one per K stage each), v_full, v_empty (one per
  // V stage each), per S / P buffer s_full (scores written), p_full (P
  // written), pv_done (its P . V completed), per Q tile q_full, q_empty (its
  // item stored), then o_free (O read by the epilogue), final
  constexpr int kB = 2 * (kKStages + kVStages);
  const uint32_t b_k_full = tc::smem_u32(&bars[0]);
  const uint32_t b_k_empty = tc::smem_u32(&bars[kKStages]);
  const uint32_t b_v_full = tc::smem_u32(&bars[2 * kKStages]);
  const uint32_t b_v_empty = tc::smem_u32(&bars[2 * kKStages + kVStages]);
  const uint32_t b_s_full = tc::smem_u32(&bars[kB]);
  const uint32_t b_p_full = tc::smem_u32(&bars[kB + kSBuf]);
  const uint32_t b_pv_done = tc::smem_u32(&bars[kB + 2 * kSBuf]);
  const uint32_t b_q_full = tc::smem_u32(&bars[kB + 3 * kSBuf]);
  const uint32_t b_q_empty = tc::smem_u32(&bars[kB + 3 * kSBuf + 2]);
  const uint32_t b_o_free = tc::smem_u32(&bars[kB + 3 * kSBuf + 4]);
  const uint32_t b_final = tc::smem_u32(&bars[kB + 3 * kSBuf + 5]);
  const uint32_t b_item_full = tc::smem_u32(&bars[kB + 3 * kSBuf + 6]);
  const uint32_t b_item_empty = tc::smem_u32(&bars[kB + 3 * kSBuf + 6 + kRingSlots]);
  // the four softmax warps: staging written (per item), staging read (per
  // ragged item)
  const uint32_t b_staged = tc::smem_u32(&bars[kB + 3 * kSBuf + 6 + 2 * kRingSlots]);
  const uint32_t b_read = tc::smem_u32(&bars[kB + 3 * kSBuf + 7 + 2 * kRingSlots]);
  constexpr int kNB = kB + 3 * kSBuf + 8 + 2 * kRingSlots;  // barriers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNB);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(bars + kNB + 1);
  volatile int64_t* item_q = reinterpret_cast<volatile int64_t*>(bars + kNB + 2);  // the ring

  const int64_t n_items = static_cast<int64_t>(a.tiles) * a.num_kv_heads * a.batch;
  const int G = a.group;
  const int bs = a.block_size;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kAB = PrefillPSplit<T>::value ? 1u : 0u;  // operand format: bf16 1, fp16 0

  if (threadIdx.x == 0) {
    for (int i = 0; i < kB; ++i) tc::mbar_init(tc::smem_u32(&bars[i]), 1);
    for (int i = 0; i < kSBuf; ++i) {
      tc::mbar_init(b_s_full + 8 * i, 1);
      tc::mbar_init(b_p_full + 8 * i, 4);
      tc::mbar_init(b_pv_done + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(b_q_full + 8 * i, 1);
      tc::mbar_init(b_q_empty + 8 * i, 1);
    }
    tc::mbar_init(b_o_free, 4);
    tc::mbar_init(b_final, 1);
    for (int i = 0; i < kRingSlots; ++i) {
      tc::mbar_init(b_item_full + 8 * i, 1);
      tc::mbar_init(b_item_empty + 8 * i, kItemReaders);
    }
    tc::mbar_init(b_staged, 4);
    tc::mbar_init(b_read, 4);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&qmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&kmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&omap)) : "memory");
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

  if (warp == 0 || warp == kVWarp) {
    // ======================== Q and K / V producers =========================
    const int which = warp == 0 ? 0 : 1;  // 0: keys (and Q), 1: values
    const int n_st = which ? kVStages : kKStages;
    const uint32_t full0 = which ? b_v_full : b_k_full;
    const uint32_t empty0 = which ? b_v_empty : b_k_empty;
    const uint32_t ring = base + (which ? kVOff : kKOff);
    const T* src = static_cast<const T*>(which ? a.v_cache : a.k_cache);
    const CUtensorMap* map = which ? &vmap : &kmap;
    int tg = 0;  // tiles of this CTA so far
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
      if (which == 0) {
        // Q: 128 / G consecutive tokens x the G heads of kv head g, one
        // {64, G, 128 / G} box per 64-column block (rows past the sequence's
        // tokens are other tokens or zeros; their rows are never stored)
        const int qb = ig & 1;
        if (ig >= 2 && !wait_ok(b_q_empty + 8 * qb, ((ig >> 1) - 1) & 1, abort_flag, a.dev_error))
          break;
        if (lane == 0) {
          const uint32_t qf = b_q_full + 8 * qb;
          tc::mbar_arrive_expect_tx(qf, kTileBytes);
          const uint32_t qs = base + kQOff + qb * kTileBytes;
          tma_3d(qs, &qmap, 0, it.g * G, it.q0 + it.r0 / G, qf);
          tma_3d(qs + kColBlock, &qmap, 64, it.g * G, it.q0 + it.r0 / G, qf);
        }
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
        // tile's N are never read
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
  } else if (warp == 1) {
    // ============================= UMMA issuer ==============================
    // Two cursors walk the CTA's tiles: the next S and the next P . V.  S_n
    // (global tile n) needs K_n, its item's Q, and its TMEM buffer, which held
    // P_{n-3}: free once P_{n-3} . V has completed.  P_n . V needs P_n and
    // V_n, and for an item's first tile the previous item's O read out.
    const bool leader = lane == 0;
    // cursor states: 0 waiting for its next item from the ring, 1 on an
    // item, 2 past the last item
    struct Cursor {
      int ig, t, state;
      Item it;
    };
    auto try_fetch = [&](Cursor& c) {  // non-blocking; warp-uniform
      const int slot = c.ig % kRingSlots;
      bool got = false;
      if (leader) got = mbar_test(b_item_full + 8 * slot, (c.ig / kRingSlots) & 1);
      if (!__shfl_sync(kFull, got, 0)) return false;
      // the leader observed the phase (acquire), so the leader reads the slot
      const int64_t w = __shfl_sync(kFull, leader ? static_cast<long long>(item_q[slot]) : 0ll, 0);
      __syncwarp();
      if (leader) tc::mbar_arrive(b_item_empty + 8 * slot);
      if (w < 0) {
        c.state = 2;
      } else {
        item_at(a, w, c.it, false);
        c.t = 0;
        c.state = 1;
      }
      return true;
    };
    auto advance = [&](Cursor& c) {
      if (++c.t < c.it.n_tiles) return;
      ++c.ig;
      c.state = 0;
    };
    Cursor cs{0, 0, 0, {}}, cp{0, 0, 0, {}};
    int ns = 0, npv = 0;
    bool ok = true;
    long long idle0 = clock64();
    while (ok && cp.state != 2) {
      bool progress = false;
      if (cs.state == 0 && try_fetch(cs)) progress = true;
      if (cp.state == 0 && try_fetch(cp)) progress = true;
      if (cs.state == 1 && ns <= npv + kSBuf - 1) {
        bool ready = false;
        if (leader)
          ready = (ns < kSBuf || mbar_test(b_pv_done + 8 * (ns % kSBuf),
                                           ((ns - kSBuf) / kSBuf) & 1)) &&
                  mbar_test(b_k_full + 8 * (ns % kKStages), (ns / kKStages) & 1) &&
                  (cs.t > 0 || mbar_test(b_q_full + 8 * (cs.ig & 1), (cs.ig >> 1) & 1));
        if (__shfl_sync(kFull, ready, 0)) {
          if (leader) {
            fence_after();
            const uint32_t q_s = base + kQOff + (cs.ig & 1) * kTileBytes;
            const uint32_t kt = base + kKOff + (ns % kKStages) * kTileBytes;
            const uint32_t d = tmem + kColS + (ns % kSBuf) * kKeys;
            const uint32_t id =
                idesc(kAB, 0, cs.t == cs.it.n_tiles - 1 ? cs.it.n_last : kKeys);
#pragma unroll
            for (int s = 0; s < kD / 16; ++s) {
              const uint32_t off = (s >> 2) * kColBlock + (s & 3) * 32;
              mma_ss(d, smem_desc(q_s + off, 16, 1024), smem_desc(kt + off, 16, 1024), id, s > 0);
            }
            commit(b_s_full + 8 * (ns % kSBuf));
            commit(b_k_empty + 8 * (ns % kKStages));  // K_ns may be refilled
          }
          ++ns;
          advance(cs);
          progress = true;
        }
      }
      if (cp.state == 1 && npv < ns) {
        bool ready = false;
        if (leader)
          ready = mbar_test(b_p_full + 8 * (npv % kSBuf), (npv / kSBuf) & 1) &&
                  mbar_test(b_v_full + 8 * (npv % kVStages), (npv / kVStages) & 1) &&
                  (cp.t > 0 || cp.ig == 0 || mbar_test(b_o_free, (cp.ig - 1) & 1));
        if (__shfl_sync(kFull, ready, 0)) {
          if (leader) {
            fence_after();
            const uint32_t vt = base + kVOff + (npv % kVStages) * kTileBytes;
            const uint32_t p = tmem + kColS + (npv % kSBuf) * kKeys;  // P head: columns 0..63
            const int steps = cp.t == cp.it.n_tiles - 1 ? cp.it.n_last / 16 : kKeys / 16;
            constexpr uint32_t kIdO = idesc(kAB, 1, kD);
            for (int s = 0; s < steps; ++s) {
              // group s: column blocks 2 KB apart (N), 8-key core groups 1 KB apart (K)
              const uint64_t bd = smem_desc(vt + s * 2 * kGroupBytes, kGroupBytes, 1024);
              mma_ts(tmem + kColO, p + 8 * s, bd, kIdO, (cp.t > 0 || s > 0) ? 1u : 0u);
              if (PrefillPSplit<T>::value) mma_ts(tmem + kColO, p + 64 + 8 * s, bd, kIdO, 1u);
            }
            commit(b_v_empty + 8 * (npv % kVStages));  // V_npv may be refilled
            commit(b_pv_done + 8 * (npv % kSBuf));     // O holds this item's P . V so far
          }
          ++npv;
          advance(cp);
          progress = true;
        }
      }
      if (progress) {
        idle0 = clock64();
      } else {
        if (clock64() - idle0 > kSpinLimit || *abort_flag) ok = false;
        __nanosleep(20);
      }
      ok = __all_sync(kFull, ok);
    }
    if (!ok && lane == 0) {
      if (!*abort_flag) report(a.dev_error, PA_DEVERR_TIMEOUT);
      *abort_flag = 1;
    }
    // every UMMA this thread issued has completed before TMEM is released
    if (leader) commit(b_final);
    __syncwarp();
    tc::mbar_wait_bounded(b_final, 0);
  } else {
    // ======================= softmax and epilogue ===========================
    // The four warps run the same items; they meet at two mbarriers (bounded
    // waits, so a warp that stops after an abort holds no one up for good).
    const int quarter = warp & 3;            // TMEM lanes 32 quarter .. +31
    const int r = 32 * quarter + lane;       // this thread's row of an item
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
    const float c = a.scale_log2;  // > 0
    int tg = 0, n_ragged = 0;
    bool ok = true;
    for (int ig = 0;; ++ig) {
      // every softmax warp reads the ring, so all four see the same items
      const int64_t w = ring_read(ig);
      if (w < 0) break;
      Item it;
      item_at(a, w, it, false);
      const int grow = it.r0 + r;
      const int pos = grow < it.rows ? it.past + grow / G : -1;
      float m = -INFINITY;  // running reference, scaled (log2) domain
      float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
      for (int t = 0; t < it.n_tiles; ++t, ++tg) {
        if (ok) ok = wait_ok(b_s_full + 8 * (tg % kSBuf), (tg / kSBuf) & 1, abort_flag, a.dev_error);
        if (!ok) continue;
        fence_after();
        const uint32_t sp = trow + kColS + (tg % kSBuf) * kKeys;
        uint32_t su[4][32];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_ld32_issue(sp + 32 * ch, su[ch]);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_ld_wait(su[ch]);  // the first waits for all four
        float sv[4][32];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[ch][i] = __uint_as_float(su[ch][i]);
        // causal mask where the tile reaches past some row's position (and
        // for rows past the sequence); columns past the tile's N are masked too
        if (__any_sync(kFull, t * kKeys + kKeys - 1 > pos)) {
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (t * kKeys + 32 * ch + i > pos) sv[ch][i] = -INFINITY;
        }
        float x0 = -INFINITY, x1 = -INFINITY, x2 = -INFINITY, x3 = -INFINITY;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            x0 = fmaxf(x0, sv[ch][i]);
            x1 = fmaxf(x1, sv[ch][i + 1]);
            x2 = fmaxf(x2, sv[ch][i + 2]);
            x3 = fmaxf(x3, sv[ch][i + 3]);
          }
        const float mx_raw = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3));
        const float mx = mx_raw == -INFINITY ? -INFINITY : mx_raw * c;
        // a row whose maximum rose by more than 2^kSlack takes it as its new
        // reference and rescales its row of O once the previous P . V is done.
        // TMEM loads and stores are warp-collective, so the warp does this
        // together; rows that keep their reference scale by 1.
        const bool moves = mx > m + kSlack;
        if (__any_sync(kFull, moves)) {
          const float mnew = moves ? mx : m;
          const float alpha = m == -INFINITY ? 0.f : ex2(m - mnew);
          if (t > 0) {
            ok = wait_ok(b_pv_done + 8 * ((tg - 1) % kSBuf), ((tg - 1) / kSBuf) & 1, abort_flag,
                         a.dev_error);
            if (!ok) continue;
            fence_after();
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t ou[32];
              tmem_ld32_issue(trow + kColO + 32 * ch, ou);
              tmem_ld_wait(ou);
#pragma unroll
              for (int i = 0; i < 32; ++i)
                ou[i] = __float_as_uint(__uint_as_float(ou[i]) * alpha);
              tmem_st32(trow + kColO + 32 * ch, ou);
            }
          }
          l0 *= alpha;
          l1 *= alpha;
          l2 *= alpha;
          l3 *= alpha;
          m = mnew;
        }
        const float neg = m == -INFINITY ? 0.f : -m;
        // P over this tile's S columns: head pairs in columns 0..63, tails in 64..127
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t ph[16], pt[16];
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const float p0 = ex2(fmaf(sv[ch][2 * i], c, neg));
            const float p1 = ex2(fmaf(sv[ch][2 * i + 1], c, neg));
            const float p2 = ex2(fmaf(sv[ch][2 * i + 2], c, neg));
            const float p3 = ex2(fmaf(sv[ch][2 * i + 3], c, neg));
            l0 += p0;
            l1 += p1;
            l2 += p2;
            l3 += p3;
            if (PrefillPSplit<T>::value) {
              tc::split2<T>(p0, p1, ph[i], pt[i]);
              tc::split2<T>(p2, p3, ph[i + 1], pt[i + 1]);
            } else {
              ph[i] = tc::pack2<T>(p0, p1);
              ph[i + 1] = tc::pack2<T>(p2, p3);
            }
          }
          tmem_st16(sp + 16 * ch, ph);
          if (PrefillPSplit<T>::value) tmem_st16(sp + 64 + 16 * ch, pt);
        }
        tmem_st_wait();
        fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(b_p_full + 8 * (tg % kSBuf));
      }
      // epilogue: O / l once the item's last P . V is done, staged in the
      // item's Q tile (its S products are complete then) in the Q layout
      const int qb = ig & 1;
      const uint32_t stage_out = base + kQOff + qb * kTileBytes;
      if (ok)
        ok = wait_ok(b_pv_done + 8 * ((tg - 1) % kSBuf), ((tg - 1) / kSBuf) & 1, abort_flag,
                     a.dev_error);
      if (ok) {
        fence_after();
        const float inv = 1.f / ((l0 + l1) + (l2 + l3));
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t ou[32];
          tmem_ld32_issue(trow + kColO + 32 * ch, ou);
          tmem_ld_wait(ou);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint4 v;
            v.x = tc::pack2<T>(__uint_as_float(ou[8 * k]) * inv,
                               __uint_as_float(ou[8 * k + 1]) * inv);
            v.y = tc::pack2<T>(__uint_as_float(ou[8 * k + 2]) * inv,
                               __uint_as_float(ou[8 * k + 3]) * inv);
            v.z = tc::pack2<T>(__uint_as_float(ou[8 * k + 4]) * inv,
                               __uint_as_float(ou[8 * k + 5]) * inv);
            v.w = tc::pack2<T>(__uint_as_float(ou[8 * k + 6]) * inv,
                               __uint_as_float(ou[8 * k + 7]) * inv);
            st_shared4(stage_out + tile_off(r, 4 * ch + k), v);
          }
        }
      }
      // O has been read: the next item's first P . V may overwrite it
      fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(b_o_free);
      // the staged tile is read by TMA (async proxy) or by the other warps
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(b_staged);
      if (it.r0 + kRows <= it.rows) {
        // a whole tile: two TMA stores, the same boxes as the Q loads
        if (warp == 2) {
          const bool go = wait_ok(b_staged, ig & 1, abort_flag, a.dev_error);
          if (lane == 0) {
            if (go) {
              tma_store_3d(&omap, 0, it.g * G, it.q0 + it.r0 / G, stage_out);
              tma_store_3d(&omap, 64, it.g * G, it.q0 + it.r0 / G, stage_out + kColBlock);
              asm volatile("cp.async.bulk.commit_group;" ::: "memory");
              asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            }
            tc::mbar_arrive(b_q_empty + 8 * qb);
          }
        }
      } else {
        // the sequence's ragged end: the valid rows, as whole 16-byte chunks
        if (wait_ok(b_staged, ig & 1, abort_flag, a.dev_error)) {
          const int i = threadIdx.x - 64;  // 0..127
          const int cc = i & 15;
#pragma unroll 4
          for (int k = 0; k < kRows / 8; ++k) {
            const int rr = 8 * k + (i >> 4);
            const int gr = it.r0 + rr;
            if (gr < it.rows) {
              const int tok = gr / G, hh = gr - tok * G;
              T* dst = static_cast<T*>(a.out) +
                       (static_cast<int64_t>(it.q0 + tok) * a.num_q_heads + it.g * G + hh) * kD;
              reinterpret_cast<uint4*>(dst)[cc] = ld_shared4(stage_out + tile_off(rr, cc));
            }
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(b_read);
        if (warp == 2) {
          wait_ok(b_read, n_ragged & 1, abort_flag, a.dev_error);
          if (lane == 0) tc::mbar_arrive(b_q_empty + 8 * qb);
        }
        ++n_ragged;
      }
    }
    if (threadIdx.x == 64) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
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
                            const CUtensorMap& vmap, const CUtensorMap& omap,
                            cudaStream_t stream) {
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
  kern<<<grid, kThreads, kSmem, stream>>>(qmap, kmap, vmap, omap, a);
  return cudaGetLastError();
}

}  // namespace t5

cudaError_t launch_prefill_tc5(PrefillArgs a, pa_dtype dtype, const CUtensorMap& qmap,
                               const CUtensorMap& kmap2d, const CUtensorMap& vmap3d,
                               const CUtensorMap& omap, cudaStream_t stream) {
  a.tiles = static_cast<int>((static_cast<int64_t>(a.max_q) * a.group + t5::kRows - 1) / t5::kRows);
  return dtype == PA_F16 ? t5::launch_t<__half>(a, qmap, kmap2d, vmap3d, omap, stream)
                         : t5::launch_t<__nv_bfloat16>(a, qmap, kmap2d, vmap3d, omap, stream);
}

}  // namespace pa
