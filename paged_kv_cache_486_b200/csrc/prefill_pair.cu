// Paged prefill on pairs of SMs (tcgen05 with cta_group::2).
//
// Same definition, row layout and per-row softmax as prefill_tc5.cu (causal
// attention of each sequence's new tokens over its paged cache, "What is
// PagedAttention and what did it change in LLM serving" / "What is
// PagedAttention, simply": the prompt phase runs over the same paged cache).
// What changes is who loads what.  A cluster of two CTAs on two SMs takes a
// work item of 256 rows (new token, head of one kv head's group) of one
// sequence and kv head; CTA r keeps rows 128 r .. 128 r + 127 with its own S /
// P buffers and O in its own TMEM, exactly as the one-SM kernel does.  The
// products are UMMAs of M = 256 issued by CTA 0 for both:
//   S = Q . K_tile^T   A = Q (each CTA its 128 rows), B = the key tile split by
//                      N: CTA r holds keys [r N/2, (r + 1) N/2) of the tile;
//   O += P . V_tile    A = P (each CTA's TMEM), B = the value tile split by N:
//                      CTA r holds head_dim [64 r, 64 r + 64) of all its keys.
// So each SM loads half of every key tile and half of every value tile: 32 KB
// per 128-key tile instead of 64 KB, for the same tensor-core work per SM.
// Every load is a plain TMA copy (no multicast) into the loading CTA's own
// shared memory that signals CTA 0's barrier (the cta_group::2 form of the
// copy); completions of the products reach both CTAs through a multicast
// tcgen05.commit.
//
// Warps (per CTA): 0 the key producer (in CTA 0 also the item scheduler, which
// hands every item to both CTAs through a four-slot ring in each CTA's shared
// memory) and the loads of the CTA's Q rows, 6 the value producer, 1 the TMEM
// allocation (both CTAs) and, in CTA 0, the UMMA issuer, 2..5 the softmax and
// epilogue of the CTA's 128 rows.  Barriers the issuer waits on live in CTA 0
// and count both CTAs' arrivals; every other wait is on the waiting CTA's own
// barriers.  Waits are bounded; an abort in one CTA is passed to the other.
//
// Shared memory per CTA (1024-byte aligned, 128-byte swizzled rows): Q 2 x
// 32 KB, key halves 4 x 16 KB (two 64-column blocks of 64 rows), value halves
// 4 x 16 KB (eight 16-key groups of 16 rows x this CTA's 64 columns).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_tc.cuh"
#include "prefill_launch.h"
#include "tc5_ptx.cuh"

namespace pa {
namespace t5p {

using namespace t5;  // the shared PTX wrappers
using tc::kFull;

constexpr int kRows = 128;                   // query rows per CTA
constexpr int kPairRows = 2 * kRows;         // rows per item
constexpr int kKeys = 128;                   // keys per tile (the pair's S product N)
constexpr int kHalfKeys = kKeys / 2;         // keys of a full tile one CTA loads
constexpr int kD = 128;
constexpr int kThreads = 224;
constexpr int kVWarp = 6;
constexpr int kQColBlock = kRows * 128;      // 64 columns of the CTA's 128 rows: 16 KB
constexpr int kQTileBytes = 2 * kQColBlock;
constexpr int kKColBlock = kHalfKeys * 128;  // 64 columns of 64 keys: 8 KB
constexpr int kKHalfBytes = 2 * kKColBlock;
constexpr int kGroupBytes = 16 * 128;        // 16 rows of 64 columns: 2 KB
constexpr int kVHalfBytes = (kKeys / 16) * kGroupBytes;
constexpr int kKStages = 4;
constexpr int kVStages = 4;
constexpr int kQOff = 0;
constexpr int kKOff = 2 * kQTileBytes;
constexpr int kVOff = kKOff + kKStages * kKHalfBytes;
constexpr int kRing = kVOff + kVStages * kVHalfBytes;  // 192 KB
constexpr int kRingSlots = 4;
constexpr int kItemReaders = 7 + 6;  // CTA 0: V producer, issuer (twice), 4 softmax warps;
                                     // CTA 1: K producer, V producer, 4 softmax warps
constexpr int kSmem = 1024 + kRing + 512;
constexpr uint32_t kTmemCols = 512;
constexpr int kSBuf = 3;
constexpr uint32_t kColS = 0, kColO = kSBuf * kKeys;
constexpr float kSlack = 8.f;
constexpr long long kSpinLimit = 1ll << 31;

// ---- cluster and cta_group::2 wrappers ----
__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t at_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ void arrive_cl(uint32_t cl_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_bar)
               : "memory");
}
__device__ __forceinline__ void arrive_expect_cl(uint32_t cl_bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], %1;"
               ::"r"(cl_bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void st_cl_u32(uint32_t cl_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cl_addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cl_s64(uint32_t cl_addr, int64_t v) {
  asm volatile("st.shared::cluster.s64 [%0], %1;" ::"r"(cl_addr), "l"(v) : "memory");
}
__device__ __forceinline__ bool try_wait_cl(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool test_wait_cl(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// false after ~2^31 clock cycles or 2^24 polls, whichever comes first
__device__ __forceinline__ bool wait_bounded_cl(uint32_t bar, uint32_t parity) {
  if (try_wait_cl(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 0; i < (1u << 24); ++i) {
    if (try_wait_cl(bar, parity)) return true;
    if (clock64() - t0 > kSpinLimit) break;
  }
  return false;
}

// A CTA's abort flag, and the peer's, set together.
struct Abort {
  volatile int32_t* mine;
  uint32_t peer_cl;
  __device__ void raise() const {
    *mine = 1;
    st_cl_u32(peer_cl, 1u);
  }
};

// Warp-uniform bounded wait that gives up at once after an abort (reporting a
// timeout, and aborting both CTAs, when its own wait runs out).
__device__ __forceinline__ bool wait_ok2(uint32_t bar, uint32_t parity, const Abort& ab,
                                         int32_t* dev_error) {
  bool done = false;
  if (!*ab.mine) done = wait_bounded_cl(bar, parity);
  done = __all_sync(kFull, done);
  if (!done && (threadIdx.x & 31) == 0) {
    if (!*ab.mine) report(dev_error, PA_DEVERR_TIMEOUT);
    ab.raise();
  }
  return done;
}

// kind::f16 instruction descriptor for M = 256 (the pair): fp32 accumulator,
// A / B fp16 (0) or bf16 (1), A K-major, B K-major (0) or MN-major (1), N = n.
__host__ __device__ constexpr uint32_t idesc2(uint32_t ab_format, uint32_t b_major, uint32_t n) {
  return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (b_major << 16) | ((n >> 3) << 17) |
         ((kPairRows >> 4) << 24);
}

__device__ __forceinline__ void mma2_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t id,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;"
      "\n\t}"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(id), "r"(accumulate), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void mma2_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t id,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, "
      "p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b), "r"(id), "r"(accumulate), "r"(0u)
      : "memory");
}

// Arrive on the barrier at this offset in both CTAs once the issued products complete.
__device__ __forceinline__ void commit2(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar), "h"(static_cast<uint16_t>(3))
      : "memory");
}

// TMA tile loads into this CTA's shared memory that signal a barrier in either CTA.
__device__ __forceinline__ void tma2_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                        uint32_t cl_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x),
      "r"(y), "r"(cl_bar)
      : "memory");
}
__device__ __forceinline__ void tma2_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                        uint32_t cl_bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(z), "r"(cl_bar)
      : "memory");
}

// Byte offset of 16-byte chunk c (0..15) of row r in a Q tile (64-column blocks
// of 128 rows) and in a key half (64-column blocks of 64 rows).
__device__ __forceinline__ uint32_t q_off(int r, int c) {
  return (c >> 3) * kQColBlock + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}
__device__ __forceinline__ uint32_t k_off(int r, int c) {
  return (c >> 3) * kKColBlock + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}
// Chunk c (0..7) of row rr of 16-key group k of a value half.
__device__ __forceinline__ uint32_t v_off(int k, int rr, int c) {
  return k * kGroupBytes + rr * 128 + (((c & 7) ^ (rr & 7)) << 4);
}

// One work item: 256 rows of sequence b, kv head g (CTA r: rows r0 + 128 r ..).
struct Item {
  int b, g, q0, r0, rows, past, n_keys, n_tiles, n_last;
};

// Item w: (sequence, kv head) w / tiles, its 256-row query tile tiles - 1 - w %
// tiles (latest first).  n_last: the last tile's keys rounded up to 32, so each
// CTA's half of it is whole 16-key groups.
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
  it.r0 = tile_q * kPairRows;
  if (it.r0 >= it.rows) return false;
  it.past = ctx - nq;
  it.n_keys = it.past + (min(it.r0 + kPairRows, it.rows) - 1) / a.group + 1;
  it.n_tiles = (it.n_keys + kKeys - 1) / kKeys;
  it.n_last = ((it.n_keys - (it.n_tiles - 1) * kKeys) + 31) & ~31;
  return true;
}

template <typename T>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap qmap,
                        const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap,
                        const __grid_constant__ CUtensorMap omap, PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase + kRing);
  const uint32_t rank = cta_rank();
  const bool leader = rank == 0;
  // Barriers (the same offsets in both CTAs).  In CTA 0, with both CTAs'
  // arrivals: k_full, v_full (per stage), q_full (per Q tile), p_full (per S /
  // P buffer), o_free, item_empty (per ring slot).  In each CTA, from the
  // multicast commits: k_empty, v_empty, s_full, pv_done, final; and its own:
  // q_empty, item_full, staged, read.
  int nb = 0;
  auto bar_at = [&](int n) {
    const uint32_t b = tc::smem_u32(&bars[nb]);
    nb += n;
    return b;
  };
  const uint32_t b_k_full = bar_at(kKStages), b_k_empty = bar_at(kKStages);
  const uint32_t b_v_full = bar_at(kVStages), b_v_empty = bar_at(kVStages);
  const uint32_t b_s_full = bar_at(kSBuf), b_p_full = bar_at(kSBuf), b_pv_done = bar_at(kSBuf);
  const uint32_t b_q_full = bar_at(2), b_q_empty = bar_at(2);
  const uint32_t b_o_free = bar_at(1), b_final = bar_at(1);
  const uint32_t b_item_full = bar_at(kRingSlots), b_item_empty = bar_at(kRingSlots);
  const uint32_t b_staged = bar_at(1), b_read = bar_at(1);
  const int kNB = nb;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNB);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(bars + kNB + 1);
  volatile int64_t* item_q = reinterpret_cast<volatile int64_t*>(bars + kNB + 2);  // the ring
  const Abort ab{abort_flag, at_rank(tc::smem_u32(const_cast<int32_t*>(abort_flag)), rank ^ 1u)};

  const int64_t n_items = static_cast<int64_t>(a.tiles) * a.num_kv_heads * a.batch;
  const int G = a.group;
  const int bs = a.block_size;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kAB = PrefillPSplit<T>::value ? 1u : 0u;  // operand format: bf16 1, fp16 0

  if (threadIdx.x == 0) {
    for (int i = 0; i < kKStages; ++i) {
      tc::mbar_init(b_k_full + 8 * i, 2);
      tc::mbar_init(b_k_empty + 8 * i, 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      tc::mbar_init(b_v_full + 8 * i, 2);
      tc::mbar_init(b_v_empty + 8 * i, 1);
    }
    for (int i = 0; i < kSBuf; ++i) {
      tc::mbar_init(b_s_full + 8 * i, 1);
      tc::mbar_init(b_p_full + 8 * i, 8);
      tc::mbar_init(b_pv_done + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(b_q_full + 8 * i, 2);
      tc::mbar_init(b_q_empty + 8 * i, 1);
    }
    tc::mbar_init(b_o_free, 8);
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
    // both CTAs' warp 1 allocate together, into the same slot offset
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(tc::smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  cluster_sync();  // barriers initialised and TMEM allocated in both CTAs
  fence_after();
  const uint32_t tmem = *tmem_slot;

  // A barrier of CTA 0 (by its local offset) as a cluster address, for arrivals
  // from either CTA.
  auto in_leader = [](uint32_t local_bar) { return at_rank(local_bar, 0); };

  // The ring's item ig: the item index, or -1 after the last.
  auto ring_read = [&](int ig) -> int64_t {
    const int slot = ig % kRingSlots;
    if (!wait_ok2(b_item_full + 8 * slot, (ig / kRingSlots) & 1, ab, a.dev_error)) return -1;
    const int64_t w = item_q[slot];
    __syncwarp();
    if (lane == 0) arrive_cl(in_leader(b_item_empty + 8 * slot));
    return w;
  };

  if (warp == 0 || warp == kVWarp) {
    // ======================== Q and K / V producers =========================
    const int which = warp == 0 ? 0 : 1;  // 0: keys (and Q), 1: values
    const int n_st = which ? kVStages : kKStages;
    const uint32_t full0 = which ? b_v_full : b_k_full;
    const uint32_t empty0 = which ? b_v_empty : b_k_empty;
    const uint32_t ring = base + (which ? kVOff : kKOff);
    const uint32_t stage_bytes = which ? kVHalfBytes : kKHalfBytes;
    const T* src = static_cast<const T*>(which ? a.v_cache : a.k_cache);
    const CUtensorMap* map = which ? &vmap : &kmap;
    int tg = 0;  // tiles of this CTA so far
    bool live = true;
    int64_t w_static = cluster_index();
    for (int ig = 0; live; ++ig) {
      Item it;
      int64_t w = -1;
      if (which == 0 && leader) {
        // take the next item that has work (reporting invalid lengths) and pass
        // it to both CTAs; -1 after the last
        const int slot = ig % kRingSlots;
        if (ig >= kRingSlots &&
            !wait_ok2(b_item_empty + 8 * slot, ((ig / kRingSlots) - 1) & 1, ab, a.dev_error))
          break;
        if (lane == 0) {
          for (;;) {
            if (a.sched) {
              w = atomicAdd(reinterpret_cast<unsigned long long*>(a.sched), 1ull);
            } else {
              w = w_static;
              w_static += cluster_count();
            }
            if (w >= n_items) {
              w = -1;
              break;
            }
            if (item_at(a, w, it, true)) break;
          }
          const uint32_t slot_addr = tc::smem_u32(const_cast<int64_t*>(&item_q[slot]));
          item_q[slot] = w;
          st_cl_s64(at_rank(slot_addr, 1), w);
          arrive_cl(at_rank(b_item_full + 8 * slot, 0));
          arrive_cl(at_rank(b_item_full + 8 * slot, 1));
        }
        w = __shfl_sync(kFull, w, 0);
      } else {
        w = ring_read(ig);
      }
      if (w < 0) break;
      item_at(a, w, it, false);
      const int cr0 = it.r0 + kRows * static_cast<int>(rank);  // this CTA's first row
      if (which == 0) {
        // this CTA's 128 Q rows: 128 / G tokens x the G heads of kv head g, one
        // {64, G, 128 / G} box per 64-column block (rows past the sequence are
        // other tokens or zeros; their rows are never stored)
        const int qb = ig & 1;
        if (ig >= 2 && !wait_ok2(b_q_empty + 8 * qb, ((ig >> 1) - 1) & 1, ab, a.dev_error))
          break;
        if (lane == 0) {
          const uint32_t qf = in_leader(b_q_full + 8 * qb);
          arrive_expect_cl(qf, kQTileBytes);
          const uint32_t qs = base + kQOff + qb * kQTileBytes;
          tma2_3d(qs, &qmap, 0, it.g * G, it.q0 + cr0 / G, qf);
          tma2_3d(qs + kQColBlock, &qmap, 64, it.g * G, it.q0 + cr0 / G, qf);
        }
      }
      const int32_t* bt = a.block_tables + static_cast<int64_t>(it.b) * a.max_blocks;
      for (int t = 0; t < it.n_tiles; ++t, ++tg) {
        const int stage = tg % n_st;
        const int n_tile = t == it.n_tiles - 1 ? it.n_last : kKeys;
        // keys: this CTA's half of the tile, 16-key groups k < n_tile / 32;
        // values: every 16-key group of the tile, this CTA's 64 columns
        const int n_grp = which ? n_tile / 16 : n_tile / 32;
        const int key0 = t * kKeys + (which ? 0 : static_cast<int>(rank) * (n_tile / 2));
        const int key_mine = key0 + 16 * (lane & 7);
        int id_mine = (lane < n_grp && key_mine < it.n_keys) ? __ldg(&bt[key_mine / bs]) : -1;
        if (lane < n_grp && key_mine < it.n_keys && (id_mine < 0 || id_mine >= a.num_blocks)) {
          if (which == 0) report(a.dev_error, PA_DEVERR_BAD_BLOCK);
          id_mine = -1;
        }
        // whole groups in a valid block go by tensor map; the group holding key
        // n_keys - 1 when it is partial, groups past the keys (inside the
        // rounded-up last tile) and groups of invalid blocks, by hand with zeros
        // in the rows that hold no key
        const uint32_t tma_mask =
            __ballot_sync(kFull, lane < n_grp && id_mine >= 0 && key_mine + 16 <= it.n_keys);
        const uint32_t hand_mask = __ballot_sync(kFull, lane < n_grp) & ~tma_mask;
        const int row_mine =
            (id_mine < 0 ? 0 : id_mine * a.num_kv_heads + it.g) * bs + key_mine % bs;
        if (tg >= n_st && !wait_ok2(empty0 + 8 * stage, ((tg / n_st) - 1) & 1, ab, a.dev_error)) {
          live = false;
          break;
        }
        const uint32_t dst = ring + stage * stage_bytes;
        if (hand_mask) {
          for (int k = 0; k < 8; ++k) {
            if (!(hand_mask >> k & 1)) continue;
            const int id = __shfl_sync(kFull, id_mine, k);
            const int key = key0 + 16 * k;
            const int valid = id >= 0 ? max(0, min(16, it.n_keys - key)) : 0;
            const T* rows0 =
                src + (static_cast<int64_t>(id < 0 ? 0 : id * a.num_kv_heads + it.g) * bs +
                       (key % bs)) * kD;
            if (which) {
              for (int i = lane; i < 16 * 8; i += 32) {  // 16 rows x this CTA's 8 chunks
                const int rr = i >> 3, c = i & 7;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (rr < valid)
                  v = __ldg(reinterpret_cast<const uint4*>(rows0 + rr * kD) + 8 * rank + c);
                st_shared4(dst + v_off(k, rr, c), v);
              }
            } else {
              for (int i = lane; i < 16 * 16; i += 32) {  // 16 rows x 16 chunks
                const int rr = i >> 4, c = i & 15;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (rr < valid) v = __ldg(reinterpret_cast<const uint4*>(rows0 + rr * kD) + c);
                st_shared4(dst + k_off(16 * k + rr, c), v);
              }
            }
          }
          // generic writes above are read by the tensor core (async proxy)
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        const uint32_t full = in_leader(full0 + 8 * stage);
        __syncwarp();
        if (lane == 0) {
          const uint32_t per_group = which ? kGroupBytes : 2 * kGroupBytes;
          arrive_expect_cl(full, __popc(tma_mask) * per_group);
        }
        __syncwarp();
        if (tma_mask >> lane & 1) {
          const int k = lane;
          if (which) {
            tma2_2d(dst + k * kGroupBytes, map, 64 * static_cast<int>(rank), row_mine, full);
          } else {
            tma2_2d(dst + 16 * k * 128, map, 0, row_mine, full);
            tma2_2d(dst + kKColBlock + 16 * k * 128, map, 64, row_mine, full);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (leader) {
      // =========================== UMMA issuer ==============================
      // As in the one-SM kernel: S_n needs K_n (both halves), its item's Q (both
      // CTAs) and its TMEM buffer, free once P_{n-3} . V has completed; P_n . V
      // needs P_n (both CTAs) and V_n (both halves), and for an item's first
      // tile the previous item's O read out in both CTAs.
      struct Cursor {
        int ig, t, state;  // state: 0 waiting for an item, 1 on one, 2 past the last
        Item it;
      };
      const bool elected = lane == 0;
      auto try_fetch = [&](Cursor& c) {  // non-blocking; warp-uniform
        const int slot = c.ig % kRingSlots;
        bool got = false;
        if (elected) got = test_wait_cl(b_item_full + 8 * slot, (c.ig / kRingSlots) & 1);
        if (!__shfl_sync(kFull, got, 0)) return false;
        const int64_t w =
            __shfl_sync(kFull, elected ? static_cast<long long>(item_q[slot]) : 0ll, 0);
        __syncwarp();
        if (elected) arrive_cl(in_leader(b_item_empty + 8 * slot));
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
          if (elected)
            ready = (ns < kSBuf || test_wait_cl(b_pv_done + 8 * (ns % kSBuf),
                                                ((ns - kSBuf) / kSBuf) & 1)) &&
                    test_wait_cl(b_k_full + 8 * (ns % kKStages), (ns / kKStages) & 1) &&
                    (cs.t > 0 || test_wait_cl(b_q_full + 8 * (cs.ig & 1), (cs.ig >> 1) & 1));
          if (__shfl_sync(kFull, ready, 0)) {
            if (elected) {
              fence_after();
              const uint32_t q_s = base + kQOff + (cs.ig & 1) * kQTileBytes;
              const uint32_t kt = base + kKOff + (ns % kKStages) * kKHalfBytes;
              const uint32_t d = tmem + kColS + (ns % kSBuf) * kKeys;
              const uint32_t id =
                  idesc2(kAB, 0, cs.t == cs.it.n_tiles - 1 ? cs.it.n_last : kKeys);
#pragma unroll
              for (int s = 0; s < kD / 16; ++s) {
                const uint32_t qo = (s >> 2) * kQColBlock + (s & 3) * 32;
                const uint32_t ko = (s >> 2) * kKColBlock + (s & 3) * 32;
                mma2_ss(d, smem_desc(q_s + qo, 16, 1024), smem_desc(kt + ko, 16, 1024), id,
                        s > 0);
              }
              commit2(b_s_full + 8 * (ns % kSBuf));
              commit2(b_k_empty + 8 * (ns % kKStages));  // K_ns may be refilled
            }
            ++ns;
            advance(cs);
            progress = true;
          }
        }
        if (cp.state == 1 && npv < ns) {
          bool ready = false;
          if (elected)
            ready = test_wait_cl(b_p_full + 8 * (npv % kSBuf), (npv / kSBuf) & 1) &&
                    test_wait_cl(b_v_full + 8 * (npv % kVStages), (npv / kVStages) & 1) &&
                    (cp.t > 0 || cp.ig == 0 || test_wait_cl(b_o_free, (cp.ig - 1) & 1));
          if (__shfl_sync(kFull, ready, 0)) {
            if (elected) {
              fence_after();
              const uint32_t vt = base + kVOff + (npv % kVStages) * kVHalfBytes;
              const uint32_t p = tmem + kColS + (npv % kSBuf) * kKeys;  // P head: columns 0..63
              const int steps = cp.t == cp.it.n_tiles - 1 ? cp.it.n_last / 16 : kKeys / 16;
              constexpr uint32_t kIdO = idesc2(kAB, 1, kD);
              for (int s = 0; s < steps; ++s) {
                // group s: this CTA's 64 columns of 16 keys, 8-key core groups 1 KB apart
                const uint64_t bd = smem_desc(vt + s * kGroupBytes, kGroupBytes, 1024);
                mma2_ts(tmem + kColO, p + 8 * s, bd, kIdO, (cp.t > 0 || s > 0) ? 1u : 0u);
                if (PrefillPSplit<T>::value) mma2_ts(tmem + kColO, p + 64 + 8 * s, bd, kIdO, 1u);
              }
              commit2(b_v_empty + 8 * (npv % kVStages));  // V_npv may be refilled
              commit2(b_pv_done + 8 * (npv % kSBuf));     // O holds this item's P . V so far
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
        ab.raise();
      }
      // every product issued has completed (in both CTAs) before TMEM is released
      if (elected) commit2(b_final);
      __syncwarp();
      wait_bounded_cl(b_final, 0);
    }
  } else {
    // ======================= softmax and epilogue ===========================
    const int quarter = warp & 3;            // TMEM lanes 32 quarter .. +31
    const int r = 32 * quarter + lane;       // this thread's row of the CTA's 128
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
    const float c = a.scale_log2;  // > 0
    int tg = 0, n_ragged = 0;
    bool ok = true;
    for (int ig = 0;; ++ig) {
      const int64_t w = ring_read(ig);
      if (w < 0) break;
      Item it;
      item_at(a, w, it, false);
      const int cr0 = it.r0 + kRows * static_cast<int>(rank);
      const int grow = cr0 + r;
      const int pos = grow < it.rows ? it.past + grow / G : -1;
      float m = -INFINITY;  // running reference, scaled (log2) domain
      float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
      for (int t = 0; t < it.n_tiles; ++t, ++tg) {
        if (ok) ok = wait_ok2(b_s_full + 8 * (tg % kSBuf), (tg / kSBuf) & 1, ab, a.dev_error);
        if (!ok) continue;
        fence_after();
        const uint32_t sp = trow + kColS + (tg % kSBuf) * kKeys;
        uint32_t su[4][32];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_ld32_issue(sp + 32 * ch, su[ch]);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_ld_wait(su[ch]);
        float sv[4][32];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[ch][i] = __uint_as_float(su[ch][i]);
        // causal mask where the tile reaches past some row's position (and for
        // rows past the sequence); columns past the tile's N are masked too
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
        // reference and rescales its row of O once the previous P . V is done
        const bool moves = mx > m + kSlack;
        if (__any_sync(kFull, moves)) {
          const float mnew = moves ? mx : m;
          const float alpha = m == -INFINITY ? 0.f : ex2(m - mnew);
          if (t > 0) {
            ok = wait_ok2(b_pv_done + 8 * ((tg - 1) % kSBuf), ((tg - 1) / kSBuf) & 1, ab,
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
        if (lane == 0) arrive_cl(in_leader(b_p_full + 8 * (tg % kSBuf)));
      }
      // epilogue: O / l once the item's last P . V is done, staged in the item's
      // Q tile (its S products are complete then) in the Q layout
      const int qb = ig & 1;
      const uint32_t stage_out = base + kQOff + qb * kQTileBytes;
      if (ok)
        ok = wait_ok2(b_pv_done + 8 * ((tg - 1) % kSBuf), ((tg - 1) / kSBuf) & 1, ab,
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
            st_shared4(stage_out + q_off(r, 4 * ch + k), v);
          }
        }
      }
      // O has been read: the next item's first P . V may overwrite it
      fence_before();
      __syncwarp();
      if (lane == 0) arrive_cl(in_leader(b_o_free));
      // the staged tile is read by TMA (async proxy) or by the other warps
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(b_staged);
      if (cr0 + kRows <= it.rows) {
        // a whole tile: two TMA stores, the same boxes as the Q loads
        if (warp == 2) {
          const bool go = wait_ok2(b_staged, ig & 1, ab, a.dev_error);
          if (lane == 0) {
            if (go) {
              tma_store_3d(&omap, 0, it.g * G, it.q0 + cr0 / G, stage_out);
              tma_store_3d(&omap, 64, it.g * G, it.q0 + cr0 / G, stage_out + kQColBlock);
              asm volatile("cp.async.bulk.commit_group;" ::: "memory");
              asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            }
            tc::mbar_arrive(b_q_empty + 8 * qb);
          }
        }
      } else {
        // the sequence's ragged end (or rows wholly past it): the valid rows, as
        // whole 16-byte chunks
        if (wait_ok2(b_staged, ig & 1, ab, a.dev_error)) {
          const int i = threadIdx.x - 64;  // 0..127
          const int cc = i & 15;
#pragma unroll 4
          for (int k = 0; k < kRows / 8; ++k) {
            const int rr = 8 * k + (i >> 4);
            const int gr = cr0 + rr;
            if (gr < it.rows) {
              const int tok = gr / G, hh = gr - tok * G;
              T* dst = static_cast<T*>(a.out) +
                       (static_cast<int64_t>(it.q0 + tok) * a.num_q_heads + it.g * G + hh) * kD;
              reinterpret_cast<uint4*>(dst)[cc] = ld_shared4(stage_out + q_off(rr, cc));
            }
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(b_read);
        if (warp == 2) {
          wait_ok2(b_read, n_ragged & 1, ab, a.dev_error);
          if (lane == 0) tc::mbar_arrive(b_q_empty + 8 * qb);
        }
        ++n_ragged;
      }
    }
    if (threadIdx.x == 64) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  // every role of both CTAs is done (and CTA 0's issuer has seen every product
  // complete): no CTA touches the other's shared memory any more, and TMEM can
  // be released
  fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols) : "memory");
  }
  // the last CTA to finish returns the scheduling counter to zero
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
  auto kern = prefill_pair_kernel<T>;
  static bool raised[64] = {};
  static int max_clusters[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < 64;
  if (!cached || !raised[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    if (cached) raised[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = stream;
  int n_clusters = cached ? max_clusters[dev] : 0;
  if (n_clusters == 0) {
    cfg.gridDim = dim3(2);
    e = cudaOccupancyMaxActiveClusters(&n_clusters, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (n_clusters < 1) return cudaErrorInvalidConfiguration;
    if (cached) max_clusters[dev] = n_clusters;
  }
  const int64_t n_items = static_cast<int64_t>(a.tiles) * a.num_kv_heads * a.batch;
  // persistent (one cluster per SM pair that fits) with a scheduling counter,
  // else one item per cluster
  const int64_t cap = a.sched ? n_clusters : (INT32_MAX / 2);
  const int64_t clusters = n_items < cap ? n_items : cap;
  if (clusters <= 0) return cudaSuccess;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
  return cudaLaunchKernelEx(&cfg, kern, qmap, kmap, vmap, omap, a);
}

}  // namespace t5p

cudaError_t launch_prefill_pair(PrefillArgs a, pa_dtype dtype, const CUtensorMap& qmap,
                                const CUtensorMap& kmap2d, const CUtensorMap& vmap2d,
                                const CUtensorMap& omap, cudaStream_t stream) {
  a.tiles = static_cast<int>((static_cast<int64_t>(a.max_q) * a.group + t5p::kPairRows - 1) /
                             t5p::kPairRows);
  return dtype == PA_F16 ? t5p::launch_t<__half>(a, qmap, kmap2d, vmap2d, omap, stream)
                         : t5p::launch_t<__nv_bfloat16>(a, qmap, kmap2d, vmap2d, omap, stream);
}

}  // namespace pa
