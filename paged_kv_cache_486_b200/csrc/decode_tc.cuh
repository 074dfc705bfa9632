// Paged decode attention on B200 tensor cores, KV tiles staged by TMA: the
// kernel skeleton shared by every cache format.
//
// Shape of the work.  For one (sequence b, kv head) the G query heads that
// share the KV head ("KV Cache for intermediates..." / "The four solutions",
// GQA) form an 8-column operand, so each 16-token tile of keys and values is
// read from HBM once per KV head and used by all G heads:
//   S^T[16 tok x 8 heads] = K[16 x D] . Q^T[D x 8]          (mma m16n8k16)
//   O^T[D x 8 heads]     += V^T[D x 16] . P^T[16 x 8]       (mma m16n8k16)
// Heads beyond G (G < 8) are zero query rows whose results are not stored.
// Scores are kept in base-2 units (scale * log2 e) with an online softmax in
// fp32 registers.  The exchange of P^T between the two products is a register
// transpose (movmatrix), so P never goes through shared memory.
//
// Data movement.  Every warp is an independent worker (see decode_common.cuh)
// with its own ring of stage buffers.  Lane 0 issues, a ring's depth ahead of
// the consumer, the TMA loads of a stage (16 tokens of one KV block and kv
// head); each stage signals an mbarrier with its byte count, and every wait on
// it is bounded in time.  The consumer copies a stage into registers and hands
// the slot straight back to TMA before it computes.  Block ids come from the
// block table through a per-warp window of 32 ids held one per lane and loaded
// one window ahead.
//
// Cache formats.  What a stage holds, how it is loaded and how its fragments
// enter the two products is a policy class (`Tiles`):
//   Tiles16 (decode_tc.cu):   fp16 / bf16 keys and values;
//   Tiles8  (decode_int8.cu): 8-bit codes with a per-token fp32 scale.
// A policy provides:
//   kStages, kStageBytes (bytes TMA delivers per stage), kRingBytes (shared
//   memory of all rings, a multiple of 1024), kConsumerRegs / kProducerRegs
//   (the register split, below), Maps (tensor maps, a kernel
//   parameter), Frag (one stage in registers), Seg (per-segment state);
//   prefetch(maps); issue(maps, a, ring0, warp, slot, tile, tok, bar) (lane 0);
//   q_off(kc, cq, half) (head_dim offset of a query fragment register);
//   prep_q(qf, seg, a, lane) (once per segment, after seg.reset(), on the
//     segment's query fragments: whatever the policy's products need);
//   load(a, ring0, warp, slot, n_valid, lane, frag);
//   scores(frag, qf, seg, a, n_valid, lane, t[4]);
//   pre_pv(frag, o, seg, n_valid, lane) (right after scores: the value
//     product's work that does not need P, overlapping the score products);
//   pv(frag, p[4], o, seg, n_valid, lane);
//   rescale(seg, a0, a1) (the softmax reference moved: what the policy keeps
//     alongside O is scaled like O's heads 2cq, 2cq + 1);
//   finish(o, seg) (at the segment's end, before O is scaled and written).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "decode_common.cuh"
#include "decode_launch.h"

namespace pa {
namespace tc {

constexpr int kTok = 16;     // tokens per stage (one mma tile of keys)
constexpr int kWarps = 8;    // workers per CTA
constexpr unsigned kFull = 0xffffffffu;
constexpr float kSlack = 8.f;  // base-2 units a score may exceed the softmax reference

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with `parity` to complete; false after ~2^31 clock
// cycles (about a second) or 2^24 polls, whichever comes first.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t i = 0; i < (1u << 24); ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > (1ll << 31)) break;
  }
  return false;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

constexpr int kBoxBytes = kTok * 64 * 2;  // one 16 x 64 box of 16-bit elements

// The tile of 16 rows x D lands as D/64 column blocks of 16 rows x 64 columns
// (block h = columns [64h, 64h + 64)).  With a 3-D map {64 columns, rows, D/64
// column blocks} it is one copy; with a 2-D map {D, rows} it is one copy per
// column block.
template <int D>
__device__ __forceinline__ void tma_tile(uint32_t dst, const CUtensorMap* map, int row,
                                         bool three_d, uint32_t bar) {
  if (three_d) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(row), "r"(0), "r"(bar)
        : "memory");
    return;
  }
#pragma unroll
  for (int h = 0; h < D / 64; ++h) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst + h * kBoxBytes),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(64 * h), "r"(row), "r"(bar)
        : "memory");
  }
}

// Byte address of 16-byte chunk `chunk` (0 .. D/8-1) of token row `tok`: box
// chunk / 8, line tok, position (chunk mod 8) ^ (tok mod 8) (128-byte swizzle).
__device__ __forceinline__ uint32_t swz(uint32_t tile, int tok, int chunk) {
  return tile + (chunk >> 3) * kBoxBytes + tok * 128 + (((chunk & 7) ^ (tok & 7)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

template <typename T>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4],
                                         const uint32_t (&b)[2]);

template <>
__device__ __forceinline__ void mma16816<__half>(float (&c)[4], const uint32_t (&a)[4],
                                                 const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

template <>
__device__ __forceinline__ void mma16816<__nv_bfloat16>(float (&c)[4], const uint32_t (&a)[4],
                                                        const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <typename T>
__device__ __forceinline__ float2 unpack2(uint32_t x);
template <>
__device__ __forceinline__ float2 unpack2<__half>(uint32_t x) {
  return __half22float2(*reinterpret_cast<const __half2*>(&x));
}
template <>
__device__ __forceinline__ float2 unpack2<__nv_bfloat16>(uint32_t x) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x));
}

// Softmax weights as a head + tail pair of 16-bit values (p = head + tail up to
// ~16 significant bits), so that P . V keeps fp32-like accuracy even for bf16,
// whose 8-bit significand alone would cost ~2^-9 |v| wherever outputs cancel.
template <typename T>
__device__ __forceinline__ void split2(float a, float b, uint32_t& head, uint32_t& tail) {
  head = pack2<T>(a, b);
  const float2 h = unpack2<T>(head);
  tail = pack2<T>(a - h.x, b - h.y);
}

// What the producer lane tells the consumer about a stage it issued.
constexpr int kHasData = 1;       // the tile was loaded (its block id was in range)
constexpr int kSegStart = 2;      // first stage of a segment
constexpr int kSegEnd = 4;        // last stage of a segment
constexpr int kComplete = 8;      // the segment is a whole (sequence, kv head)
constexpr int kFirstInRange = 16; // the segment holds its range's first unit (piece slot 0)
constexpr int kMoreInRange = 32;  // the range continues after this (sequence, kv head)

struct StageMeta {
  int32_t b;
  int32_t kvh_flags;  // kv head << 16 | flags
  int32_t n_valid;    // tokens of the stage inside the context (1 .. kTok)
  int32_t range;      // range the stage belongs to (piece slots)
};

// What the producer needs about one unit (one KV block of one (sequence, kv
// head) pair inside a range [r0, r1)), packed in four words.  Each lane of a
// warp computes the descriptor of one unit of a 32-unit window, a window
// ahead of its use, so the producer's per-stage work is four shuffles.
struct UnitDesc {
  int32_t id;   // physical block id (-1 past the range)
  int32_t bk;   // b << 16 | kv head
  int32_t j;    // logical block index in the sequence
  int32_t nf;   // tokens of the block inside the context | unit flags << 8
};

__device__ __forceinline__ UnitDesc unit_desc(const DecodeArgs& a, const int32_t* cum,
                                              const int32_t* ctx_s, int64_t u, int64_t r0,
                                              int64_t r1) {
  UnitDesc d{-1, 0, 0, 0};
  if (u >= r1) return d;
  const int Hkv = a.num_kv_heads, bs = a.block_size;
  const int b = find_seq(cum, a.batch, u, Hkv);
  const int nblk = cum[b + 1] - cum[b];
  const int rem = static_cast<int>(u - static_cast<int64_t>(Hkv) * cum[b]);  // < Hkv * nblk
  const int kvh = rem / nblk;
  const int j = rem - kvh * nblk;
  const int64_t pair0 = u - j, pair1 = pair0 + nblk;
  const int left = ctx_s[b] - j * bs;
  const int ntok = left < bs ? left : bs;
  const int flags = ((j == 0 || u == r0) ? kSegStart : 0) |
                    ((u + 1 == r1 || j + 1 == nblk) ? kSegEnd : 0) |
                    ((pair0 >= r0 && pair1 <= r1) ? kComplete : 0) |
                    (pair0 <= r0 ? kFirstInRange : 0) | (pair1 < r1 ? kMoreInRange : 0);
  d.id = __ldg(&a.block_tables[static_cast<int64_t>(b) * a.max_blocks + j]);
  d.bk = (b << 16) | kvh;
  d.j = j;
  d.nf = ntok | (flags << 8);
  return d;
}

__device__ __forceinline__ UnitDesc shfl_desc(const UnitDesc& d, int k) {
  return UnitDesc{__shfl_sync(kFull, d.id, k), __shfl_sync(kFull, d.bk, k),
                  __shfl_sync(kFull, d.j, k), __shfl_sync(kFull, d.nf, k)};
}


// Warp roles.  A CTA runs kWarps worker (consumer) warps and, paired with
// each, one producer warp (warp w + kWarps): the producer walks the worker's
// ranges and issues the copies of its stages into the worker's ring; the
// worker waits for a stage (the slot's "full" mbarrier, which counts the
// copied bytes), copies it into registers, releases the slot (its "empty"
// mbarrier) and computes.  Issue and math overlap instead of alternating in one
// warp.  Registers: the CTA is launched with kLaunchRegs per thread; producer
// warpgroups give most of theirs up (setmaxnreg.dec to kProducerRegs), worker
// warpgroups take them (setmaxnreg.inc to kConsumerRegs).  The two counts add
// up to twice the launch count, the most the hand-over can provide.  A policy
// may set its own split (P::kConsumerRegs, P::kProducerRegs); the 8-bit one
// gives its workers 208 (the codes' conversions need them) and its producers 48.
constexpr int kLaunchRegs = 128;
constexpr int kConsumerRegs = 216;
constexpr int kProducerRegs = 40;
static_assert(kConsumerRegs + kProducerRegs <= 2 * kLaunchRegs, "register split");
static_assert(kLaunchRegs * kWarps * 2 * 32 <= 65536, "launch registers");
constexpr int kDone = 64;  // stage metadata: the worker has no more stages

template <typename T, int D, class P>
__global__ void __launch_bounds__(2 * kWarps * 32, 1)
    decode_tc_kernel(const __grid_constant__ typename P::Maps maps, DecodeArgs a) {
  constexpr int KC = D / 16;  // 16-wide chunks of head_dim
  constexpr int kStages = P::kStages;
  static_assert(P::kConsumerRegs + P::kProducerRegs <= 2 * kLaunchRegs, "register split");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t ring0 = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (ring0 - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(gbase + P::kRingBytes);
  uint64_t* empty = full + kWarps * kStages;
  StageMeta* meta = reinterpret_cast<StageMeta*>(empty + kWarps * kStages);
  int32_t* cum = reinterpret_cast<int32_t*>(meta + kWarps * kStages);
  int32_t* ctx_s = cum + a.batch + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kWarps * kStages; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    P::prefetch(maps);
  }
  prefetch_tables(a);
  scan_context(a, cum, ctx_s);  // ends with __syncthreads()
  // Until here the kernel has read only context_lens and block_tables: with
  // overlap enabled this prologue runs while the preceding kernel finishes.
  wait_prior_grid();
  zero_empty_rows<T>(a, ctx_s);

  const int B = a.batch, Hkv = a.num_kv_heads, G = a.group, Hq = a.num_q_heads;
  const Split sp = make_split(static_cast<int64_t>(Hkv) * cum[B], a.workers);
  const int ww = warp % kWarps;  // the worker this warp belongs to
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kWarps + ww;
  const bool active = w < sp.W;  // the same for a worker and its producer
  const uint32_t full0 = smem_u32(&full[ww * kStages]);
  const uint32_t empty0 = smem_u32(&empty[ww * kStages]);
  StageMeta* wmeta = meta + ww * kStages;

  if (warp >= kWarps) {
    // =============================== producer ===============================
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(P::kProducerRegs));
    if (!active) return;
    int64_t prange = w;
    int64_t pr0 = sp.start(w);
    int64_t pend = sp.end(w);
    int64_t pu = pr0;   // next unit to enter
    int64_t win = pr0;  // first unit of the descriptor window
    UnitDesc dcur = unit_desc(a, cum, ctx_s, win + lane, pr0, pend);
    UnitDesc dnext = unit_desc(a, cum, ctx_s, win + 32 + lane, pr0, pend);
    UnitDesc cur{-1, 0, 0, 0};
    int psub = 0, pnsub = 0;
    int k = 0;  // stages issued
    for (;; ++k) {
      const int slot = k % kStages;
      if (k >= kStages) {
        // the worker must have released this slot's previous stage
        if (!__all_sync(kFull, mbar_wait_bounded(empty0 + slot * 8, ((k / kStages) - 1) & 1))) {
          if (lane == 0) report(a.dev_error, PA_DEVERR_TIMEOUT);
          break;
        }
      }
      bool more = true;
      if (psub == 0) {
        if (pu >= pend) {
          const int64_t chunk = sp.NC ? claim_chunk(a, lane) : sp.NC;
          if (chunk >= sp.NC) {
            more = false;
          } else {
            prange = sp.W + chunk;
            pr0 = pu = win = sp.start(prange);
            pend = sp.end(prange);
            dcur = unit_desc(a, cum, ctx_s, win + lane, pr0, pend);
            dnext = unit_desc(a, cum, ctx_s, win + 32 + lane, pr0, pend);
          }
        }
        if (more) {
          if (pu >= win + 32) {
            win += 32;
            dcur = dnext;
            dnext = unit_desc(a, cum, ctx_s, win + 32 + lane, pr0, pend);
          }
          cur = shfl_desc(dcur, static_cast<int>(pu - win));
          pnsub = ((cur.nf & 0xff) + kTok - 1) / kTok;
        }
      }
      const uint32_t bar = full0 + slot * 8;
      if (!more) {
        if (lane == 0) {
          wmeta[slot] = StageMeta{0, kDone, 0, 0};
          mbar_arrive(bar);
        }
        ++k;
        break;
      }
      const int uflags = cur.nf >> 8;
      const int left = (cur.nf & 0xff) - psub * kTok;
      const bool ok = cur.id >= 0 && cur.id < a.num_blocks;
      const int flags = (ok ? kHasData : 0) | (psub == 0 ? uflags & kSegStart : 0) |
                        (psub + 1 == pnsub ? uflags & kSegEnd : 0) |
                        (uflags & (kComplete | kFirstInRange | kMoreInRange));
      if (lane == 0) {
        const int kvh = cur.bk & 0xffff;
        wmeta[slot] = StageMeta{cur.bk >> 16, (kvh << 16) | flags, left < kTok ? left : kTok,
                                static_cast<int32_t>(prange)};
        if (ok) {
          mbar_arrive_expect_tx(bar, P::kStageBytes);
          P::issue(maps, a, ring0, ww, slot, cur.id * Hkv + kvh, psub * kTok, bar);
        } else {
          report(a.dev_error, PA_DEVERR_BAD_BLOCK);
          mbar_arrive(bar);
        }
      }
      if (++psub == pnsub) {
        psub = 0;
        ++pu;
      }
    }
    worker_finished(a, sp.W, lane);
    // copies still in flight land before the CTA's shared memory goes away
    for (int i = k - kStages > 0 ? k - kStages : 0; i < k; ++i)
      mbar_wait_bounded(full0 + (i % kStages) * 8, (i / kStages) & 1);
    return;
  }

  // ================================ worker ==================================
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(P::kConsumerRegs));
  if (!active) return;
  const int g = lane >> 2, cq = lane & 3;
  uint32_t qf[KC][2], qn[KC][2];
  int qn_b = -1, qn_kvh = -1;
  float o[KC][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  typename P::Seg seg;

  // Query fragments (B operand, k = head_dim, n = head) of pair (b, kvh): lane
  // (g, cq) holds two pairs of head g's query at the policy's offsets.
  auto load_q = [&](uint32_t (&dst)[KC][2], int b, int kvh) {
    const T* qb = static_cast<const T*>(a.q) + (static_cast<int64_t>(b) * Hq + kvh * G) * D;
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
      if (g < G) {
        dst[kc][0] = __ldg(reinterpret_cast<const uint32_t*>(qb + g * D + P::q_off(kc, cq, 0)));
        dst[kc][1] = __ldg(reinterpret_cast<const uint32_t*>(qb + g * D + P::q_off(kc, cq, 1)));
      } else {
        dst[kc][0] = dst[kc][1] = 0u;
      }
    }
  };

  for (int k = 0;; ++k) {
    const int slot = k % kStages;
    // all lanes take the same decision, so the warp never splits on a timeout
    // (a test of the failure path makes the first wait count as run out)
    if (!__all_sync(kFull, (k > 0 || !a.test_expire) &&
                               mbar_wait_bounded(full0 + slot * 8, (k / kStages) & 1))) {
      if (lane == 0) report(a.dev_error, PA_DEVERR_TIMEOUT);
      // let stages the producer issued after this one land before exiting
      for (int i = 1; i < kStages; ++i)
        mbar_wait_bounded(full0 + ((k + i) % kStages) * 8, ((k + i) / kStages) & 1);
      return;
    }
    const StageMeta md = wmeta[slot];
    if (md.kvh_flags & kDone) break;
    const int b = md.b, kvh = md.kvh_flags >> 16, flags = md.kvh_flags & 0xffff;

    if (flags & kSegStart) {
      if (qn_b == b && qn_kvh == kvh) {
#pragma unroll
        for (int kc = 0; kc < KC; ++kc) {
          qf[kc][0] = qn[kc][0];
          qf[kc][1] = qn[kc][1];
        }
      } else {
        load_q(qf, b, kvh);
      }
#pragma unroll
      for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
        for (int i = 0; i < 4; ++i) o[kc][i] = 0.f;
      }
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
      seg.reset();
      P::prep_q(qf, seg, a, lane);
      // start fetching the next pair's queries now; they are used only then
      qn_b = -1;
      if (flags & kMoreInRange) {
        int nb = b, nk = kvh + 1;
        if (nk == Hkv) {
          nk = 0;
          do {
            ++nb;
          } while (cum[nb + 1] == cum[nb]);
        }
        load_q(qn, nb, nk);
        qn_b = nb;
        qn_kvh = nk;
      }
    }

    const int n_valid = md.n_valid;
    const bool have = (flags & kHasData) != 0;
    // Move the stage into registers and hand the slot straight back.  The
    // arrive (release semantics) orders the warp's reads of the slot before the
    // producer's next copy into it; a policy that writes the slot itself fences
    // those writes against the copy (async proxy) inside load().
    typename P::Frag fr;
    if (have) P::load(a, ring0, ww, slot, n_valid, lane, fr);
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + slot * 8);

    if (have) {
      // scores of (row g, head 2cq), (g, 2cq+1), (g+8, 2cq), (g+8, 2cq+1), base-2
      // units, -inf past the context
      float t[4];
      P::scores(fr, qf, seg, a, n_valid, lane, t);
      P::pre_pv(fr, o, seg, n_valid, lane);
      // Lazy running maximum: weights are taken against the current reference m
      // unless some score of the stage is more than kSlack above it (then the
      // stage's maximum is reduced across the warp and the sums are rescaled).
      // Weights stay <= 2^kSlack; l and o share m, so the result is unchanged.
      float x0 = fmaxf(t[0], t[2]), x1 = fmaxf(t[1], t[3]);
      if (__any_sync(kFull, x0 > m0 + kSlack || x1 > m1 + kSlack)) {
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          x0 = fmaxf(x0, __shfl_xor_sync(kFull, x0, off));
          x1 = fmaxf(x1, __shfl_xor_sync(kFull, x1, off));
        }
        const float n0 = fmaxf(m0, x0), n1 = fmaxf(m1, x1);
        const float a0 = exp2f(m0 - n0), a1 = exp2f(m1 - n1);
        l0 *= a0;
        l1 *= a1;
#pragma unroll
        for (int kc = 0; kc < KC; ++kc) {
          o[kc][0] *= a0;
          o[kc][1] *= a1;
          o[kc][2] *= a0;
          o[kc][3] *= a1;
        }
        P::rescale(seg, a0, a1);
        m0 = n0;
        m1 = n1;
      }
      const float p[4] = {exp2f(t[0] - m0), exp2f(t[1] - m1), exp2f(t[2] - m0),
                          exp2f(t[3] - m1)};
      l0 += p[0] + p[2];
      l1 += p[1] + p[3];
      P::pv(fr, p, o, seg, n_valid, lane);
    }

    if (flags & kSegEnd) {
      P::finish(o, seg);
      float L0 = l0, L1 = l1;
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        L0 += __shfl_xor_sync(kFull, L0, off);
        L1 += __shfl_xor_sync(kFull, L1, off);
      }
      const float os = seg.out_scale();
      const int h0 = 2 * cq, h1 = 2 * cq + 1;
      if (flags & kComplete) {
        T* ob = static_cast<T*>(a.out) + (static_cast<int64_t>(b) * Hq + kvh * G) * D;
        const float i0 = os / L0, i1 = os / L1;
#pragma unroll
        for (int mt = 0; mt < KC; ++mt) {
          const int d = mt * 16 + g;
          if (h0 < G) {
            ob[h0 * D + d] = Num<T>::from_f(o[mt][0] * i0);
            ob[h0 * D + d + 8] = Num<T>::from_f(o[mt][2] * i0);
          }
          if (h1 < G) {
            ob[h1 * D + d] = Num<T>::from_f(o[mt][1] * i1);
            ob[h1 * D + d + 8] = Num<T>::from_f(o[mt][3] * i1);
          }
        }
      } else {
        const int pslot = (flags & kFirstInRange) ? 0 : 1;
        float* piece =
            a.ws_pieces + (static_cast<int64_t>(md.range) * 2 + pslot) * (G * (D + 2));
        if (g == 0) {
          if (h0 < G) { piece[h0] = m0; piece[G + h0] = L0; }
          if (h1 < G) { piece[h1] = m1; piece[G + h1] = L1; }
        }
        float* po = piece + 2 * G;
#pragma unroll
        for (int mt = 0; mt < KC; ++mt) {
          const int d = mt * 16 + g;
          if (h0 < G) {
            po[h0 * D + d] = o[mt][0] * os;
            po[h0 * D + d + 8] = o[mt][2] * os;
          }
          if (h1 < G) {
            po[h1 * D + d] = o[mt][1] * os;
            po[h1 * D + d + 8] = o[mt][3] * os;
          }
        }
        piece_done<T, D>(a, cum, b, kvh, sp, lane);
      }
    }
  }
}

// Shared memory of one CTA: the rings (1024-aligned), then per stage two
// mbarriers (full, empty) and a StageMeta, then the context scan (2 * batch + 1
// words).
template <class P>
inline size_t tc_smem_bytes(int batch) {
  return 1024 + P::kRingBytes + kWarps * P::kStages * (16 + sizeof(StageMeta)) +
         sizeof(int32_t) * (2 * static_cast<size_t>(batch) + 1);
}

template <typename T, int D, class P>
cudaError_t launch_tc(const DecodeArgs& a, const typename P::Maps& maps, int num_ctas,
                      bool overlap, cudaStream_t stream) {
  const size_t smem = tc_smem_bytes<P>(a.batch);
  auto kern = decode_tc_kernel<T, D, P>;
  // the opt-in shared-memory limit is per device; raise it once to the most any
  // batch can ask for
  static bool raised[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !raised[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(tc_smem_bytes<P>(kMaxBatch)));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) raised[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_ctas);
  cfg.blockDim = dim3(2 * kWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = overlap ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, maps, a);
}

}  // namespace tc
}  // namespace pa
