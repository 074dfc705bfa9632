// Paged decode attention on tensor cores over an INT8 cache.
//
// Cache ("KV Cache for intermediates..." / "The four solutions", KV-cache
// quantisation): per (token, kv head) 128 signed 8-bit codes and one fp32
// scale, for keys and for values; an element reads back as code * scale.  The
// pools hold one record per 16-token group of a (block, kv head) (layout in
// int8_launch.h), so a stage is two bulk copies of kRecordBytes.
//
// Products.  Key record line r holds token tau(r) = key_token(r), so row r of
// S^T = K . Q^T is token tau(r).  The contraction index of the first product
// is reordered so that a lane's four key bytes (one 32-bit ldmatrix element,
// d = 16kc + 4cq .. +3) are its four A elements; the query fragment uses the
// same order.  In O^T += V^T . P^T a lane's four value bytes are tokens
// 4cq .. 4cq+3, which is exactly the token order that the register transpose
// of S^T rows tau(.) gives the P^T fragment, so neither operand is shuffled.
// Every product is an fp16 mma whatever the query dtype: the codes are exact in
// fp16, and bf16 queries (8-bit significand) become fp16 exactly after a
// power-of-two prescale per head that puts the head's largest |q| in
// [2^13, 2^14); the prescale is divided out of the scores.
//  * Keys enter as 1024 + u (u = code + 128, the stored byte), exact in fp16
//    and two byte permutes per four codes; the product then carries
//    1152 * sum_d q_d too, which is subtracted once per segment (the
//    accumulator starts at -1152 * sum_d q_d).
//  * Values enter the same way, as 1024 + u: O then carries 1152 * sum_j p'_j
//    in every row, which one more product per stage (an all-ones A operand
//    against the same P fragment) accumulates exactly; it is subtracted at the
//    segment's end.  (Two byte permutes per four codes instead of two byte
//    permutes and two fp16 subtractions.)
// Scales.  Key scales multiply the score rows (with scale * log2 e).  Value
// scales are folded into P: p'_j = p_j * vs_j / sigma with sigma a lazily
// updated running maximum of the segment's value scales (p' stays within a
// fixed range whatever the scales' magnitude; O is rescaled when sigma moves,
// and the output is O * sigma).  The softmax sum l keeps the unscaled p.
//
// Roofline.  Per context token and KV head the kernel must read 128 + 128 bytes
// of codes and 4 + 4 bytes of scales: 264 bytes against 512 for fp16.
#include <type_traits>

#include "decode_tc.cuh"
#include "int8_launch.h"

namespace pa {
namespace tc {

// Four codes (bytes of w, stored offset-binary: u = c + 128) as two pairs of
// fp16 values, .x = bytes 0, 1, .y = bytes 2, 3.  0x64 in the high byte makes
// the fp16 value 1024 + u exactly.
__device__ __forceinline__ uint2 codes_biased(uint32_t w) {
  return make_uint2(__byte_perm(w, 0x64646464u, 0x5140), __byte_perm(w, 0x64646464u, 0x7362));
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Token of S^T row g (g < 8); row g + 8 holds that token + 2.
__device__ __forceinline__ int row_token(int g) { return i8::key_token(g); }

template <typename T>
struct Tiles8 {
  static constexpr int D = i8::kDim;
  static constexpr int KC = D / 16;
  static constexpr int kStages = 5;
  static constexpr int kConsumerRegs = 208;
  static constexpr int kProducerRegs = 48;
  static constexpr int kRec = i8::kRecordBytes;
  static constexpr int kStageBytes = 2 * kRec;  // key record + value record
  static constexpr int kRingBytes = (kWarps * kStages * kStageBytes + 1023) / 1024 * 1024;
  struct Maps {
    int unused;
  };
  struct Frag {
    uint32_t k[KC][2];  // [kc][row g, row g + 8]: 4 codes, d = 16kc + 4cq .. +3
    uint32_t v[KC][2];  // [mt][d = 16mt + g, +8]: 4 codes, tokens 4cq .. +3
    float ks0, ks1, vs0, vs1;  // scales of the lane's tokens row_token(g), +2
    uint32_t va[KC][4];        // value A operands (biased fp16 pairs)
    float u0, u1;              // value weights vs / sigma of the lane's tokens
  };
  struct Seg {
    float sig, inv;  // value-scale normaliser sigma and 1 / sigma
    float c0, c1;    // scale * log2 e / prescale, heads 2cq and 2cq + 1
    float qs0, qs1;  // -1152 * sum_d q'_d, heads 2cq and 2cq + 1
    float bsum[4];   // sum_j p'_j in O's fragment layout (every row the same)
    __device__ void reset() {
      sig = inv = 0.f;
      bsum[0] = bsum[1] = bsum[2] = bsum[3] = 0.f;
    }
    __device__ float out_scale() const { return sig; }
  };
  // the softmax reference moved: sum_j p'_j scales like O (heads 2cq, 2cq + 1)
  __device__ static void rescale(Seg& seg, float a0, float a1) {
    seg.bsum[0] *= a0;
    seg.bsum[1] *= a1;
    seg.bsum[2] *= a0;
    seg.bsum[3] *= a1;
  }
  // O = O' - 1152 sum_j p'_j: the value offset carried by the biased codes
  __device__ static void finish(float (&o)[KC][4], const Seg& seg) {
#pragma unroll
    for (int mt = 0; mt < KC; ++mt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) o[mt][e] = fmaf(-1152.f, seg.bsum[e], o[mt][e]);
    }
  }

  __device__ static void prefetch(const Maps&) {}
  __device__ static uint32_t stage(uint32_t ring0, int warp, int slot) {
    return ring0 + (warp * kStages + slot) * kStageBytes;
  }
  __device__ static void issue(const Maps&, const DecodeArgs& a, uint32_t ring0, int warp,
                               int slot, int tile, int tok, uint32_t bar) {
    const int64_t rec = static_cast<int64_t>(tile) * (a.block_size / i8::kGroup) + tok / i8::kGroup;
    const uint32_t dst = stage(ring0, warp, slot);
    bulk_copy(dst, static_cast<const uint8_t*>(a.k_cache) + rec * kRec, kRec, bar);
    bulk_copy(dst + kRec, static_cast<const uint8_t*>(a.v_cache) + rec * kRec, kRec, bar);
  }
  // lane (g, cq) holds q[g][16kc + 4cq, +1] and q[g][16kc + 4cq + 2, +3]
  __device__ static int q_off(int kc, int cq, int half) { return kc * 16 + 4 * cq + 2 * half; }

  // The segment's query fragments (pairs of T) become fp16 pairs q' = q * f, f a
  // power of two per head (1 for fp16 queries); seg gets each of the lane's two
  // heads' score factor (scale * log2 e / f) and key-offset term.
  __device__ static void prep_q(uint32_t (&qf)[KC][2], Seg& seg, const DecodeArgs& a, int lane) {
    float finv = 1.f;
    if (!std::is_same<T, __half>::value) {
      float amax = 0.f;
#pragma unroll
      for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 x = unpack2<T>(qf[kc][h]);
          amax = fmaxf(amax, fmaxf(fabsf(x.x), fabsf(x.y)));
        }
      }
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
      // amax < 2^e; f = 2^(14 - e) puts it in [2^13, 2^14) (capped for tiny heads)
      const int e = ((__float_as_int(amax) >> 23) & 0xff) - 126;
      const int fe = min(14 - e, 126);
      const float f = amax > 0.f ? __int_as_float((127 + fe) << 23) : 1.f;
      finv = amax > 0.f ? __int_as_float((127 - fe) << 23) : 1.f;
#pragma unroll
      for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 x = unpack2<T>(qf[kc][h]);
          qf[kc][h] = pack2<__half>(x.x * f, x.y * f);
        }
      }
    }
    float sum = 0.f;
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 x = unpack2<__half>(qf[kc][h]);
        sum += x.x + x.y;
      }
    }
    sum += __shfl_xor_sync(kFull, sum, 1);
    sum += __shfl_xor_sync(kFull, sum, 2);
    // heads 2cq and 2cq + 1 are held by lanes 8cq and 8cq + 4
    const int cq = lane & 3;
    seg.qs0 = -1152.f * __shfl_sync(kFull, sum, 8 * cq);
    seg.qs1 = -1152.f * __shfl_sync(kFull, sum, 8 * cq + 4);
    seg.c0 = a.scale_log2 * __shfl_sync(kFull, finv, 8 * cq);
    seg.c1 = a.scale_log2 * __shfl_sync(kFull, finv, 8 * cq + 4);
  }

  __device__ static void load(const DecodeArgs&, uint32_t ring0, int warp, int slot, int,
                              int lane, Frag& f) {
    const uint32_t kt = stage(ring0, warp, slot), vt = kt + kRec;
    const int mi = lane >> 3, r8 = lane & 7;
    const int line = r8 + ((mi & 1) << 3);
#pragma unroll
    for (int kk = 0; kk < KC / 2; ++kk) {
      uint32_t r[4];
      ldsm_x4(kt + line * 128 + (((2 * kk + (mi >> 1)) ^ r8) << 4), r);
      f.k[2 * kk][0] = r[0];
      f.k[2 * kk][1] = r[1];
      f.k[2 * kk + 1][0] = r[2];
      f.k[2 * kk + 1][1] = r[3];
      ldsm_x4(vt + (32 * kk + 16 * (mi >> 1) + line) * 16, r);
      f.v[2 * kk][0] = r[0];
      f.v[2 * kk][1] = r[1];
      f.v[2 * kk + 1][0] = r[2];
      f.v[2 * kk + 1][1] = r[3];
    }
    const int tk = row_token(lane >> 2);
    f.ks0 = lds_f32(kt + i8::kCodeBytes + 4 * tk);
    f.ks1 = lds_f32(kt + i8::kCodeBytes + 4 * (tk + 2));
    f.vs0 = lds_f32(vt + i8::kCodeBytes + 4 * tk);
    f.vs1 = lds_f32(vt + i8::kCodeBytes + 4 * (tk + 2));
  }

  __device__ static void scores(const Frag& f, const uint32_t (&qf)[KC][2], const Seg& seg,
                                const DecodeArgs&, int n_valid, int lane, float (&t)[4]) {
    // accumulator element i is (row g or g + 8, head 2cq or 2cq + 1): start from
    // the head's key-offset term; two accumulators halve the dependent chain
    float s[4] = {seg.qs0, seg.qs1, seg.qs0, seg.qs1}, s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
      const uint2 r0 = codes_biased(f.k[kc][0]);
      const uint2 r1 = codes_biased(f.k[kc][1]);
      const uint32_t A[4] = {r0.x, r1.x, r0.y, r1.y};
      if (kc & 1) mma16816<__half>(s2, A, qf[kc]); else mma16816<__half>(s, A, qf[kc]);
    }
    const int tk = row_token(lane >> 2);
    t[0] = (s[0] + s2[0]) * (f.ks0 * seg.c0);
    t[1] = (s[1] + s2[1]) * (f.ks0 * seg.c1);
    t[2] = (s[2] + s2[2]) * (f.ks1 * seg.c0);
    t[3] = (s[3] + s2[3]) * (f.ks1 * seg.c1);
    if (tk >= n_valid) t[0] = t[1] = -INFINITY;
    if (tk + 2 >= n_valid) t[2] = t[3] = -INFINITY;
  }

  // Work of the value product that does not need P, done while the score
  // products are in flight: the value codes' conversion and the normaliser.
  __device__ static void pre_pv(Frag& f, float (&o)[KC][4], Seg& seg, int n_valid, int lane) {
#pragma unroll
    for (int mt = 0; mt < KC; ++mt) {
      const uint2 r0 = codes_biased(f.v[mt][0]);
      const uint2 r1 = codes_biased(f.v[mt][1]);
      f.va[mt][0] = r0.x;
      f.va[mt][1] = r1.x;
      f.va[mt][2] = r0.y;
      f.va[mt][3] = r1.y;
    }
    const int tk = row_token(lane >> 2);
    const float w0 = tk < n_valid ? f.vs0 : 0.f;
    const float w1 = tk + 2 < n_valid ? f.vs1 : 0.f;
    // Lazy normaliser: sigma moves only when a value scale exceeds 16 sigma
    // (then to the stage's largest scale, the same in every lane), so
    // vs / sigma <= 16 and p' = p vs / sigma <= 2^12, well inside fp16.  (O
    // is rescaled here before the stage's softmax may rescale it: the two
    // factors commute.)
    if (__any_sync(kFull, fmaxf(w0, w1) > seg.sig * 16.f)) {
      float mx = fmaxf(w0, w1);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
      const float r = seg.sig / mx;
#pragma unroll
      for (int mt = 0; mt < KC; ++mt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) o[mt][e] *= r;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) seg.bsum[e] *= r;
      seg.sig = mx;
      seg.inv = 1.f / mx;
    }
    f.u0 = w0 * seg.inv;
    f.u1 = w1 * seg.inv;
  }

  __device__ static void pv(const Frag& f, const float (&p)[4], float (&o)[KC][4], Seg& seg,
                            int, int) {
    // fp16 weights (11-bit significand, p' <= 2^12) in one product
    const uint32_t pb[2] = {transpose8x8(pack2<__half>(p[0] * f.u0, p[1] * f.u0)),
                            transpose8x8(pack2<__half>(p[2] * f.u1, p[3] * f.u1))};
#pragma unroll
    for (int mt = 0; mt < KC; ++mt) mma16816<__half>(o[mt], f.va[mt], pb);
    // sum_j p'_j of the 16 tokens for each head (fp16 1.0 pairs)
    const uint32_t ones[4] = {0x3c003c00u, 0x3c003c00u, 0x3c003c00u, 0x3c003c00u};
    mma16816<__half>(seg.bsum, ones, pb);
  }
};

}  // namespace tc

int decode_int8_workers_per_cta() { return tc::kWarps; }

cudaError_t launch_decode_int8(const DecodeArgs& a, pa_dtype dtype, int num_ctas, bool overlap,
                               cudaStream_t stream) {
  if (dtype == PA_F16)
    return tc::launch_tc<__half, 128, tc::Tiles8<__half>>(a, {0}, num_ctas, overlap, stream);
  return tc::launch_tc<__nv_bfloat16, 128, tc::Tiles8<__nv_bfloat16>>(a, {0}, num_ctas, overlap,
                                                                      stream);
}

}  // namespace pa
