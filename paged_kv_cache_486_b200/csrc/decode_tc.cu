// Paged decode attention on tensor cores over an fp16 / bf16 cache.
//
// Stage: 16 rows x D of the key pool and of the value pool, rows
// (block * Hkv + kv_head) * block_size + 16 s, each loaded by one TMA copy as
// D/64 column blocks of 16 rows x 64 columns (a 3-D box; two 2-D boxes if the
// driver declines the 3-D map).  A column block lands 128-byte-swizzled with
// one row per 128-byte line, so the eight rows an ldmatrix reads sit in eight
// different bank groups (with whole 256-byte rows per line, rows t and t+4
// would share banks).  Keys enter S^T = K . Q^T as the A operand straight from ldmatrix;
// values enter O^T += V^T . P^T through ldmatrix.trans.
//
// Roofline.  Per context token and KV head the kernel must read D*2 bytes of
// key and D*2 of value; tensor-core work is ~4*8*D flops per token and KV head
// (8 padded heads), far below the tensor rate, so HBM bandwidth bounds it.
#include "decode_tc.cuh"

namespace pa {
namespace tc {

template <typename T, int D>
struct Tiles16 {
  static constexpr int KC = D / 16;
  static constexpr int kStages = 3;
  static constexpr int kConsumerRegs = tc::kConsumerRegs;
  static constexpr int kProducerRegs = tc::kProducerRegs;
  static constexpr int kTileBytes = kTok * D * 2;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kRingBytes = kWarps * kStages * kStageBytes;
  struct Maps {
    CUtensorMap k, v;
    int three_d;  // maps are {64, rows, D/64} (one copy per tile), else {D, rows}
  };
  struct Frag {
    uint32_t k[KC][4], v[KC][4];
  };
  struct Seg {
    __device__ void reset() {}
    __device__ float out_scale() const { return 1.f; }
  };
  __device__ static void rescale(Seg&, float, float) {}
  __device__ static void pre_pv(Frag&, float (&)[D / 16][4], Seg&, int, int) {}
  __device__ static void finish(float (&)[D / 16][4], const Seg&) {}

  __device__ static void prefetch(const Maps& m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&m.k)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&m.v)) : "memory");
  }
  __device__ static uint32_t stage(uint32_t ring0, int warp, int slot) {
    return ring0 + (warp * kStages + slot) * kStageBytes;
  }
  __device__ static void issue(const Maps& m, const DecodeArgs& a, uint32_t ring0, int warp,
                               int slot, int tile, int tok, uint32_t bar) {
    const int row = tile * a.block_size + tok;
    const uint32_t dst = stage(ring0, warp, slot);
    tma_tile<D>(dst, &m.k, row, m.three_d != 0, bar);
    tma_tile<D>(dst + kTileBytes, &m.v, row, m.three_d != 0, bar);
  }
  // lane (g, cq) holds q[g][16kc + 2cq, +1] and q[g][16kc + 8 + 2cq, +1]
  __device__ static int q_off(int kc, int cq, int half) { return kc * 16 + 8 * half + 2 * cq; }
  __device__ static void prep_q(uint32_t (&)[KC][2], Seg&, const DecodeArgs&, int) {}

  __device__ static void load(const DecodeArgs&, uint32_t ring0, int warp, int slot,
                              int n_valid, int lane, Frag& f) {
    const uint32_t kt = stage(ring0, warp, slot);
    const uint32_t vt = kt + kTileBytes;
    if (n_valid < kTok) {
      // rows past the context may hold anything (even NaN): clear them in V
      const int per_box = (kTok - n_valid) * 8;  // 16-byte chunks past the context
      for (int i = lane; i < per_box * (D / 64); i += 32) {
        const int h = i / per_box, r = i - h * per_box;
        const uint32_t addr = vt + h * kBoxBytes + n_valid * 128 + r * 16;
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
      }
      // generic writes to a slot that TMA refills later
      fence_proxy_async_smem();
      __syncwarp();
    }
    const int mi = lane >> 3;
    const int ktok = ((mi & 1) << 3) + (lane & 7);
    const int vtok = ((mi >> 1) << 3) + (lane & 7);
#pragma unroll
    for (int c = 0; c < KC; ++c) {
      ldsm_x4(swz(kt, ktok, 2 * c + (mi >> 1)), f.k[c]);
      ldsm_x4_trans(swz(vt, vtok, 2 * c + (mi & 1)), f.v[c]);
    }
  }

  __device__ static void scores(const Frag& f, const uint32_t (&qf)[KC][2], const Seg&,
                                const DecodeArgs& a, int n_valid, int lane, float (&t)[4]) {
    // two accumulators halve the dependent chain
    float s[4] = {0.f, 0.f, 0.f, 0.f}, s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kc = 0; kc < KC; ++kc) {
      if (kc & 1) mma16816<T>(s2, f.k[kc], qf[kc]); else mma16816<T>(s, f.k[kc], qf[kc]);
    }
    const int g = lane >> 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) t[i] = (s[i] + s2[i]) * a.scale_log2;
    if (g >= n_valid) t[0] = t[1] = -INFINITY;
    if (g + 8 >= n_valid) t[2] = t[3] = -INFINITY;
  }

  __device__ static void pv(const Frag& f, const float (&p)[4], float (&o)[KC][4], Seg&, int,
                            int) {
    uint32_t h01, t01, h23, t23;
    split2<T>(p[0], p[1], h01, t01);
    split2<T>(p[2], p[3], h23, t23);
    const uint32_t pb[2] = {transpose8x8(h01), transpose8x8(h23)};
    const uint32_t pt[2] = {transpose8x8(t01), transpose8x8(t23)};
    // O^T += V^T . (P_head + P_tail)^T
#pragma unroll
    for (int mt = 0; mt < KC; ++mt) {
      mma16816<T>(o[mt], f.v[mt], pb);
      mma16816<T>(o[mt], f.v[mt], pt);
    }
  }
};

}  // namespace tc

int decode_tc_workers_per_cta() { return tc::kWarps; }

size_t decode_tc_smem_bytes(int head_dim, int batch) {
  return head_dim == 128 ? tc::tc_smem_bytes<tc::Tiles16<__half, 128>>(batch)
                         : tc::tc_smem_bytes<tc::Tiles16<__half, 64>>(batch);
}

cudaError_t launch_decode_tc(const DecodeArgs& a, pa_dtype dtype, const CUtensorMap& kmap,
                             const CUtensorMap& vmap, bool three_d, int num_ctas, bool overlap,
                             cudaStream_t stream) {
  using tc::Tiles16;
  const int td = three_d ? 1 : 0;
  if (a.head_dim == 128) {
    if (dtype == PA_F16) {
      using P = Tiles16<__half, 128>;
      return tc::launch_tc<__half, 128, P>(a, P::Maps{kmap, vmap, td}, num_ctas, overlap, stream);
    }
    using P = Tiles16<__nv_bfloat16, 128>;
    return tc::launch_tc<__nv_bfloat16, 128, P>(a, P::Maps{kmap, vmap, td}, num_ctas, overlap,
                                                stream);
  }
  if (dtype == PA_F16) {
    using P = Tiles16<__half, 64>;
    return tc::launch_tc<__half, 64, P>(a, P::Maps{kmap, vmap, td}, num_ctas, overlap, stream);
  }
  using P = Tiles16<__nv_bfloat16, 64>;
  return tc::launch_tc<__nv_bfloat16, 64, P>(a, P::Maps{kmap, vmap, td}, num_ctas, overlap,
                                             stream);
}

}  // namespace pa
