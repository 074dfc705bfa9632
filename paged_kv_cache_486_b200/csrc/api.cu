// C ABI entry points for the device calls: argument checks, path and launch
// choices, TMA tensor maps, and the device error word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "cache_ops.h"
#include "decode_common.cuh"
#include "decode_launch.h"
#include "host_common.h"
#include "int8_launch.h"
#include "prefill_launch.h"

namespace {

using pa::fail;

int elem_bytes(pa_dtype d) { return d == PA_F32 ? 4 : 2; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool valid_dtype(pa_dtype d) { return d == PA_F32 || d == PA_F16 || d == PA_BF16; }

pa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int sm_count() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) return 0;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

// ------------------------------ tensor maps --------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A pool [num_blocks, Hkv, bs, D] seen as `rows` rows of D elements.  Preferred
// form (three_d): {64 columns, rows, D / 64 column blocks} with strides D * 2
// (row) and 128 bytes (column block), box {64, 16, D / 64}: one copy lands a
// whole 16-row tile as D / 64 column blocks of 16 lines x 128 bytes.  If the
// driver declines that map, {D, rows} with box {64, 16}, one copy per block.
bool make_tile_map(CUtensorMap* map, bool* three_d, const void* base, int64_t rows,
                   int head_dim, pa_dtype dt) {
  auto enc = encode_fn();
  if (!enc) return false;
  const CUtensorMapDataType t =
      dt == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (head_dim > 64) {
    cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(head_dim / 64)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2, 128};
    cuuint32_t box[3] = {64, 16, static_cast<cuuint32_t>(head_dim / 64)};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(map, t, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
        CUDA_SUCCESS) {
      *three_d = true;
      return true;
    }
  }
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(head_dim) * 2};
  cuuint32_t box[2] = {64, 16};
  cuuint32_t es[2] = {1, 1};
  *three_d = false;
  return enc(map, t, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// q (or out) as {head_dim, num_q_heads, total_q} with a {64, group, 128 /
// group} box: 128 rows of (token, head of one kv head's group) pairs per
// 64-column block.
static bool make_q_map(CUtensorMap* map, const void* q, int total_q, int num_q_heads,
                       int head_dim, int group, pa_dtype dt) {
  auto enc = encode_fn();
  if (!enc) return false;
  const CUtensorMapDataType t =
      dt == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_q_heads),
                        static_cast<cuuint64_t>(total_q)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                           static_cast<cuuint64_t>(head_dim) * 2 * num_q_heads};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(128 / group)};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(map, t, 3, const_cast<void*>(q), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// The {D, rows} form with a {64, 16} box only (the tcgen05 prefill addresses
// each 64-column block itself).
bool make_tile_map_2d(CUtensorMap* map, const void* base, int64_t rows, int head_dim,
                      pa_dtype dt) {
  auto enc = encode_fn();
  if (!enc) return false;
  const CUtensorMapDataType t =
      dt == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(head_dim) * 2};
  cuuint32_t box[2] = {64, 16};
  cuuint32_t es[2] = {1, 1};
  return enc(map, t, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Small per-thread cache: encoding is cheap but not free, and decode is called
// with the same pools every step.
struct MapEntry {
  const void* base;
  int64_t rows;
  int head_dim;
  int dtype;
  bool three_d;
  CUtensorMap map;
};
thread_local MapEntry g_maps[8];
thread_local int g_maps_next = 0;

bool tile_map(CUtensorMap* out, bool* three_d, const void* base, int64_t rows, int head_dim,
              pa_dtype dt) {
  for (auto& e : g_maps) {
    if (e.base == base && e.rows == rows && e.head_dim == head_dim && e.dtype == dt) {
      *out = e.map;
      *three_d = e.three_d;
      return true;
    }
  }
  MapEntry& e = g_maps[g_maps_next];
  if (!make_tile_map(&e.map, &e.three_d, base, rows, head_dim, dt)) return false;
  e.base = base;
  e.rows = rows;
  e.head_dim = head_dim;
  e.dtype = dt;
  g_maps_next = (g_maps_next + 1) % 8;
  *out = e.map;
  *three_d = e.three_d;
  return true;
}

// ------------------------------ decode plan --------------------------------
int max_workers(int group) {
  int w = pa::kPieceHeadBudget / group;
  if (w > pa::kMaxWorkers) w = pa::kMaxWorkers;
  return w < 1 ? 1 : w;
}

bool tc_applies(int group, int head_dim, int block_size, pa_dtype dt) {
  return (dt == PA_F16 || dt == PA_BF16) && (head_dim == 64 || head_dim == 128) && group <= 8 &&
         block_size % 16 == 0;
}

// Workspace layout, the same for every shape so that one zero-filled
// workspace can serve calls of any batch and head count:
//   [0, 256)                  chunk counter, finished-worker counter
//   [256, kArrivalsEnd)       one arrival count per (sequence, kv head), for
//                             up to kMaxArrivals pairs (pair b * Hkv + kvh)
//   [kArrivalsEnd, ...)       piece slots (written before they are read)
// Only the first two regions must start at zero, and a completed call leaves
// every word it used there at zero.
constexpr size_t kArrivalsOffset = 256;
constexpr size_t kArrivalsEnd = kArrivalsOffset + sizeof(uint32_t) * pa::kMaxArrivals;

size_t pieces_bytes(int group, int head_dim) {
  return sizeof(float) * 2 * static_cast<size_t>(pa::max_ranges(max_workers(group))) * group *
         (head_dim + 2);
}

// Host checks shared by the 16-bit decode entry points (nothing touches the
// device here).
pa_status check_decode_args(pa_dtype dtype, int32_t batch, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                            int32_t num_blocks, int32_t max_blocks, float scale) {
  if (!valid_dtype(dtype))
    return fail(PA_ERR_INVALID, "pa_decode_attention: unknown dtype %d", static_cast<int>(dtype));
  if (batch < 0 || batch > pa::kMaxBatch)
    return fail(PA_ERR_INVALID, "pa_decode_attention: batch %d outside [0, %d]", batch,
                pa::kMaxBatch);
  if (num_kv_heads < 1 || num_kv_heads > pa::kMaxKvHeads || num_q_heads < num_kv_heads ||
      num_q_heads % num_kv_heads)
    return fail(PA_ERR_INVALID, "pa_decode_attention: num_q_heads %d not a multiple of "
                "num_kv_heads %d (at most %d)", num_q_heads, num_kv_heads, pa::kMaxKvHeads);
  if (head_dim != 64 && head_dim != 128)
    return fail(PA_ERR_INVALID, "pa_decode_attention: head_dim %d not in {64, 128}", head_dim);
  if (block_size != 8 && block_size != 16 && block_size != 32 && block_size != 64 &&
      block_size != 128)
    return fail(PA_ERR_INVALID, "pa_decode_attention: block_size %d not in {8,16,32,64,128}",
                block_size);
  if (num_blocks < 0 || max_blocks < 0)
    return fail(PA_ERR_INVALID, "pa_decode_attention: negative num_blocks or max_blocks");
  const int64_t rows = static_cast<int64_t>(num_blocks) * num_kv_heads * block_size;
  if (rows >= (int64_t(1) << 31))
    return fail(PA_ERR_INVALID, "pa_decode_attention: num_blocks * num_kv_heads * block_size "
                "= %lld >= 2^31", static_cast<long long>(rows));
  if (static_cast<int64_t>(num_kv_heads) * max_blocks >= (int64_t(1) << 31))
    return fail(PA_ERR_INVALID, "pa_decode_attention: num_kv_heads * max_blocks >= 2^31");
  if (!(scale == scale)) return fail(PA_ERR_INVALID, "pa_decode_attention: scale is NaN");
  if (static_cast<int64_t>(batch) * num_kv_heads > pa::kMaxArrivals)
    return fail(PA_ERR_INVALID, "pa_decode_attention: batch * num_kv_heads = %lld > %d",
                static_cast<long long>(batch) * num_kv_heads, pa::kMaxArrivals);
  return PA_OK;
}

}  // namespace

extern "C" {

int32_t pa_device_sm_count(void) { return sm_count(); }

pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                               const int64_t* slot_mapping, int32_t n_tokens,
                               int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                               int32_t num_blocks, pa_dtype dtype, int32_t* dev_error,
                               pa_stream stream) {
  if (!valid_dtype(dtype) || n_tokens < 0 || num_kv_heads < 1 || head_dim < 1 ||
      block_size < 1 || num_blocks < 0)
    return fail(PA_ERR_INVALID, "pa_reshape_and_cache: bad sizes (n_tokens=%d kv_heads=%d "
                "head_dim=%d block_size=%d num_blocks=%d)", n_tokens, num_kv_heads, head_dim,
                block_size, num_blocks);
  const int row_bytes = head_dim * elem_bytes(dtype);
  if (row_bytes % 16)
    return fail(PA_ERR_INVALID, "pa_reshape_and_cache: head_dim * element size = %d bytes is "
                "not a multiple of 16", row_bytes);
  if (n_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping)
    return fail(PA_ERR_INVALID, "pa_reshape_and_cache: NULL pointer");
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(slot_mapping, 8))
    return fail(PA_ERR_INVALID, "pa_reshape_and_cache: misaligned pointer");
  const cudaError_t e = pa::launch_reshape_and_cache(
      key, value, k_cache, v_cache, slot_mapping, n_tokens, num_kv_heads, row_bytes, block_size,
      num_blocks, dev_error, sm_count() ? sm_count() : 148, stream);
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "pa_reshape_and_cache");
}

pa_status pa_copy_blocks(void* const* k_caches_host, void* const* v_caches_host,
                         int32_t num_layers, const int32_t* pairs, int32_t n_pairs,
                         int32_t num_blocks, int64_t block_bytes, int32_t* dev_error,
                         pa_stream stream) {
  if (num_layers < 1 || num_layers > pa::kMaxLayers || n_pairs < 0 || num_blocks < 0 ||
      block_bytes <= 0 || block_bytes % 16)
    return fail(PA_ERR_INVALID, "pa_copy_blocks: bad sizes (layers=%d pairs=%d block_bytes=%lld)",
                num_layers, n_pairs, static_cast<long long>(block_bytes));
  if (n_pairs == 0) return PA_OK;
  if (!k_caches_host || !v_caches_host || !pairs)
    return fail(PA_ERR_INVALID, "pa_copy_blocks: NULL pointer");
  pa::LayerPtrs ptrs;
  std::memset(&ptrs, 0, sizeof ptrs);
  for (int i = 0; i < num_layers; ++i) {
    if (!k_caches_host[i] || !v_caches_host[i] || !aligned(k_caches_host[i], 16) ||
        !aligned(v_caches_host[i], 16))
      return fail(PA_ERR_INVALID, "pa_copy_blocks: layer %d pointer NULL or misaligned", i);
    ptrs.k[i] = k_caches_host[i];
    ptrs.v[i] = v_caches_host[i];
  }
  const cudaError_t e = pa::launch_copy_blocks(ptrs, num_layers, pairs, n_pairs, num_blocks,
                                               block_bytes, dev_error, stream);
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "pa_copy_blocks");
}

// A pointer the kernels can dereference: device memory, managed memory, or
// pinned (page-locked, registered) host memory; returns the device address.
static bool device_address(const void* p, const void** out) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged) {
    *out = p;
    return true;
  }
  if (attr.type == cudaMemoryTypeHost && attr.devicePointer) {
    *out = attr.devicePointer;
    return true;
  }
  return false;
}

pa_status pa_swap_blocks(void* const* dst_k_host, void* const* dst_v_host,
                         void* const* src_k_host, void* const* src_v_host, int32_t num_layers,
                         const int32_t* pairs, int32_t n_pairs, int32_t src_num_blocks,
                         int32_t dst_num_blocks, int64_t block_bytes, int32_t* dev_error,
                         pa_stream stream) {
  if (num_layers < 1 || num_layers > pa::kMaxLayers || n_pairs < 0 || src_num_blocks < 0 ||
      dst_num_blocks < 0 || block_bytes <= 0 || block_bytes % 16)
    return fail(PA_ERR_INVALID, "pa_swap_blocks: bad sizes (layers=%d pairs=%d block_bytes=%lld)",
                num_layers, n_pairs, static_cast<long long>(block_bytes));
  if (n_pairs == 0) return PA_OK;
  if (!dst_k_host || !dst_v_host || !src_k_host || !src_v_host || !pairs)
    return fail(PA_ERR_INVALID, "pa_swap_blocks: NULL pointer");
  const void* pairs_dev = nullptr;
  if (!device_address(pairs, &pairs_dev))
    return fail(PA_ERR_INVALID, "pa_swap_blocks: pairs is neither device nor pinned host memory");
  pa::LayerPtrs dst, src;
  std::memset(&dst, 0, sizeof dst);
  std::memset(&src, 0, sizeof src);
  void* const* in[4] = {dst_k_host, dst_v_host, src_k_host, src_v_host};
  void** outp[4] = {dst.k, dst.v, src.k, src.v};
  for (int a = 0; a < 4; ++a) {
    for (int i = 0; i < num_layers; ++i) {
      const void* d = nullptr;
      if (!in[a][i] || !aligned(in[a][i], 16) || !device_address(in[a][i], &d))
        return fail(PA_ERR_INVALID, "pa_swap_blocks: layer %d pool pointer is NULL, misaligned "
                    "or not device-accessible (use device or pinned host memory)", i);
      outp[a][i] = const_cast<void*>(d);
    }
  }
  const cudaError_t e = pa::launch_swap_blocks(
      dst, src, num_layers, static_cast<const int32_t*>(pairs_dev), n_pairs, src_num_blocks,
      dst_num_blocks, block_bytes, dev_error, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "pa_swap_blocks");
}

size_t pa_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                int32_t head_dim) {
  if (batch < 0 || num_kv_heads < 1 || num_q_heads < num_kv_heads ||
      num_q_heads % num_kv_heads || head_dim < 1)
    return 0;
  return kArrivalsEnd + pieces_bytes(num_q_heads / num_kv_heads, head_dim);
}

pa_status pa_decode_plan(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                         int32_t head_dim, int32_t block_size, pa_dtype dtype, int32_t* path_out,
                         int32_t* num_workers_out) {
  if (num_kv_heads < 1 || num_q_heads < num_kv_heads || num_q_heads % num_kv_heads)
    return fail(PA_ERR_INVALID, "pa_decode_plan: bad head counts");
  const int group = num_q_heads / num_kv_heads;
  const int sms = sm_count() ? sm_count() : 148;
  int path, workers;
  if (tc_applies(group, head_dim, block_size, dtype)) {
    path = PA_PATH_TC;
    workers = sms * pa::decode_tc_workers_per_cta();
  } else {
    path = PA_PATH_SIMT;
    workers = sms * 16;
  }
  const int cap = max_workers(group);
  if (workers > cap) workers = cap;
  (void)batch;
  if (path_out) *path_out = path;
  if (num_workers_out) *num_workers_out = workers;
  return PA_OK;
}

pa_status pa_decode_attention_ex(void* out, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, int32_t batch, int32_t num_q_heads,
                                 int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                 int32_t num_blocks, int32_t max_blocks, float scale,
                                 pa_dtype dtype, void* workspace, size_t workspace_bytes,
                                 int32_t* dev_error, int32_t path, int32_t num_workers,
                                 int32_t flags, pa_stream stream) {
  const pa_status chk = check_decode_args(dtype, batch, num_q_heads, num_kv_heads, head_dim,
                                          block_size, num_blocks, max_blocks, scale);
  if (chk != PA_OK) return chk;
  const int64_t rows = static_cast<int64_t>(num_blocks) * num_kv_heads * block_size;
  if (path != PA_PATH_AUTO && path != PA_PATH_TC && path != PA_PATH_SIMT)
    return fail(PA_ERR_INVALID, "pa_decode_attention: unknown path %d", path);
  if (flags & ~(PA_DECODE_OVERLAP_PROLOGUE | PA_DECODE_TEST_WAIT_EXPIRY))
    return fail(PA_ERR_INVALID, "pa_decode_attention: unknown flags 0x%x", flags);
  const bool overlap = (flags & PA_DECODE_OVERLAP_PROLOGUE) != 0;
  if (batch == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !workspace)
    return fail(PA_ERR_INVALID, "pa_decode_attention: NULL pointer");
  if (!aligned(q, 4) || !aligned(out, 4) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(workspace, 16) || !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return fail(PA_ERR_INVALID, "pa_decode_attention: misaligned pointer");
  const size_t need = pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim);
  if (workspace_bytes < need)
    return fail(PA_ERR_INVALID, "pa_decode_attention: workspace %zu bytes < %zu needed",
                workspace_bytes, need);

  const int group = num_q_heads / num_kv_heads;
  const bool tc_ok = tc_applies(group, head_dim, block_size, dtype);
  if (path == PA_PATH_TC && !tc_ok)
    return fail(PA_ERR_INVALID, "pa_decode_attention: tensor-core path needs fp16/bf16, "
                "group <= 8 and block_size a multiple of 16");
  const bool use_tc = path == PA_PATH_TC || (path == PA_PATH_AUTO && tc_ok);
  if ((flags & PA_DECODE_TEST_WAIT_EXPIRY) && !use_tc)
    return fail(PA_ERR_INVALID, "pa_decode_attention: PA_DECODE_TEST_WAIT_EXPIRY needs the "
                "tensor-core path");
  int32_t planned_path = 0, workers = 0;
  pa_status st = pa_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, block_size, dtype,
                                &planned_path, &workers);
  if (st != PA_OK) return st;
  if (!use_tc && planned_path == PA_PATH_TC) workers = (sm_count() ? sm_count() : 148) * 16;
  if (num_workers > 0) workers = num_workers;
  if (workers > max_workers(group)) workers = max_workers(group);

  pa::DecodeArgs a;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.dev_error = dev_error;
  a.ws_ctrl = static_cast<uint32_t*>(workspace);
  a.ws_arrivals = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + kArrivalsOffset);
  a.ws_pieces = reinterpret_cast<float*>(static_cast<char*>(workspace) + kArrivalsEnd);
  a.batch = batch;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.group = group;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.max_blocks = max_blocks;
  a.workers = workers;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.test_expire = (flags & PA_DECODE_TEST_WAIT_EXPIRY) ? 1 : 0;

  cudaError_t e;
  if (use_tc) {
    CUtensorMap kmap, vmap;
    bool k3 = false, v3 = false;
    if (!tile_map(&kmap, &k3, k_cache, rows, head_dim, dtype) ||
        !tile_map(&vmap, &v3, v_cache, rows, head_dim, dtype))
      return fail(PA_ERR_CUDA, "pa_decode_attention: cuTensorMapEncodeTiled failed");
    if (k3 != v3) return fail(PA_ERR_CUDA, "pa_decode_attention: inconsistent tensor maps");
    const int per = pa::decode_tc_workers_per_cta();
    e = pa::launch_decode_tc(a, dtype, kmap, vmap, k3, (workers + per - 1) / per, overlap,
                             static_cast<cudaStream_t>(stream));
  } else {
    e = pa::launch_decode_simt(a, dtype, overlap, static_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "pa_decode_attention (decode kernel)");
  return PA_OK;
}

pa_status pa_decode_attention(void* out, const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables, const int32_t* context_lens,
                              int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                              int32_t head_dim, int32_t block_size, int32_t num_blocks,
                              int32_t max_blocks, float scale, pa_dtype dtype, void* workspace,
                              size_t workspace_bytes, int32_t* dev_error, pa_stream stream) {
  return pa_decode_attention_ex(out, q, k_cache, v_cache, block_tables, context_lens, batch,
                                num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                max_blocks, scale, dtype, workspace, workspace_bytes, dev_error,
                                PA_PATH_AUTO, 0, 0, stream);
}

pa_status pa_reshape_and_cache_int8(const void* key, const void* value, void* k_pool,
                                    void* v_pool, const int64_t* slot_mapping, int32_t n_tokens,
                                    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                    int32_t num_blocks, pa_dtype dtype, int32_t* dev_error,
                                    pa_stream stream) {
  if (!valid_dtype(dtype) || n_tokens < 0 || num_kv_heads < 1 || block_size < 16 ||
      block_size % 16 || num_blocks < 0 || head_dim != pa::i8::kDim)
    return fail(PA_ERR_INVALID, "pa_reshape_and_cache_int8: bad sizes (n_tokens=%d "
                "kv_heads=%d head_dim=%d block_size=%d num_blocks=%d; head_dim must be 128 and "
                "block_size a multiple of 16)", n_tokens, num_kv_heads, head_dim, block_size,
                num_blocks);
  if (n_tokens == 0) return PA_OK;
  if (!key || !value || !k_pool || !v_pool || !slot_mapping)
    return fail(PA_ERR_INVALID, "pa_reshape_and_cache_int8: NULL pointer");
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
      !aligned(slot_mapping, 8))
    return fail(PA_ERR_INVALID, "pa_reshape_and_cache_int8: misaligned pointer");
  pa::Int8WriteArgs a;
  a.key = key;
  a.value = value;
  a.k_pool = static_cast<uint8_t*>(k_pool);
  a.v_pool = static_cast<uint8_t*>(v_pool);
  a.slots = slot_mapping;
  a.n_tokens = n_tokens;
  a.num_kv_heads = num_kv_heads;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.dev_error = dev_error;
  const cudaError_t e =
      pa::launch_reshape_and_cache_int8(a, dtype, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "pa_reshape_and_cache_int8");
}

size_t pa_int8_block_bytes(int32_t num_kv_heads, int32_t head_dim, int32_t block_size) {
  if (num_kv_heads < 1 || head_dim != pa::i8::kDim || block_size < 16 || block_size % 16)
    return 0;
  return static_cast<size_t>(num_kv_heads) * (block_size / pa::i8::kGroup) *
         pa::i8::kRecordBytes;
}

pa_status pa_decode_attention_int8(void* out, const void* q, const void* k_pool,
                                   const void* v_pool, const int32_t* block_tables,
                                   const int32_t* context_lens, int32_t batch,
                                   int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                   int32_t block_size, int32_t num_blocks, int32_t max_blocks,
                                   float scale, pa_dtype dtype, void* workspace,
                                   size_t workspace_bytes, int32_t* dev_error,
                                   int32_t num_workers, int32_t flags, pa_stream stream) {
  if (dtype != PA_F16 && dtype != PA_BF16)
    return fail(PA_ERR_INVALID, "pa_decode_attention_int8: queries must be fp16 or bf16");
  if (batch < 0 || batch > pa::kMaxBatch)
    return fail(PA_ERR_INVALID, "pa_decode_attention_int8: batch %d outside [0, %d]", batch,
                pa::kMaxBatch);
  if (num_kv_heads < 1 || num_kv_heads > pa::kMaxKvHeads || num_q_heads < num_kv_heads ||
      num_q_heads % num_kv_heads || num_q_heads / num_kv_heads > 8)
    return fail(PA_ERR_INVALID, "pa_decode_attention_int8: num_q_heads %d must be 1..8 times "
                "num_kv_heads %d (at most %d)", num_q_heads, num_kv_heads, pa::kMaxKvHeads);
  if (head_dim != pa::i8::kDim)
    return fail(PA_ERR_INVALID, "pa_decode_attention_int8: head_dim %d is not 128", head_dim);
  if (block_size != 16 && block_size != 32 && block_size != 64 && block_size != 128)
    return fail(PA_ERR_INVALID, "pa_decode_attention_int8: block_size %d not in "
                "{16, 32, 64, 128}", block_size);
  if (num_blocks < 0 || max_blocks < 0)
    return fail(PA_ERR_INVALID, "pa_decode_attention_int8: negative num_blocks or max_blocks");
  if (static_cast<int64_t>(num_blocks) * num_kv_heads * block_size >= (int64_t(1) << 31) ||
      static_cast<int64_t>(num_kv_heads) * max_blocks >= (int64_t(1) << 31))
    return fail(PA_ERR_INVALID, "pa_decode_attention_int8: num_blocks * num_kv_heads * "
                "block_size or num_kv_heads * max_blocks >= 2^31");
  if (!(scale == scale)) return fail(PA_ERR_INVALID, "pa_decode_attention_int8: scale is NaN");
  if (static_cast<int64_t>(batch) * num_kv_heads > pa::kMaxArrivals)
    return fail(PA_ERR_INVALID, "pa_decode_attention_int8: batch * num_kv_heads > %d",
                pa::kMaxArrivals);
  if (flags & ~(PA_DECODE_OVERLAP_PROLOGUE | PA_DECODE_TEST_WAIT_EXPIRY))
    return fail(PA_ERR_INVALID, "pa_decode_attention_int8: unknown flags 0x%x", flags);
  if (batch == 0) return PA_OK;
  if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens || !workspace)
    return fail(PA_ERR_INVALID, "pa_decode_attention_int8: NULL pointer");
  if (!aligned(q, 4) || !aligned(out, 4) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
      !aligned(workspace, 16) || !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return fail(PA_ERR_INVALID, "pa_decode_attention_int8: misaligned pointer");
  const size_t need = pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim);
  if (workspace_bytes < need)
    return fail(PA_ERR_INVALID, "pa_decode_attention_int8: workspace %zu bytes < %zu needed",
                workspace_bytes, need);
  const int group = num_q_heads / num_kv_heads;
  int workers = (sm_count() ? sm_count() : 148) * pa::decode_int8_workers_per_cta();
  if (num_workers > 0) workers = num_workers;
  if (workers > max_workers(group)) workers = max_workers(group);

  pa::DecodeArgs a;
  a.out = out;
  a.q = q;
  a.k_cache = k_pool;
  a.v_cache = v_pool;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.dev_error = dev_error;
  a.ws_ctrl = static_cast<uint32_t*>(workspace);
  a.ws_arrivals = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + kArrivalsOffset);
  a.ws_pieces = reinterpret_cast<float*>(static_cast<char*>(workspace) + kArrivalsEnd);
  a.batch = batch;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.group = group;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.max_blocks = max_blocks;
  a.workers = workers;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.test_expire = (flags & PA_DECODE_TEST_WAIT_EXPIRY) ? 1 : 0;
  const int per = pa::decode_int8_workers_per_cta();
  const cudaError_t e = pa::launch_decode_int8(a, dtype, (workers + per - 1) / per,
                                               (flags & PA_DECODE_OVERLAP_PROLOGUE) != 0,
                                               static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "pa_decode_attention_int8 (decode kernel)");
}

pa_status pa_prefill_attention_ex(void* out, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* block_tables,
                                  const int32_t* context_lens, const int32_t* query_start,
                                  int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                  int32_t max_blocks, int32_t total_q, int32_t max_q, float scale,
                                  pa_dtype dtype, int32_t* dev_error, void* workspace,
                                  int32_t path, pa_stream stream) {
  if (path != PA_PREFILL_AUTO && path != PA_PREFILL_TCGEN05 && path != PA_PREFILL_MMA_SYNC &&
      path != PA_PREFILL_TCGEN05_PAIR)
    return fail(PA_ERR_INVALID, "pa_prefill_attention: unknown path %d", path);
  if (dtype != PA_F16 && dtype != PA_BF16)
    return fail(PA_ERR_INVALID, "pa_prefill_attention: dtype must be fp16 or bf16");
  if (total_q < 0) return fail(PA_ERR_INVALID, "pa_prefill_attention: negative total_q");
  if (batch < 0 || batch > 65535)
    return fail(PA_ERR_INVALID, "pa_prefill_attention: batch %d outside [0, 65535]", batch);
  if (num_kv_heads < 1 || num_kv_heads > 65535 || num_q_heads < num_kv_heads ||
      num_q_heads % num_kv_heads || 64 % (num_q_heads / num_kv_heads))
    return fail(PA_ERR_INVALID, "pa_prefill_attention: num_q_heads %d / num_kv_heads %d must be "
                "a divisor of 64", num_q_heads, num_kv_heads);
  if (head_dim != 64 && head_dim != 128)
    return fail(PA_ERR_INVALID, "pa_prefill_attention: head_dim %d not in {64, 128}", head_dim);
  if (block_size < 16 || block_size % 16 || block_size > 1024)
    return fail(PA_ERR_INVALID, "pa_prefill_attention: block_size %d must be a multiple of 16",
                block_size);
  if (num_blocks < 0 || max_blocks < 0 || max_q < 0)
    return fail(PA_ERR_INVALID, "pa_prefill_attention: negative size");
  const int64_t rows = static_cast<int64_t>(num_blocks) * num_kv_heads * block_size;
  if (rows >= (int64_t(1) << 31) ||
      static_cast<int64_t>(max_blocks) * block_size >= (int64_t(1) << 31))
    return fail(PA_ERR_INVALID, "pa_prefill_attention: pool or table too large");
  const int group = num_q_heads / num_kv_heads;
  if (static_cast<int64_t>(max_q) * group > INT32_MAX - 256)
    return fail(PA_ERR_INVALID, "pa_prefill_attention: max_q too large");
  if (!(scale == scale)) return fail(PA_ERR_INVALID, "pa_prefill_attention: scale is NaN");
  if (batch == 0 || max_q == 0 || total_q == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start)
    return fail(PA_ERR_INVALID, "pa_prefill_attention: NULL pointer");
  if (!aligned(q, 4) || !aligned(out, 4) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(query_start, 4) ||
      !aligned(workspace, 8))
    return fail(PA_ERR_INVALID, "pa_prefill_attention: misaligned pointer");
  const bool tc5_ok = head_dim == 128 && 128 % group == 0 && aligned(q, 16) &&
                      aligned(out, 16) && scale > 0.f;
  if ((path == PA_PREFILL_TCGEN05 || path == PA_PREFILL_TCGEN05_PAIR) && !tc5_ok)
    return fail(PA_ERR_INVALID, "pa_prefill_attention: the tcgen05 kernels need head_dim 128, "
                "num_q_heads / num_kv_heads dividing 128, scale > 0 and q, out 16-byte aligned");
  const bool use_pair = path == PA_PREFILL_TCGEN05_PAIR;
  const bool use_tc5 = path == PA_PREFILL_TCGEN05 || (path == PA_PREFILL_AUTO && tc5_ok);
  CUtensorMap qmap, omap, kmap, vmap;
  bool k3 = false, v3 = false;
  if (use_pair) {
    if (!make_q_map(&qmap, q, total_q, num_q_heads, head_dim, group, dtype) ||
        !make_q_map(&omap, out, total_q, num_q_heads, head_dim, group, dtype) ||
        !make_tile_map_2d(&kmap, k_cache, rows, head_dim, dtype) ||
        !make_tile_map_2d(&vmap, v_cache, rows, head_dim, dtype))
      return fail(PA_ERR_CUDA, "pa_prefill_attention: cuTensorMapEncodeTiled failed");
  } else if (use_tc5) {
    if (!make_q_map(&qmap, q, total_q, num_q_heads, head_dim, group, dtype) ||
        !make_tile_map_2d(&kmap, k_cache, rows, head_dim, dtype) ||
        !make_tile_map(&vmap, &v3, v_cache, rows, head_dim, dtype) || !v3)
      return fail(PA_ERR_CUDA, "pa_prefill_attention: cuTensorMapEncodeTiled failed");
  } else if (!tile_map(&kmap, &k3, k_cache, rows, head_dim, dtype) ||
             !tile_map(&vmap, &v3, v_cache, rows, head_dim, dtype) || k3 != v3) {
    return fail(PA_ERR_CUDA, "pa_prefill_attention: cuTensorMapEncodeTiled failed");
  }
  pa::PrefillArgs a;
  a.out = out;
  a.q = q;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.query_start = query_start;
  a.dev_error = dev_error;
  a.batch = batch;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.group = group;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.max_blocks = max_blocks;
  a.max_q = max_q;
  a.total_q = total_q;
  a.three_d = k3 ? 1 : 0;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.tiles = 0;
  a.sched = static_cast<uint64_t*>(workspace);
  {
    // Pairs whose keys and values (at the table's full length) fit in about a
    // third of L2 form one scheduling block: within it the items go longest
    // first, so the kernel does not end on a long item, while the pairs being
    // read at one time still fit in L2.
    const int64_t pair_bytes =
        std::max<int64_t>(1, static_cast<int64_t>(max_blocks) * block_size * head_dim * 2 * 2);
    const int64_t pairs = static_cast<int64_t>(batch) * num_kv_heads;
    a.pair_block = static_cast<int32_t>(
        std::min<int64_t>(pairs, std::max<int64_t>(1, (int64_t(40) << 20) / pair_bytes)));
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e =
      use_pair  ? pa::launch_prefill_pair(a, dtype, qmap, kmap, vmap, omap, st)
      : use_tc5 ? pa::launch_prefill_tc5(a, dtype, qmap, kmap, vmap, st)
                : pa::launch_prefill(a, dtype, kmap, vmap, st);
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "pa_prefill_attention");
}

pa_status pa_prefill_attention(void* out, const void* q, const void* k_cache,
                               const void* v_cache, const int32_t* block_tables,
                               const int32_t* context_lens, const int32_t* query_start,
                               int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                               int32_t head_dim, int32_t block_size, int32_t num_blocks,
                               int32_t max_blocks, int32_t total_q, int32_t max_q, float scale,
                               pa_dtype dtype, int32_t* dev_error, pa_stream stream) {
  return pa_prefill_attention_ex(out, q, k_cache, v_cache, block_tables, context_lens,
                                 query_start, batch, num_q_heads, num_kv_heads, head_dim,
                                 block_size, num_blocks, max_blocks, total_q, max_q, scale, dtype,
                                 dev_error, nullptr, PA_PREFILL_AUTO, stream);
}

pa_status pa_check_device_error(int32_t* dev_error, int32_t* flags_out, pa_stream stream) {
  if (!dev_error) return fail(PA_ERR_INVALID, "pa_check_device_error: NULL pointer");
  int32_t h = 0;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&h, dev_error, sizeof h, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "pa_check_device_error");
  if (flags_out) *flags_out = h;
  if (h) {
    e = cudaMemsetAsync(dev_error, 0, sizeof(int32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "pa_check_device_error");
    return fail(PA_ERR_DEVICE, "device error bits 0x%x", h);
  }
  return PA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode attention for callers that cannot allocate device memory.
//
// pa_decode_attention needs a scratch buffer from its caller.  Some callers
// have no way to provide one: an embedding host that owns every device
// allocation and exposes none to plug-ins, a serving loop that must never call
// cudaMalloc while requests are in flight (the call can synchronise the device
// and stall every other stream), or a process whose memory is fully reserved
// by another runtime's caching allocator.  For them the library keeps one
// scratch area of its own in device memory, declared below, and
// pa_decode_attention_static_ws uses it instead of a caller buffer.
//
// The area is kStaticScratchBytes (28 MiB).  That covers the workspace of every
// shape pa_decode_attention accepts whose group (num_q_heads / num_kv_heads)
// is at most 2048 -- at most 3073 ranges x 2 piece slots x 8 heads x
// (128 + 2) floats for groups up to 8, and no more than 27.7 MB of pieces for
// any group up to 2048 -- plus the 1 MiB of arrival counts and the 256-byte
// header.  Larger groups can need more and are rejected.  Every GPU that loads
// this library holds those 28 MiB until the process exits.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kStaticScratchBytes = size_t(28) << 20;
}

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

namespace {

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};

// Device address of g_decode_scratch on the current device.  In host code the
// symbol name is only a host-side handle, so the address is looked up once per
// device (with that device current) and remembered.
pa_status static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "pa_decode_attention_static_ws (cudaGetDevice)");
  if (dev < 0 || dev >= 64)
    return fail(PA_ERR_INVALID, "pa_decode_attention_static_ws: device %d not supported", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess)
      return cuda_fail(e, "pa_decode_attention_static_ws (cudaGetSymbolAddress)");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_attention_static_ws(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, int32_t batch,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
    int32_t num_blocks, int32_t max_blocks, float scale, pa_dtype dtype, int32_t* dev_error,
    pa_stream stream) {
  // Every argument is checked before the device is touched.
  const pa_status chk = check_decode_args(dtype, batch, num_q_heads, num_kv_heads, head_dim,
                                          block_size, num_blocks, max_blocks, scale);
  if (chk != PA_OK) return chk;
  const size_t need = pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim);
  if (need > kStaticScratchBytes)
    return fail(PA_ERR_INVALID,
                "pa_decode_attention_static_ws: this shape needs %zu bytes of scratch, more "
                "than the library's fixed %zu-byte area; use pa_decode_attention with a "
                "caller-provided workspace", need, kStaticScratchBytes);
  if (batch == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return fail(PA_ERR_INVALID, "pa_decode_attention: NULL pointer");
  void* scratch = nullptr;
  const pa_status st = static_scratch(&scratch);
  if (st != PA_OK) return st;
  // The counters this call uses (the header and one arrival word per
  // (sequence, kv head)) are cleared on the call's stream first, so a call
  // that an earlier one left unfinished (PA_DEVERR_TIMEOUT) starts clean; the
  // piece slots are written before they are read.
  const size_t counters = kArrivalsOffset + sizeof(uint32_t) * static_cast<size_t>(batch) *
                                                num_kv_heads;
  const cudaError_t e =
      cudaMemsetAsync(scratch, 0, counters, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pa_decode_attention_static_ws (clear counters)");
  return pa_decode_attention_ex(out, q, k_cache, v_cache, block_tables, context_lens, batch,
                                num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                max_blocks, scale, dtype, scratch, kStaticScratchBytes,
                                dev_error, PA_PATH_AUTO, 0, 0, stream);
}
