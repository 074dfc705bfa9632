"""Python binding for libpagedattn (paged KV cache + paged decode attention, sm_100a).

Argument marshalling only: every step of the hot path runs in the CUDA library
(``libpagedattn.so``, built by ``build.py`` from ``csrc/``).  There is no CPU or
PyTorch fallback: importing this package fails if the library is missing, and
every device call requires CUDA tensors.  Names follow the C ABI in
``include/pa.h``.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

PA_OK, PA_ERR_INVALID, PA_ERR_OOM, PA_ERR_NOT_FOUND, PA_ERR_CUDA, PA_ERR_DEVICE = range(6)
PA_F32, PA_F16, PA_BF16 = 0, 1, 2
PA_PATH_AUTO, PA_PATH_TC, PA_PATH_SIMT = 0, 1, 2
PA_DECODE_OVERLAP_PROLOGUE = 1
PA_DECODE_TEST_WAIT_EXPIRY = 0x100  # tests of the failure path only (see include/pa.h)
PA_PREFILL_AUTO, PA_PREFILL_TCGEN05, PA_PREFILL_MMA_SYNC, PA_PREFILL_TCGEN05_PAIR = 0, 1, 2, 3
PA_PREFILL_WORKSPACE_BYTES = 16
PA_DEVERR_BAD_SLOT, PA_DEVERR_BAD_BLOCK, PA_DEVERR_BAD_CTX, PA_DEVERR_TIMEOUT = 1, 2, 4, 8

DTYPE_CODE = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}

_P = C.c_void_p
_I32 = C.c_int32
_I64 = C.c_int64

# name -> (restype, argtypes), mirroring include/pa.h
SIGNATURES = {
    "pa_pool_create": (_I32, [_I32, _I32, C.POINTER(_P)]),
    "pa_pool_destroy": (None, [_P]),
    "pa_alloc": (_I32, [_P, _I64, _I32, _P, _P, _I32, _P]),
    "pa_alloc_batch": (_I32, [_P, _P, _I32, _I32, _P, _P, _I32, _P]),
    "pa_swap": (_I32, [_P, _P, _I64, _P, _I32, _P]),
    "pa_swap_blocks": (_I32, [_P, _P, _P, _P, _I32, _P, _I32, _I32, _I32, _I64, _P, _P]),
    "pa_alloc_tokens": (_I32, [_P, _I64, _P, _I32, _P, _P, _I32, _P, _P]),
    "pa_pool_set_prefix_caching": (_I32, [_P, _I32]),
    "pa_num_cached_blocks": (_I32, [_P]),
    "pa_num_evictable_blocks": (_I32, [_P]),
    "pa_free": (_I32, [_P, _I64]),
    "pa_fork": (_I32, [_P, _I64, _I64]),
    "pa_block_table": (_I32, [_P, _P, _I32, _I32, _P, _P]),
    "pa_num_free_blocks": (_I32, [_P]),
    "pa_refcount": (_I32, [_P, _I32]),
    "pa_seq_len": (_I64, [_P, _I64]),
    "pa_kv_bytes": (C.c_uint64, [_I32, _I64, _I32, _I32, _I32]),
    "pa_reshape_and_cache": (_I32, [_P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, C.c_int,
                                    _P, _P]),
    "pa_copy_blocks": (_I32, [_P, _P, _I32, _P, _I32, _I32, _I64, _P, _P]),
    "pa_decode_workspace_size": (C.c_size_t, [_I32, _I32, _I32, _I32]),
    "pa_decode_attention": (_I32, [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32,
                                   _I32, C.c_float, C.c_int, _P, C.c_size_t, _P, _P]),
    "pa_decode_attention_ex": (_I32, [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                      _I32, _I32, C.c_float, C.c_int, _P, C.c_size_t, _P, _I32,
                                      _I32, _I32, _P]),
    "pa_decode_attention_static_ws": (_I32, [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32,
                                             _I32, _I32, _I32, C.c_float, C.c_int, _P, _P]),
    "pa_prefill_attention": (_I32, [_P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                    _I32, _I32, _I32, _I32, C.c_float, C.c_int, _P, _P]),
    "pa_prefill_attention_ex": (_I32, [_P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                       _I32, _I32, _I32, _I32, C.c_float, C.c_int, _P, _P, _I32,
                                       _P]),
    "pa_int8_block_bytes": (C.c_size_t, [_I32, _I32, _I32]),
    "pa_reshape_and_cache_int8": (_I32, [_P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                         C.c_int, _P, _P]),
    "pa_decode_attention_int8": (_I32, [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                        _I32, _I32, C.c_float, C.c_int, _P, C.c_size_t, _P, _I32,
                                        _I32, _P]),
    "pa_decode_plan": (_I32, [_I32, _I32, _I32, _I32, _I32, C.c_int, _P, _P]),
    "pa_validate_slot_mapping": (_I32, [_P, _I32, _I32, _I32]),
    "pa_validate_block_table": (_I32, [_P, _P, _I32, _I32, _I32, _I32]),
    "pa_validate_copy_pairs": (_I32, [_P, _I32, _I32]),
    "pa_check_device_error": (_I32, [_P, _P, _P]),
    "pa_last_error": (C.c_char_p, []),
    "pa_device_sm_count": (_I32, []),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python paged_kv_cache_486_b200/build.py` "
            "(there is no fallback implementation)")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


class PagedAttnError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"[status {status}] {message}")
        self.status = status


def _check(st, name):
    if st != PA_OK:
        raise PagedAttnError(st, f"{name}: {lib.pa_last_error().decode()}")


def _np_ptr(a):
    return a.ctypes.data_as(_P)


def _dev_ptr(t, name, dtype=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return _P(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return _P(s.cuda_stream)


# ---------------------------------------------------------------- host pool
class Pool:
    """Host block pool (``pa_pool_*``): free stack, holder counts, block lists."""

    def __init__(self, num_blocks: int, block_size: int):
        h = _P()
        _check(lib.pa_pool_create(num_blocks, block_size, C.byref(h)), "pa_pool_create")
        self._h = h
        self.num_blocks = num_blocks
        self.block_size = block_size
        self._pair = np.zeros(2, dtype=np.int32)
        self._ncow = np.zeros(1, dtype=np.int32)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and lib is not None:  # the library may be gone at interpreter shutdown
            lib.pa_pool_destroy(h)
            self._h = None

    def pa_alloc(self, seq_id: int, n_new: int):
        """-> (slot_mapping int64[n_new], cow_pairs int32[k, 2]), k in {0, 1}."""
        slots = np.empty(max(n_new, 1), dtype=np.int64)
        st = lib.pa_alloc(self._h, seq_id, n_new, _np_ptr(slots), _np_ptr(self._pair), 1,
                          _np_ptr(self._ncow))
        _check(st, "pa_alloc")
        return slots[:n_new], self._pair.reshape(1, 2)[: int(self._ncow[0])].copy()

    def pa_alloc_batch(self, seq_ids, n_new_each: int, slots_out=None):
        """-> (slot_mapping int64[n * n_new_each], cow_pairs int32[k, 2]); all or nothing."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        n = len(ids)
        slots = slots_out if slots_out is not None else np.empty(max(n * n_new_each, 1),
                                                                 dtype=np.int64)
        pairs = np.empty((max(n, 1), 2), dtype=np.int32)
        st = lib.pa_alloc_batch(self._h, _np_ptr(ids), n, n_new_each, _np_ptr(slots),
                                _np_ptr(pairs), n, _np_ptr(self._ncow))
        _check(st, "pa_alloc_batch")
        return slots[:n * n_new_each], pairs[: int(self._ncow[0])].copy()

    def pa_alloc_tokens(self, seq_id: int, token_ids):
        """Grow seq_id by the given token ids -> (slot_mapping int64[n] with -1 for tokens
        served from the prefix cache, cow_pairs int32[k, 2], n_cached)."""
        ids = np.ascontiguousarray(token_ids, dtype=np.int32)
        n = len(ids)
        slots = np.empty(max(n, 1), dtype=np.int64)
        cached = np.zeros(1, dtype=np.int32)
        st = lib.pa_alloc_tokens(self._h, seq_id, _np_ptr(ids) if n else None, n, _np_ptr(slots),
                                 _np_ptr(self._pair), 1, _np_ptr(self._ncow), _np_ptr(cached))
        _check(st, "pa_alloc_tokens")
        return (slots[:n], self._pair.reshape(1, 2)[: int(self._ncow[0])].copy(),
                int(cached[0]))

    def pa_set_prefix_caching(self, enable: bool):
        _check(lib.pa_pool_set_prefix_caching(self._h, 1 if enable else 0),
               "pa_pool_set_prefix_caching")

    def pa_num_cached_blocks(self) -> int:
        return lib.pa_num_cached_blocks(self._h)

    def pa_num_evictable_blocks(self) -> int:
        return lib.pa_num_evictable_blocks(self._h)

    def pa_free(self, seq_id: int):
        _check(lib.pa_free(self._h, seq_id), "pa_free")

    def pa_fork(self, parent_id: int, child_id: int):
        _check(lib.pa_fork(self._h, parent_id, child_id), "pa_fork")

    def pa_block_table(self, seq_ids, max_blocks: int, out_table=None, out_ctx=None):
        """-> (block_tables int32[n, max_blocks] padded with -1, context_lens int32[n])."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        table = out_table if out_table is not None else np.empty((len(ids), max_blocks), np.int32)
        ctx = out_ctx if out_ctx is not None else np.empty(len(ids), np.int32)
        _check(lib.pa_block_table(self._h, _np_ptr(ids), len(ids), max_blocks, _np_ptr(table),
                                  _np_ptr(ctx)), "pa_block_table")
        return table, ctx

    def pa_num_free_blocks(self) -> int:
        return lib.pa_num_free_blocks(self._h)

    def pa_refcount(self, block: int) -> int:
        return lib.pa_refcount(self._h, block)

    def pa_seq_len(self, seq_id: int) -> int:
        return lib.pa_seq_len(self._h, seq_id)


def pa_swap(from_pool, to_pool, seq_id):
    """Move seq_id between pools -> (from_block, to_block) pairs int32[n, 2]."""
    n_max = max(from_pool.num_blocks, 1)
    pairs = np.empty((n_max, 2), dtype=np.int32)
    n = _I32(0)
    _check(lib.pa_swap(from_pool._h, to_pool._h, seq_id, _np_ptr(pairs), n_max, C.byref(n)),
           "pa_swap")
    return pairs[: n.value].copy()


def _any_ptr(t, name):
    if not isinstance(t, torch.Tensor) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous tensor")
    if not t.is_cuda and not t.is_pinned():
        raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
    return _P(t.data_ptr())


def pa_swap_blocks(dst_k, dst_v, src_k, src_v, pairs, dev_error=None, stream=None):
    """Lists of per-layer pools (CUDA or pinned host tensors) [NB, Hkv, bs, D];
    pairs int32 [n, 2] (from, to), CUDA or pinned host."""
    L = len(dst_k)
    arr = lambda xs, nm: (_P * L)(*[_any_ptr(x, nm).value for x in xs])
    n = 0 if pairs is None else pairs.shape[0]
    if n and pairs.dtype != torch.int32:
        raise ValueError("pairs must be int32")
    block_bytes = src_k[0][0].numel() * src_k[0].element_size()
    st = lib.pa_swap_blocks(arr(dst_k, "dst_k"), arr(dst_v, "dst_v"), arr(src_k, "src_k"),
                            arr(src_v, "src_v"), L, _any_ptr(pairs, "pairs") if n else None, n,
                            src_k[0].shape[0], dst_k[0].shape[0], block_bytes,
                            _dev_ptr(dev_error, "dev_error", torch.int32), _stream(stream))
    _check(st, "pa_swap_blocks")


def pa_kv_bytes(num_layers, num_tokens, num_kv_heads, head_dim, dtype_bytes) -> int:
    return int(lib.pa_kv_bytes(num_layers, num_tokens, num_kv_heads, head_dim, dtype_bytes))


# ------------------------------------------------------------- device calls
def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, dev_error=None,
                         stream=None):
    """key/value [T, Hkv, D]; caches [NB, Hkv, bs, D]; slot_mapping int64 [T] (CUDA)."""
    T, Hkv, D = key.shape
    NB, Hkv2, bs, D2 = k_cache.shape
    if (Hkv, D) != (Hkv2, D2) or value.shape != key.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between key/value and the caches")
    dt = DTYPE_CODE[key.dtype]
    st = lib.pa_reshape_and_cache(
        _dev_ptr(key, "key"), _dev_ptr(value, "value", key.dtype),
        _dev_ptr(k_cache, "k_cache", key.dtype), _dev_ptr(v_cache, "v_cache", key.dtype),
        _dev_ptr(slot_mapping, "slot_mapping", torch.int64), T, Hkv, D, bs, NB, dt,
        _dev_ptr(dev_error, "dev_error", torch.int32), _stream(stream))
    _check(st, "pa_reshape_and_cache")


def pa_copy_blocks(k_caches, v_caches, pairs, dev_error=None, stream=None):
    """k_caches / v_caches: lists of per-layer pools; pairs int32 [n, 2] (CUDA)."""
    L = len(k_caches)
    kp = (_P * L)(*[c.data_ptr() for c in k_caches])
    vp = (_P * L)(*[c.data_ptr() for c in v_caches])
    for c in list(k_caches) + list(v_caches):
        _dev_ptr(c, "cache")
    NB = k_caches[0].shape[0]
    block_bytes = k_caches[0][0].numel() * k_caches[0].element_size()
    n = 0 if pairs is None else pairs.shape[0]
    st = lib.pa_copy_blocks(kp, vp, L, _dev_ptr(pairs, "pairs", torch.int32) if n else None, n,
                            NB, block_bytes, _dev_ptr(dev_error, "dev_error", torch.int32),
                            _stream(stream))
    _check(st, "pa_copy_blocks")


def pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim) -> int:
    return int(lib.pa_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim))


def pa_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, block_size, dtype):
    path, workers = _I32(), _I32()
    _check(lib.pa_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, block_size,
                              DTYPE_CODE[dtype], C.byref(path), C.byref(workers)),
           "pa_decode_plan")
    return path.value, workers.value


def pa_decode_attention(out, q, k_cache, v_cache, block_tables, context_lens, scale, workspace,
                        dev_error=None, path=PA_PATH_AUTO, num_workers=0, flags=0, stream=None):
    """q/out [B, Hq, D]; caches [NB, Hkv, bs, D]; block_tables int32 [B, MB];
    context_lens int32 [B]; workspace uint8 [>= pa_decode_workspace_size], zero-filled
    before its first use (all CUDA)."""
    B, Hq, D = q.shape
    NB, Hkv, bs, _ = k_cache.shape
    MB = block_tables.shape[1]
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    st = lib.pa_decode_attention_ex(
        _dev_ptr(out, "out", q.dtype), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache", q.dtype),
        _dev_ptr(v_cache, "v_cache", q.dtype), _dev_ptr(block_tables, "block_tables", torch.int32),
        _dev_ptr(context_lens, "context_lens", torch.int32), B, Hq, Hkv, D, bs, NB, MB,
        float(scale), DTYPE_CODE[q.dtype], _dev_ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(),
        _dev_ptr(dev_error, "dev_error", torch.int32), path, num_workers, flags, _stream(stream))
    _check(st, "pa_decode_attention")


def pa_decode_attention_static_ws(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                                  dev_error=None, stream=None):
    """pa_decode_attention for callers that cannot allocate device memory: the
    library's own fixed 28 MiB device scratch replaces the workspace.  Calls that
    overlap on the GPU share that scratch and race; order them on one stream."""
    B, Hq, D = q.shape
    NB, Hkv, bs, _ = k_cache.shape
    MB = block_tables.shape[1]
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    st = lib.pa_decode_attention_static_ws(
        _dev_ptr(out, "out", q.dtype), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache", q.dtype),
        _dev_ptr(v_cache, "v_cache", q.dtype), _dev_ptr(block_tables, "block_tables", torch.int32),
        _dev_ptr(context_lens, "context_lens", torch.int32), B, Hq, Hkv, D, bs, NB, MB,
        float(scale), DTYPE_CODE[q.dtype], _dev_ptr(dev_error, "dev_error", torch.int32),
        _stream(stream))
    _check(st, "pa_decode_attention_static_ws")


def pa_prefill_attention(out, q, k_cache, v_cache, block_tables, context_lens, query_start,
                         max_q, scale, dev_error=None, path=PA_PREFILL_AUTO, workspace=None,
                         stream=None):
    """Causal attention of each sequence's new tokens over its paged cache: q/out
    [T, Hq, D] fp16 or bf16, query_start int32 [B+1] (device), max_q >= every
    query_start[b+1] - query_start[b]; caches and tables as pa_decode_attention.
    workspace: None or int64 [2] zero-filled once (persistent tcgen05 kernel)."""
    T, Hq, D = q.shape
    NB, Hkv, bs, _ = k_cache.shape
    B = context_lens.shape[0]
    MB = block_tables.shape[1]
    if out.shape != q.shape or query_start.shape[0] != B + 1:
        raise ValueError("out must have q's shape and query_start batch + 1 entries")
    if workspace is not None and workspace.numel() * workspace.element_size() < \
            PA_PREFILL_WORKSPACE_BYTES:
        raise ValueError(f"workspace needs {PA_PREFILL_WORKSPACE_BYTES} bytes")
    st = lib.pa_prefill_attention_ex(
        _dev_ptr(out, "out", q.dtype), _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache", q.dtype),
        _dev_ptr(v_cache, "v_cache", q.dtype), _dev_ptr(block_tables, "block_tables", torch.int32),
        _dev_ptr(context_lens, "context_lens", torch.int32),
        _dev_ptr(query_start, "query_start", torch.int32), B, Hq, Hkv, D, bs, NB, MB, T, int(max_q),
        float(scale), DTYPE_CODE[q.dtype], _dev_ptr(dev_error, "dev_error", torch.int32),
        _dev_ptr(workspace, "workspace", torch.int64), path, _stream(stream))
    _check(st, "pa_prefill_attention")


INT8_RECORD_BYTES = 2112  # one 16-token group of one (block, kv head): codes + fp32 scales


def pa_int8_block_bytes(num_kv_heads, head_dim, block_size) -> int:
    return int(lib.pa_int8_block_bytes(num_kv_heads, head_dim, block_size))


def pa_reshape_and_cache_int8(key, value, k_pool, v_pool, slot_mapping, dev_error=None,
                              stream=None):
    """Quantise key/value [T, Hkv, 128] into an INT8 cache: k_pool / v_pool uint8
    [NB, Hkv, bs/16, 2112] records (layout in include/pa.h)."""
    T, Hkv, D = key.shape
    NB, Hkv2, G16, R = k_pool.shape
    if (Hkv != Hkv2 or value.shape != key.shape or v_pool.shape != k_pool.shape
            or R != INT8_RECORD_BYTES):
        raise ValueError("shape mismatch between key/value and the INT8 pools")
    st = lib.pa_reshape_and_cache_int8(
        _dev_ptr(key, "key"), _dev_ptr(value, "value", key.dtype),
        _dev_ptr(k_pool, "k_pool", torch.uint8), _dev_ptr(v_pool, "v_pool", torch.uint8),
        _dev_ptr(slot_mapping, "slot_mapping", torch.int64), T, Hkv, D, 16 * G16, NB,
        DTYPE_CODE[key.dtype], _dev_ptr(dev_error, "dev_error", torch.int32), _stream(stream))
    _check(st, "pa_reshape_and_cache_int8")


def pa_decode_attention_int8(out, q, k_pool, v_pool, block_tables, context_lens, scale,
                             workspace, dev_error=None, num_workers=0, flags=0, stream=None):
    """Decode attention over an INT8 cache (pools as pa_reshape_and_cache_int8); q/out
    [B, Hq, 128] fp16 or bf16; the other arguments as pa_decode_attention."""
    B, Hq, D = q.shape
    NB, Hkv, G16, _ = k_pool.shape
    MB = block_tables.shape[1]
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    st = lib.pa_decode_attention_int8(
        _dev_ptr(out, "out", q.dtype), _dev_ptr(q, "q"), _dev_ptr(k_pool, "k_pool", torch.uint8),
        _dev_ptr(v_pool, "v_pool", torch.uint8),
        _dev_ptr(block_tables, "block_tables", torch.int32),
        _dev_ptr(context_lens, "context_lens", torch.int32), B, Hq, Hkv, D, 16 * G16, NB, MB,
        float(scale), DTYPE_CODE[q.dtype], _dev_ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(),
        _dev_ptr(dev_error, "dev_error", torch.int32), num_workers, flags, _stream(stream))
    _check(st, "pa_decode_attention_int8")


def pa_check_device_error(dev_error, stream=None) -> int:
    """Returns the device error bits (and clears them); 0 if none."""
    flags = _I32(0)
    st = lib.pa_check_device_error(_dev_ptr(dev_error, "dev_error", torch.int32),
                                   C.byref(flags), _stream(stream))
    if st not in (PA_OK, PA_ERR_DEVICE):
        _check(st, "pa_check_device_error")
    return flags.value


# ----------------------------------------------------------------- validators
def pa_validate_slot_mapping(slots, block_size, num_blocks):
    s = np.ascontiguousarray(slots, dtype=np.int64)
    return lib.pa_validate_slot_mapping(_np_ptr(s), len(s), block_size, num_blocks)


def pa_validate_block_table(block_tables, context_lens, block_size, num_blocks):
    t = np.ascontiguousarray(block_tables, dtype=np.int32)
    c = np.ascontiguousarray(context_lens, dtype=np.int32)
    return lib.pa_validate_block_table(_np_ptr(t), _np_ptr(c), t.shape[0], t.shape[1], block_size,
                                       num_blocks)


def pa_validate_copy_pairs(pairs, num_blocks):
    p = np.ascontiguousarray(pairs, dtype=np.int32).reshape(-1, 2)
    return lib.pa_validate_copy_pairs(_np_ptr(p), p.shape[0], num_blocks)


def pa_last_error() -> str:
    return lib.pa_last_error().decode()


def pa_device_sm_count() -> int:
    return lib.pa_device_sm_count()
