"""Python handle on the oracle (``oracle.cpp``): TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
library never imports it, and it imports nothing from the product: the two
share only the seeded input generators in ``workloads.py``.

Every function is a thin ctypes marshaller around the C++ oracle, which is the
plain fp64 restatement of the pages (see the header comment of oracle.cpp).
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None

OK, INVALID, OOM, NOT_FOUND = 0, 1, 2, 3
DTYPE_CODE = {"f32": 0, "f16": 1, "bf16": 2}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        L.orc_f16_to_f64.restype = C.c_double
        L.orc_f16_to_f64.argtypes = [C.c_uint16]
        L.orc_bf16_to_f64.restype = C.c_double
        L.orc_bf16_to_f64.argtypes = [C.c_uint16]
        L.orc_f64_to_f16.restype = C.c_uint16
        L.orc_f64_to_f16.argtypes = [C.c_double]
        L.orc_f64_to_bf16.restype = C.c_uint16
        L.orc_f64_to_bf16.argtypes = [C.c_double]
        L.orc_round_array.restype = None
        L.orc_round_array.argtypes = [P, C.c_int64, C.c_int, P]
        L.orc_kv_bytes.restype = C.c_uint64
        L.orc_kv_bytes.argtypes = [C.c_int32, C.c_int64, C.c_int32, C.c_int32, C.c_int32]
        L.orc_pool_new.restype = P
        L.orc_pool_new.argtypes = [C.c_int32, C.c_int32]
        L.orc_pool_delete.restype = None
        L.orc_pool_delete.argtypes = [P]
        L.orc_num_free.restype = C.c_int32
        L.orc_num_free.argtypes = [P]
        L.orc_holders.restype = C.c_int32
        L.orc_holders.argtypes = [P, C.c_int32]
        L.orc_alloc.restype = C.c_int
        L.orc_alloc.argtypes = [P, C.c_int64, C.c_int32, P, P, P]
        L.orc_alloc_tokens.restype = C.c_int
        L.orc_alloc_tokens.argtypes = [P, C.c_int64, P, C.c_int32, P, P, P, P]
        L.orc_paged_prefill_attention.restype = C.c_int
        L.orc_paged_prefill_attention.argtypes = [P, P, P, P, P, P, C.c_int32, C.c_int32,
                                                  C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                                                  C.c_double, C.c_int, P, P, C.c_int64,
                                                  C.c_int32]
        L.orc_set_prefix_caching.restype = None
        L.orc_set_prefix_caching.argtypes = [P, C.c_int32]
        L.orc_num_cached.restype = C.c_int32
        L.orc_num_cached.argtypes = [P]
        L.orc_num_releasable.restype = C.c_int32
        L.orc_num_releasable.argtypes = [P]
        L.orc_free.restype = C.c_int
        L.orc_free.argtypes = [P, C.c_int64]
        L.orc_fork.restype = C.c_int
        L.orc_fork.argtypes = [P, C.c_int64, C.c_int64]
        L.orc_seq_len.restype = C.c_int64
        L.orc_seq_len.argtypes = [P, C.c_int64]
        L.orc_block_table.restype = C.c_int
        L.orc_block_table.argtypes = [P, P, C.c_int32, C.c_int32, P, P]
        L.orc_reshape_and_cache.restype = C.c_int
        L.orc_reshape_and_cache.argtypes = [P, P, P, P, P, C.c_int64, C.c_int32, C.c_int32,
                                            C.c_int32, C.c_int32, C.c_int32]
        L.orc_copy_blocks.restype = C.c_int
        L.orc_copy_blocks.argtypes = [P, P, C.c_int32, P, C.c_int32, C.c_int64]
        L.orc_paged_decode_attention.restype = C.c_int
        L.orc_paged_decode_attention.argtypes = [P, P, P, P, P, C.c_int32, C.c_int32, C.c_int32,
                                                 C.c_int32, C.c_int32, C.c_int32, C.c_double,
                                                 C.c_int, P, P, C.c_int64, C.c_int32]
        L.orc_swap.restype = C.c_int
        L.orc_swap.argtypes = [P, P, C.c_int64, P, P]
        L.orc_copy_between.restype = C.c_int
        L.orc_copy_between.argtypes = [P, P, P, P, C.c_int32, P, C.c_int32, C.c_int64]
        L.orc_reshape_and_cache_int8.restype = C.c_int
        L.orc_reshape_and_cache_int8.argtypes = [P, P, P, P, P, P, P, C.c_int64, C.c_int32,
                                                 C.c_int32, C.c_int32, C.c_int32, C.c_int]
        L.orc_quantize_rows.restype = None
        L.orc_quantize_rows.argtypes = [P, C.c_int64, C.c_int32, C.c_int, P, P]
        L.orc_paged_decode_attention_int8.restype = C.c_int
        L.orc_paged_decode_attention_int8.argtypes = [P, P, P, P, P, P, P, C.c_int32, C.c_int32,
                                                      C.c_int32, C.c_int32, C.c_int32, C.c_int32,
                                                      C.c_double, C.c_int, P, P, C.c_int64,
                                                      C.c_int32]
        L.orc_contiguous_attention.restype = C.c_int
        L.orc_contiguous_attention.argtypes = [P, P, P, C.c_int64, C.c_int32, C.c_int32,
                                               C.c_int32, C.c_double, C.c_int, P, P, C.c_int32]
        L.orc_hardware_concurrency.restype = C.c_int32
        L.orc_hardware_concurrency.argtypes = []
        _lib = L
    return _lib


def hardware_concurrency():
    """std::thread::hardware_concurrency() of the oracle's C++ runtime."""
    return int(lib().orc_hardware_concurrency())


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------ numbers
def f16_to_f64(bits):
    return lib().orc_f16_to_f64(int(bits))


def bf16_to_f64(bits):
    return lib().orc_bf16_to_f64(int(bits))


def f64_to_f16(x):
    return lib().orc_f64_to_f16(float(x))


def f64_to_bf16(x):
    return lib().orc_f64_to_bf16(float(x))


def round_to(x, dtype):
    """Round fp64 values to the storage dtype; returns raw storage (uint16 or float32)."""
    x = _c(x, np.float64)
    out = np.empty(x.shape, dtype=np.float32 if dtype == "f32" else np.uint16)
    lib().orc_round_array(_ptr(x), x.size, DTYPE_CODE[dtype], _ptr(out))
    return out


def kv_bytes(num_layers, seq_length, num_kv_heads, head_dim, precision_bytes):
    return int(lib().orc_kv_bytes(num_layers, seq_length, num_kv_heads, head_dim,
                                  precision_bytes))


# --------------------------------------------------------------- pool model
class Pool:
    """The allocator restated: free stack, holder counts, per-sequence block lists."""

    def __init__(self, num_blocks, block_size):
        self.h = lib().orc_pool_new(num_blocks, block_size)
        if not self.h:
            raise ValueError("bad pool geometry")
        self.num_blocks = num_blocks
        self.block_size = block_size

    def __del__(self):
        h = getattr(self, "h", None)
        if h and _lib is not None:  # the library may be gone at interpreter shutdown
            _lib.orc_pool_delete(h)
            self.h = None

    def alloc(self, seq, n):
        """Returns (status, slots int64[n], cow pairs int32[k, 2])."""
        slots = np.zeros(max(n, 1), dtype=np.int64)
        pair = np.zeros(2, dtype=np.int32)
        ncow = np.zeros(1, dtype=np.int32)
        st = lib().orc_alloc(self.h, seq, n, _ptr(slots), _ptr(pair), _ptr(ncow))
        if st != OK:
            return st, None, None
        return st, slots[:n].copy(), pair.reshape(1, 2)[: int(ncow[0])].copy()

    def alloc_tokens(self, seq, ids):
        """Grow with token ids (prefix-cache reuse for a new sequence).
        Returns (status, slots int64[n] with -1 for cached tokens, cow pairs, n_cached)."""
        ids = _c(ids, np.int32)
        n = len(ids)
        slots = np.zeros(max(n, 1), dtype=np.int64)
        pair = np.zeros(2, dtype=np.int32)
        ncow = np.zeros(1, dtype=np.int32)
        ncached = np.zeros(1, dtype=np.int32)
        st = lib().orc_alloc_tokens(self.h, seq, _ptr(ids), n, _ptr(slots), _ptr(pair),
                                    _ptr(ncow), _ptr(ncached))
        if st != OK:
            return st, None, None, 0
        return (st, slots[:n].copy(), pair.reshape(1, 2)[: int(ncow[0])].copy(),
                int(ncached[0]))

    def set_prefix_caching(self, enable):
        lib().orc_set_prefix_caching(self.h, 1 if enable else 0)

    def num_cached(self):
        return lib().orc_num_cached(self.h)

    def num_releasable(self):
        return lib().orc_num_releasable(self.h)

    def free(self, seq):
        return lib().orc_free(self.h, seq)

    def fork(self, parent, child):
        return lib().orc_fork(self.h, parent, child)

    def num_free(self):
        return lib().orc_num_free(self.h)

    def holders(self, block):
        return lib().orc_holders(self.h, block)

    def seq_len(self, seq):
        return lib().orc_seq_len(self.h, seq)

    def block_table(self, seqs, max_blocks):
        seqs = _c(seqs, np.int64)
        table = np.empty((len(seqs), max_blocks), dtype=np.int32)
        ctx = np.empty(len(seqs), dtype=np.int32)
        st = lib().orc_block_table(self.h, _ptr(seqs), len(seqs), max_blocks, _ptr(table),
                                   _ptr(ctx))
        return st, table, ctx


def swap(from_pool, to_pool, seq):
    """Move `seq` from one pool to the other; returns (status, pairs int32[n, 2] (from, to))."""
    pairs = np.zeros((max(from_pool.num_blocks, 1), 2), dtype=np.int32)
    n = np.zeros(1, dtype=np.int32)
    st = lib().orc_swap(from_pool.h, to_pool.h, seq, _ptr(pairs), _ptr(n))
    if st != OK:
        return st, None
    return st, pairs[: int(n[0])].copy()


def copy_between(dst_k, dst_v, src_k, src_v, pairs):
    pairs = _c(pairs, np.int32).reshape(-1, 2)
    L = len(dst_k)
    arr = lambda xs: (C.c_void_p * L)(*[x.ctypes.data for x in xs])
    return lib().orc_copy_between(arr(dst_k), arr(dst_v), arr(src_k), arr(src_v), L, _ptr(pairs),
                                  pairs.shape[0], src_k[0][0].nbytes)


# ---------------------------------------------------------- data movement
def reshape_and_cache(key, value, k_cache, v_cache, slots, block_size, elem_bytes):
    """In place on numpy caches [NB, Hkv, bs, D] (raw storage dtype)."""
    T, Hkv, D = key.shape
    key = np.ascontiguousarray(key)
    value = np.ascontiguousarray(value)
    slots = _c(slots, np.int64)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    return lib().orc_reshape_and_cache(_ptr(key), _ptr(value), _ptr(k_cache), _ptr(v_cache),
                                       _ptr(slots), T, Hkv, D, block_size, k_cache.shape[0],
                                       elem_bytes)


def copy_blocks(k_caches, v_caches, pairs):
    pairs = _c(pairs, np.int32).reshape(-1, 2)
    L = len(k_caches)
    kp = (C.c_void_p * L)(*[c.ctypes.data for c in k_caches])
    vp = (C.c_void_p * L)(*[c.ctypes.data for c in v_caches])
    block_bytes = k_caches[0][0].nbytes
    return lib().orc_copy_blocks(kp, vp, L, _ptr(pairs), pairs.shape[0], block_bytes)


# --------------------------------------------------------------- attention
def paged_decode_attention(q, k_cache, v_cache, tables, ctx, scale, dtype, rows=None,
                           n_threads=None):
    """fp64 output [B, Hq, D]; rows (flat b*Hq+h) limits the work (others left NaN)."""
    q = np.ascontiguousarray(q)
    B, Hq, D = q.shape
    NB, Hkv, bs, _ = k_cache.shape
    tables = _c(tables, np.int32)
    ctx = _c(ctx, np.int32)
    out = np.full((B, Hq, D), np.nan, dtype=np.float64)
    r = None if rows is None else _c(rows, np.int64)
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    st = lib().orc_paged_decode_attention(
        _ptr(q), _ptr(np.ascontiguousarray(k_cache)), _ptr(np.ascontiguousarray(v_cache)),
        _ptr(tables), _ptr(ctx), B, Hq, Hkv, D, bs, tables.shape[1], float(scale),
        DTYPE_CODE[dtype], _ptr(out), _ptr(r), 0 if r is None else len(r), n_threads)
    if st != OK:
        raise ValueError(f"oracle attention rejected its arguments ({st})")
    return out


def contiguous_attention(q, k, v, scale, dtype, heads=None):
    """q [Hq, D], k/v [n, Hkv, D] in logical order -> fp64 [Hq, D] (unlisted heads NaN)."""
    q = np.ascontiguousarray(q)
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    Hq, D = q.shape
    n, Hkv, _ = k.shape
    out = np.full((Hq, D), np.nan, dtype=np.float64)
    hs = None if heads is None else _c(heads, np.int32)
    st = lib().orc_contiguous_attention(_ptr(q), _ptr(k), _ptr(v), n, Hq, Hkv, D, float(scale),
                                        DTYPE_CODE[dtype], _ptr(out), _ptr(hs),
                                        0 if hs is None else len(hs))
    if st != OK:
        raise ValueError(f"oracle attention rejected its arguments ({st})")
    return out


# ------------------------------------------------------------- INT8 cache
class Int8Cache:
    """Host INT8 cache in its logical layout: key codes and value codes
    [NB, Hkv, bs, D], fp32 scales [NB, Hkv, bs] for keys and values."""

    def __init__(self, num_blocks, kv_heads, block_size, head_dim):
        self.k = np.zeros((num_blocks, kv_heads, block_size, head_dim), np.int8)
        self.v = np.zeros((num_blocks, kv_heads, block_size, head_dim), np.int8)
        self.ks = np.zeros((num_blocks, kv_heads, block_size), np.float32)
        self.vs = np.zeros((num_blocks, kv_heads, block_size), np.float32)


def quantize_rows(x, dtype):
    x = np.ascontiguousarray(x)
    n, D = x.shape
    codes = np.empty((n, D), np.int8)
    scales = np.empty(n, np.float32)
    lib().orc_quantize_rows(_ptr(x), n, D, DTYPE_CODE[dtype], _ptr(codes), _ptr(scales))
    return codes, scales


def reshape_and_cache_int8(key, value, cache, slots, dtype):
    key = np.ascontiguousarray(key)
    value = np.ascontiguousarray(value)
    T, Hkv, D = key.shape
    slots = _c(slots, np.int64)
    return lib().orc_reshape_and_cache_int8(_ptr(key), _ptr(value), _ptr(cache.k), _ptr(cache.v),
                                            _ptr(cache.ks), _ptr(cache.vs), _ptr(slots), T, Hkv,
                                            D, cache.k.shape[2], cache.k.shape[0],
                                            DTYPE_CODE[dtype])


def paged_prefill_attention(q, k_cache, v_cache, tables, ctx, query_start, scale, dtype,
                            rows=None, n_threads=None):
    """Causal attention of each sequence's new tokens (the last query_start[b+1] -
    query_start[b] of its ctx[b] tokens) over its cached keys and values.
    q [total_q, Hq, D] storage bits; fp64 output [total_q, Hq, D] (rows: flat
    token * Hq + head indices to compute, others NaN)."""
    q = np.ascontiguousarray(q)
    T, Hq, D = q.shape
    NB, Hkv, bs, _ = k_cache.shape
    tables = _c(tables, np.int32)
    ctx = _c(ctx, np.int32)
    qs = _c(query_start, np.int32)
    out = np.full((T, Hq, D), np.nan)
    r = None if rows is None else _c(rows, np.int64)
    st = lib().orc_paged_prefill_attention(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(tables), _ptr(ctx), _ptr(qs), len(ctx), Hq,
        Hkv, D, bs, tables.shape[1], float(scale), DTYPE_CODE[dtype], _ptr(out), _ptr(r),
        0 if r is None else len(r), n_threads or (os.cpu_count() or 1))
    if st != OK:
        raise ValueError(f"oracle prefill attention rejected its arguments ({st})")
    return out


def paged_decode_attention_int8(q, cache, tables, ctx, scale, dtype, rows=None, n_threads=None):
    q = np.ascontiguousarray(q)
    B, Hq, D = q.shape
    NB, Hkv, bs, _ = cache.k.shape
    tables = _c(tables, np.int32)
    ctx = _c(ctx, np.int32)
    out = np.full((B, Hq, D), np.nan)
    r = None if rows is None else _c(rows, np.int64)
    st = lib().orc_paged_decode_attention_int8(
        _ptr(q), _ptr(cache.k), _ptr(cache.v), _ptr(cache.ks), _ptr(cache.vs), _ptr(tables),
        _ptr(ctx), B, Hq, Hkv, D, bs, tables.shape[1], float(scale), DTYPE_CODE[dtype], _ptr(out),
        _ptr(r), 0 if r is None else len(r), n_threads or (os.cpu_count() or 1))
    if st != OK:
        raise ValueError(f"oracle int8 attention rejected its arguments ({st})")
    return out
