"""Runs a workload's op script through the oracle (test infrastructure)."""
import concurrent.futures as cf
import os

import numpy as np
import torch

import oracle

STORAGE = {"f32": np.float32, "f16": np.uint16, "bf16": np.uint16}


def raw(t: torch.Tensor) -> np.ndarray:
    """Host numpy view of a tensor's storage bits (float32 stays float32)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.numpy()
    return t.view(torch.int16).numpy().view(np.uint16)


def run_script(wl, with_cache=True, write_tokens=True):
    """Execute every op of ``wl`` on an oracle pool.

    Returns dict(pool, table, ctx, k_cache, v_cache, records) where records[i] is
    (slots, cow_pairs) for alloc op i (None for other ops)."""
    pool = oracle.Pool(wl.num_blocks, wl.bs)
    shape = (wl.num_blocks, wl.Hkv, wl.bs, wl.D)
    kc = np.zeros(shape, dtype=STORAGE[wl.dtype]) if with_cache else None
    vc = np.zeros(shape, dtype=STORAGE[wl.dtype]) if with_cache else None
    records = []
    for op in wl.ops:
        if op[0] == "alloc":
            _, seq, n, pos0, write = op
            st, slots, cow = pool.alloc(seq, n)
            assert st == oracle.OK, (op, st)
            records.append((slots, cow))
            if with_cache:
                if len(cow):
                    oracle.copy_blocks([kc], [vc], cow)
                if write and write_tokens and n > 0:
                    k = raw(wl.tokens(seq, pos0, n, 0))
                    v = raw(wl.tokens(seq, pos0, n, 1))
                    assert oracle.reshape_and_cache(k, v, kc, vc, slots, wl.bs,
                                                    wl.elem_bytes) == oracle.OK
        elif op[0] == "fork":
            assert pool.fork(op[1], op[2]) == oracle.OK
            records.append(None)
        else:
            assert pool.free(op[1]) == oracle.OK
            records.append(None)
    st, table, ctx = pool.block_table(wl.batch, wl.max_blocks)
    assert st == oracle.OK
    return dict(pool=pool, table=table, ctx=ctx, k_cache=kc, v_cache=vc, records=records)


def attention(wl, state, rows=None, n_threads=None):
    q = raw(wl.q())
    return oracle.paged_decode_attention(q, state["k_cache"], state["v_cache"], state["table"],
                                         state["ctx"], wl.scale, wl.dtype, rows=rows,
                                         n_threads=n_threads)


def all_rows(wl, device="cuda", threads=None, visit=None):
    """Oracle attention [B, Hq, D] of every batch row from the sequence's logical
    key/value rows, which the seeded generator draws on `device` (the same bits on
    any device; on the GPU it is plain torch arithmetic, not the library).
    visit(b, k, v), if given, sees each row's logical keys and values first.
    The oracle releases the GIL, so rows run in parallel on the host cores."""
    q = raw(wl.q())

    def row(b):
        seq = int(wl.batch[b])
        k = wl.contiguous_kv(seq, 0, device)
        v = wl.contiguous_kv(seq, 1, device)
        seen = visit(b, k, v) if visit else None
        return seen, oracle.contiguous_attention(q[b], raw(k), raw(v), wl.scale, wl.dtype)

    with cf.ThreadPoolExecutor(threads or os.cpu_count() or 4) as ex:
        res = list(ex.map(row, range(wl.B)))
    return np.stack([r[1] for r in res]), [r[0] for r in res]


def contiguous_row(wl, b, heads=None):
    """Oracle attention of batch row b from its logical (unpaged) key/value rows."""
    seq = int(wl.batch[b])
    q = raw(wl.q()[b])
    if heads is None:
        k = raw(wl.contiguous_kv(seq, 0))
        v = raw(wl.contiguous_kv(seq, 1))
        return oracle.contiguous_attention(q, k, v, wl.scale, wl.dtype)
    # only the KV heads the listed query heads read
    kvh = sorted({h // wl.G for h in heads})
    k = raw(wl.contiguous_kv(seq, 0, heads=kvh))
    v = raw(wl.contiguous_kv(seq, 1, heads=kvh))
    out = np.full((wl.Hq, wl.D), np.nan)
    for h in heads:
        j = kvh.index(h // wl.G)
        o = oracle.contiguous_attention(q[h:h + 1], k[:, j:j + 1], v[:, j:j + 1], wl.scale,
                                        wl.dtype)
        out[h] = o[0]
    return out


def run_script_int8(wl):
    """The op script through the oracle pool with an INT8 cache (copy-on-write
    copies move codes and scales).  Returns dict(pool, table, ctx, cache)."""
    pool = oracle.Pool(wl.num_blocks, wl.bs)
    cache = oracle.Int8Cache(wl.num_blocks, wl.Hkv, wl.bs, wl.D)
    for op in wl.ops:
        if op[0] == "alloc":
            _, seq, n, pos0, write = op
            st, slots, cow = pool.alloc(seq, n)
            assert st == oracle.OK, (op, st)
            if len(cow):
                oracle.copy_blocks([cache.k], [cache.v], cow)      # codes
                oracle.copy_blocks([cache.ks], [cache.vs], cow)    # scales
            if write and n > 0:
                k = raw(wl.tokens(seq, pos0, n, 0))
                v = raw(wl.tokens(seq, pos0, n, 1))
                assert oracle.reshape_and_cache_int8(k, v, cache, slots, wl.dtype) == oracle.OK
        elif op[0] == "fork":
            assert pool.fork(op[1], op[2]) == oracle.OK
        else:
            assert pool.free(op[1]) == oracle.OK
    st, table, ctx = pool.block_table(wl.batch, wl.max_blocks)
    assert st == oracle.OK
    return dict(pool=pool, table=table, ctx=ctx, cache=cache)


def int8_contiguous_row(wl, b, heads):
    """Oracle INT8 attention of batch row b for the listed query heads, from the
    sequence's logical rows quantised into a fresh one-sequence oracle cache (the
    scheme is per (token, kv head), so each kv head is quantised on its own)."""
    seq = int(wl.batch[b])
    q = raw(wl.q()[b])
    out = np.full((wl.Hq, wl.D), np.nan)
    for h in heads:
        g = h // wl.G
        k = raw(wl.contiguous_kv(seq, 0, heads=[g]))
        v = raw(wl.contiguous_kv(seq, 1, heads=[g]))
        n = k.shape[0]
        nb = max(1, -(-n // wl.bs))
        cache = oracle.Int8Cache(nb, 1, wl.bs, wl.D)
        assert oracle.reshape_and_cache_int8(k, v, cache, np.arange(n), wl.dtype) == oracle.OK
        o = oracle.paged_decode_attention_int8(q[h:h + 1][None], cache, np.arange(nb)[None],
                                               [n], wl.scale, wl.dtype)
        out[h] = o[0, 0]
    return out


def int8_all_rows(wl, device="cuda", threads=None):
    """Oracle INT8 attention [B, Hq, D] of every batch row: each sequence's
    logical rows (drawn on `device`, the same bits anywhere) quantised into a
    fresh one-sequence oracle cache of all its kv heads, then the oracle's paged
    INT8 decode over it.  Rows run in parallel on the host cores."""
    q = raw(wl.q())

    def row(b):
        seq = int(wl.batch[b])
        k = raw(wl.contiguous_kv(seq, 0, device))
        v = raw(wl.contiguous_kv(seq, 1, device))
        n = k.shape[0]
        nb = max(1, -(-n // wl.bs))
        cache = oracle.Int8Cache(nb, wl.Hkv, wl.bs, wl.D)
        assert oracle.reshape_and_cache_int8(k, v, cache, np.arange(n), wl.dtype) == oracle.OK
        o = oracle.paged_decode_attention_int8(q[b][None], cache, np.arange(nb)[None], [n],
                                               wl.scale, wl.dtype, n_threads=1)
        return o[0]

    with cf.ThreadPoolExecutor(threads or os.cpu_count() or 4) as ex:
        return np.stack(list(ex.map(row, range(wl.B))))
