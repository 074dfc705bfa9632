"""PagedKVCache: one layer's paged key/value pools plus the host block pool.

Host-side orchestration of the C ABI only (no arithmetic happens here): it
keeps the call order the library requires -- allocate slots, copy any
copy-on-write blocks, then write the new tokens -- and owns the device memory
the library itself never allocates.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (INT8_RECORD_BYTES, PA_PATH_AUTO, Pool, pa_check_device_error, pa_copy_blocks,
               pa_decode_attention, pa_decode_attention_int8, pa_decode_workspace_size,
               pa_prefill_attention, pa_reshape_and_cache, pa_reshape_and_cache_int8)


class PagedKVCache:
    def __init__(self, num_blocks, block_size, num_kv_heads, head_dim, dtype, num_q_heads,
                 max_batch, device="cuda", fill_bits=None):
        self.pool = Pool(num_blocks, block_size)
        self.num_blocks, self.block_size = num_blocks, block_size
        self.num_kv_heads, self.head_dim = num_kv_heads, head_dim
        self.num_q_heads, self.dtype, self.device = num_q_heads, dtype, torch.device(device)
        shape = (num_blocks, num_kv_heads, block_size, head_dim)
        self.k_cache = torch.empty(shape, dtype=dtype, device=self.device)
        self.v_cache = torch.empty(shape, dtype=dtype, device=self.device)
        if fill_bits is not None:  # poison unwritten slots (e.g. NaN bit patterns)
            view = torch.int16 if dtype != torch.float32 else torch.int32
            self.k_cache.view(view).fill_(fill_bits)
            self.v_cache.view(view).fill_(fill_bits)
        self.dev_error = torch.zeros(1, dtype=torch.int32, device=self.device)
        ws = pa_decode_workspace_size(max_batch, num_q_heads, num_kv_heads, head_dim)
        self.workspace = torch.zeros(ws, dtype=torch.uint8, device=self.device)
        # prefill's item counter (persistent tcgen05 kernel); every call leaves it zero
        self.prefill_ws = torch.zeros(2, dtype=torch.int64, device=self.device)

    # ---- pool ops (host) with their device side effects ----
    def alloc(self, seq_id, n, stream=None):
        """Slots (host int64) for n new tokens; runs the block copy a copy-on-write needs."""
        slots, cow = self.pool.pa_alloc(seq_id, n)
        if len(cow):
            self._copy_pairs(torch.from_numpy(cow).to(self.device, non_blocking=False), stream)
        return slots, cow

    def alloc_tokens(self, seq_id, token_ids, stream=None):
        """pa_alloc_tokens (prefix-cache reuse for a new sequence when the pool has it on)
        + the block copy a copy-on-write needs -> (slots with -1 for cached tokens,
        cow pairs, n_cached)."""
        slots, cow, n_cached = self.pool.pa_alloc_tokens(seq_id, token_ids)
        if len(cow):
            self._copy_pairs(torch.from_numpy(cow).to(self.device, non_blocking=False), stream)
        return slots, cow, n_cached

    def _copy_pairs(self, pairs, stream=None):
        pa_copy_blocks([self.k_cache], [self.v_cache], pairs, self.dev_error, stream)

    def fork(self, parent, child):
        self.pool.pa_fork(parent, child)

    def free(self, seq_id):
        self.pool.pa_free(seq_id)

    def write(self, key, value, slots, stream=None):
        """key/value [T, Hkv, D] on the device; slots: host or device int64 [T]."""
        if not isinstance(slots, torch.Tensor):
            slots = torch.from_numpy(np.ascontiguousarray(slots, dtype=np.int64)).to(self.device)
        pa_reshape_and_cache(key, value, self.k_cache, self.v_cache, slots, self.dev_error, stream)

    def apply_ops(self, ops, tokens, stream=None):
        """Execute an op script: ('alloc', seq, n, pos0, write) / ('fork', p, c) / ('free', s).
        tokens(seq, pos0, n) -> (key, value) device tensors for the written rows.
        Returns the per-op (slots, cow_pairs) records (None for fork/free)."""
        records = []
        for op in ops:
            if op[0] == "alloc":
                _, seq, n, pos0, write = op
                slots, cow = self.alloc(seq, n, stream)
                records.append((slots, cow))
                if write and n > 0:
                    k, v = tokens(seq, pos0, n)
                    self.write(k, v, slots, stream)
            elif op[0] == "fork":
                self.fork(op[1], op[2])
                records.append(None)
            else:
                self.free(op[1])
                records.append(None)
        return records

    def block_tables(self, seq_ids, max_blocks):
        table, ctx = self.pool.pa_block_table(seq_ids, max_blocks)
        return (torch.from_numpy(table).to(self.device), torch.from_numpy(ctx).to(self.device))

    def decode(self, q, block_tables, context_lens, scale, out=None, path=PA_PATH_AUTO,
               num_workers=0, flags=0, stream=None):
        if out is None:
            out = torch.empty_like(q)
        pa_decode_attention(out, q, self.k_cache, self.v_cache, block_tables, context_lens, scale,
                            self.workspace, self.dev_error, path, num_workers, flags, stream)
        return out

    def prefill(self, q, block_tables, context_lens, query_start, max_q, scale, out=None,
                path=0, stream=None):
        """Causal attention of each sequence's new tokens (already written) over the cache."""
        if out is None:
            out = torch.empty_like(q)
        pa_prefill_attention(out, q, self.k_cache, self.v_cache, block_tables, context_lens,
                             query_start, max_q, scale, self.dev_error, path, self.prefill_ws,
                             stream)
        return out

    def device_errors(self, stream=None):
        return pa_check_device_error(self.dev_error, stream)


class PagedKVCacheInt8(PagedKVCache):
    """The same pool and call order over an INT8 cache: a key pool and a value pool of
    records [NB, Hkv, bs/16, 2112] (codes + per-token fp32 scales, layout in
    include/pa.h).  key / value / q stay in `dtype`; head_dim 128, block_size a
    multiple of 16."""

    def __init__(self, num_blocks, block_size, num_kv_heads, head_dim, dtype, num_q_heads,
                 max_batch, device="cuda", fill_bits=None):
        if head_dim != 128 or block_size % 16:
            raise ValueError("an INT8 cache needs head_dim 128 and block_size a multiple of 16")
        self.pool = Pool(num_blocks, block_size)
        self.num_blocks, self.block_size = num_blocks, block_size
        self.num_kv_heads, self.head_dim = num_kv_heads, head_dim
        self.num_q_heads, self.dtype, self.device = num_q_heads, dtype, torch.device(device)
        shape = (num_blocks, num_kv_heads, block_size // 16, INT8_RECORD_BYTES)
        self.k_pool = torch.empty(shape, dtype=torch.uint8, device=self.device)
        self.v_pool = torch.empty(shape, dtype=torch.uint8, device=self.device)
        if fill_bits is not None:  # poison unwritten slots: codes with a pattern, scales NaN
            for p in (self.k_pool, self.v_pool):
                p[..., :2048].fill_(fill_bits & 0xFF)
                p[..., 2048:].view(torch.float32).fill_(float("nan"))
        self.dev_error = torch.zeros(1, dtype=torch.int32, device=self.device)
        ws = pa_decode_workspace_size(max_batch, num_q_heads, num_kv_heads, head_dim)
        self.workspace = torch.zeros(ws, dtype=torch.uint8, device=self.device)

    def _copy_pairs(self, pairs, stream=None):
        pa_copy_blocks([self.k_pool], [self.v_pool], pairs, self.dev_error, stream)

    def write(self, key, value, slots, stream=None):
        if not isinstance(slots, torch.Tensor):
            slots = torch.from_numpy(np.ascontiguousarray(slots, dtype=np.int64)).to(self.device)
        pa_reshape_and_cache_int8(key, value, self.k_pool, self.v_pool, slots, self.dev_error,
                                  stream)

    def decode(self, q, block_tables, context_lens, scale, out=None, num_workers=0, flags=0,
               stream=None, **_):
        if out is None:
            out = torch.empty_like(q)
        pa_decode_attention_int8(out, q, self.k_pool, self.v_pool, block_tables, context_lens,
                                 scale, self.workspace, self.dev_error, num_workers, flags,
                                 stream)
        return out
