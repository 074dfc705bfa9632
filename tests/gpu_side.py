"""Runs a workload through the CUDA library (test infrastructure)."""
import numpy as np
import torch

import workloads
from paged_kv_cache_486_b200.engine import PagedKVCache

NAN_BITS = {"f32": 0x7FC00000, "f16": 0x7E00, "bf16": 0x7FC0}


def tol_ok(got, ref, dtype):
    """Spec bar for fp16/bf16: |got - ref| <= 2e-3 + 1e-2 |ref|; fp32: 1e-5 + 1e-4 |ref|."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    atol, rtol = (1e-5, 1e-4) if dtype == "f32" else (2e-3, 1e-2)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    ok = bool(np.all(err <= bound)) and bool(np.all(np.isfinite(got)))
    worst = float(np.max(err / bound)) if err.size else 0.0
    return ok, worst


def _tokens_fn(wl, gen):
    """tokens(seq, pos0, n) -> device (key, value) rows.  gen='cuda' draws them on the
    device; gen='cpu' draws them on the host and copies them over (no generator
    kernels on the device: used where the device's launch list should hold the
    library's kernels only)."""
    def tokens(seq, pos0, n):
        k, v = wl.tokens(seq, pos0, n, 0, gen), wl.tokens(seq, pos0, n, 1, gen)
        return k.to("cuda"), v.to("cuda")
    return tokens


def build(wl, poison=True, batched_step=True, path=0, workers=0, stream=None, gen="cuda"):
    """Prefill the pools from the op script, then run the decode step: one new
    token per sequence (one batched cache write), then decode attention."""
    dt = workloads.TORCH_DTYPE[wl.dtype]
    eng = PagedKVCache(wl.num_blocks, wl.bs, wl.Hkv, wl.D, dt, wl.Hq, wl.B, "cuda",
                       fill_bits=NAN_BITS[wl.dtype] if poison else None)
    tokens = _tokens_fn(wl, gen)

    pre = eng.apply_ops(wl.ops[:wl.n_prefill_ops], tokens, stream)
    step_ops = wl.ops[wl.n_prefill_ops:]
    if batched_step:
        slots, keys, vals, step = [], [], [], []
        for op in step_ops:
            _, seq, n, pos0, _w = op
            s, cow = eng.alloc(seq, n, stream)
            step.append((s, cow))
            slots.append(s)
            k, v = tokens(seq, pos0, n)
            keys.append(k)
            vals.append(v)
        eng.write(torch.cat(keys), torch.cat(vals), np.concatenate(slots), stream)
    else:
        step = eng.apply_ops(step_ops, tokens, stream)
    bt, ctx = eng.block_tables(wl.batch, wl.max_blocks)
    q = wl.q(gen).to("cuda")
    out = eng.decode(q, bt, ctx, wl.scale, path=path, num_workers=workers, stream=stream)
    torch.cuda.synchronize()
    return dict(eng=eng, records=pre + step, bt=bt, ctx=ctx, q=q, out=out)


def gathered(eng, bt, ctx, b, kind, heads=None):
    """Cache rows of batch row b in logical order, read back through its table (torch indexing)."""
    cache = eng.k_cache if kind == 0 else eng.v_cache
    n = int(ctx[b])
    bs = cache.shape[2]
    pos = torch.arange(n, device=cache.device)
    blocks = bt[b].long()[pos // bs]
    rows = cache[blocks, :, pos % bs, :]  # [n, Hkv, D]
    return rows if heads is None else rows[:, heads, :]


def bits(t):
    t = t.contiguous()
    return t.view(torch.int32) if t.dtype == torch.float32 else t.view(torch.int16)


def build_int8(wl, poison=True, workers=0, stream=None, gen="cuda"):
    """As build(), over an INT8 cache (PagedKVCacheInt8)."""
    from paged_kv_cache_486_b200.engine import PagedKVCacheInt8
    dt = workloads.TORCH_DTYPE[wl.dtype]
    eng = PagedKVCacheInt8(wl.num_blocks, wl.bs, wl.Hkv, wl.D, dt, wl.Hq, wl.B, "cuda",
                           fill_bits=0x5A if poison else None)
    eng.apply_ops(wl.ops, _tokens_fn(wl, gen), stream)
    bt, ctx = eng.block_tables(wl.batch, wl.max_blocks)
    q = wl.q(gen).to("cuda")
    out = eng.decode(q, bt, ctx, wl.scale, num_workers=workers, stream=stream)
    torch.cuda.synchronize()
    return dict(eng=eng, bt=bt, ctx=ctx, q=q, out=out)


def _key_record_offsets():
    """[16, 128] byte offsets of code d of group token t in a key record (the layout
    stated in include/pa.h, written out here from that statement)."""
    off = np.zeros((16, 128), np.int64)
    for t in range(16):
        i, h, e = t >> 2, (t >> 1) & 1, t & 1
        line = 2 * i + e + 8 * h
        for d in range(128):
            off[t, d] = line * 128 + 16 * ((d // 16) ^ (line % 8)) + d % 16
    return torch.from_numpy(off)


_KEY_OFF = _key_record_offsets()


def gathered_int8(eng, bt, ctx, b, kvh):
    """(k codes [n, 128], v codes [n, 128], k scales [n], v scales [n]) of batch row b and
    kv head kvh in logical order, decoded from the INT8 records through its table."""
    n = int(ctx[b])
    bs = eng.block_size
    dev = eng.k_pool.device
    pos = torch.arange(n, device=dev)
    blk = bt[b].long()[pos // bs]
    grp = (pos % bs) // 16
    t = pos % 16
    krec = eng.k_pool[:, kvh][blk, grp]           # [n, 2112] uint8
    vrec = eng.v_pool[:, kvh][blk, grp]
    # codes are stored offset-binary (code + 128)
    kc = (torch.gather(krec, 1, _KEY_OFF.to(dev)[t]) ^ 0x80).view(torch.int8)
    d = torch.arange(128, device=dev)
    vc = (torch.gather(vrec, 1, d[None, :] * 16 + t[:, None]) ^ 0x80).view(torch.int8)
    ks = krec[:, 2048:].contiguous().view(torch.float32).gather(1, t[:, None])[:, 0]
    vs = vrec[:, 2048:].contiguous().view(torch.float32).gather(1, t[:, None])[:, 0]
    return kc, vc, ks, vs
