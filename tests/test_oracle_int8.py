"""Pins the oracle's INT8 KV cache: the quantisation rule's closed-form cases and
error bound, the cache layout, and attention over the
dequantised rows against torch's fp64 scaled-dot-product attention."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads
from oracle_side import raw


def test_exact_multiples_of_a_power_of_two_quantise_exactly():
    k = np.array([127, -64, 0, 1, -127, 5, 33, -2], np.float32)
    x = (k * np.float32(2.0 ** -5)).reshape(1, -1)
    codes, scales = oracle.quantize_rows(x, "f32")
    assert scales[0] == np.float32(2.0 ** -5)
    assert list(codes[0]) == list(k.astype(np.int8))


def test_zero_row_and_extremes():
    codes, scales = oracle.quantize_rows(np.zeros((1, 16), np.float32), "f32")
    assert scales[0] == 0 and not codes.any()
    rng = np.random.default_rng(0)
    x = rng.standard_normal((200, 128)).astype(np.float32)
    codes, scales = oracle.quantize_rows(x, "f32")
    assert codes.min() >= -127 and codes.max() <= 127
    i = np.abs(x).argmax(1)
    assert np.all(np.abs(codes[np.arange(200), i]) == 127)  # the largest entry maps to 127
    assert np.array_equal(codes[np.arange(200), i], 127 * np.sign(x[np.arange(200), i]))


def test_rounding_error_bound_sign_symmetry_and_order():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((300, 64)) * rng.uniform(0.01, 100, (300, 1))).astype(np.float32)
    codes, scales = oracle.quantize_rows(x, "f32")
    err = np.abs(x.astype(np.float64) - codes * scales[:, None].astype(np.float64))
    assert np.all(err <= scales[:, None] * (0.5 + 1e-5))
    neg, _ = oracle.quantize_rows(-x, "f32")
    assert np.array_equal(neg, -codes)
    order = np.argsort(x, 1)
    assert np.all(np.diff(np.take_along_axis(codes.astype(int), order, 1), axis=1) >= 0)


def test_fp16_and_bf16_inputs_quantise_like_their_fp32_values():
    rng = np.random.default_rng(2)
    for dt, td in (("f16", torch.float16), ("bf16", torch.bfloat16)):
        t = torch.from_numpy(rng.standard_normal((50, 128)).astype(np.float32)).to(td)
        c1, s1 = oracle.quantize_rows(raw(t), dt)
        c2, s2 = oracle.quantize_rows(t.float().numpy(), "f32")
        assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def _int8_run(wl):
    """The workload's op script through the oracle pool, cache writes quantised."""
    pool = oracle.Pool(wl.num_blocks, wl.bs)
    cache = oracle.Int8Cache(wl.num_blocks, wl.Hkv, wl.bs, wl.D)
    for op in wl.ops:
        if op[0] == "alloc":
            _, seq, n, pos0, write = op
            st, slots, cow = pool.alloc(seq, n)
            assert st == oracle.OK and len(cow) == 0
            if write and n:
                k = raw(wl.tokens(seq, pos0, n, 0))
                v = raw(wl.tokens(seq, pos0, n, 1))
                assert oracle.reshape_and_cache_int8(k, v, cache, slots, wl.dtype) == oracle.OK
        elif op[0] == "fork":
            pool.fork(op[1], op[2])
        else:
            pool.free(op[1])
    st, table, ctx = pool.block_table(wl.batch, wl.max_blocks)
    return pool, cache, table, ctx


def test_cache_layout_and_attention_against_library():
    wl = workloads.custom("i8", "f16", B=4, Hq=8, Hkv=2, D=64, bs=16, ctx=[1, 17, 40, 70], seed=3)
    pool, cache, table, ctx = _int8_run(wl)
    out = oracle.paged_decode_attention_int8(raw(wl.q()), cache, table, ctx, wl.scale, "f16")
    q = wl.q().double()
    for b, seq in enumerate(wl.batch):
        n = int(ctx[b])
        k = raw(wl.contiguous_kv(int(seq), 0)).reshape(n * wl.Hkv, wl.D)
        v = raw(wl.contiguous_kv(int(seq), 1)).reshape(n * wl.Hkv, wl.D)
        kc, ks = oracle.quantize_rows(k, "f16")
        vc, vs = oracle.quantize_rows(v, "f16")
        # layout: token j of head g sits at row (blk, g, off) of both code arrays
        for j in range(n):
            blk, off = table[b, j // wl.bs], j % wl.bs
            for g in range(wl.Hkv):
                assert np.array_equal(cache.k[blk, g, off], kc[j * wl.Hkv + g])
                assert np.array_equal(cache.v[blk, g, off], vc[j * wl.Hkv + g])
                assert cache.ks[blk, g, off] == ks[j * wl.Hkv + g]
        kd = torch.from_numpy((kc * ks[:, None].astype(np.float64)).reshape(n, wl.Hkv, wl.D))
        vd = torch.from_numpy((vc * vs[:, None].astype(np.float64)).reshape(n, wl.Hkv, wl.D))
        kd = kd.permute(1, 0, 2).repeat_interleave(wl.G, 0)
        vd = vd.permute(1, 0, 2).repeat_interleave(wl.G, 0)
        ref = F.scaled_dot_product_attention(q[b][:, None, :], kd, vd, scale=wl.scale)[:, 0, :]
        np.testing.assert_allclose(out[b], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_int8_attention_stays_close_to_full_precision():
    """Not a parity bound: the quantised cache changes outputs by about 1% of their
    scale (the pages' claim for INT8 is a small quality loss)."""
    wl = workloads.custom("i8b", "bf16", B=3, Hq=8, Hkv=2, D=128, bs=16, ctx=[50, 300, 900],
                          seed=4)
    pool, cache, table, ctx = _int8_run(wl)
    out = oracle.paged_decode_attention_int8(raw(wl.q()), cache, table, ctx, wl.scale, "bf16")
    full = np.stack([oracle.contiguous_attention(raw(wl.q()[b]),
                                                 raw(wl.contiguous_kv(int(s), 0)),
                                                 raw(wl.contiguous_kv(int(s), 1)), wl.scale,
                                                 "bf16") for b, s in enumerate(wl.batch)])
    rel = np.abs(out - full).max() / np.abs(full).max()
    assert rel < 0.05
