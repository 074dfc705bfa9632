"""Pins the oracle's cache write, block copy and attention: exact special cases,
invariances, and agreement with torch's scaled-dot-product attention (fp64, CPU)
on the logical key/value rows, which the test takes from the generator directly
(never through a block table)."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads
from oracle_side import attention, raw, run_script


def _sdpa_reference(wl):
    """Library attention on each sequence's logical rows, fp64."""
    q = wl.q().double()
    out = np.zeros((wl.B, wl.Hq, wl.D))
    for b, seq in enumerate(wl.batch):
        k = wl.contiguous_kv(int(seq), 0).double()  # [n, Hkv, D]
        v = wl.contiguous_kv(int(seq), 1).double()
        k = k.permute(1, 0, 2).repeat_interleave(wl.G, dim=0)  # [Hq, n, D]
        v = v.permute(1, 0, 2).repeat_interleave(wl.G, dim=0)
        o = F.scaled_dot_product_attention(q[b][:, None, :], k, v, scale=wl.scale)
        out[b] = o[:, 0, :].numpy()
    return out


@pytest.mark.parametrize("make", [
    workloads.tiny,
    lambda: workloads.custom("c16", "f16", B=5, Hq=8, Hkv=2, D=128, bs=16,
                             ctx=[1, 16, 17, 100, 333], seed=3),
    lambda: workloads.custom("cbf", "bf16", B=4, Hq=8, Hkv=8, D=64, bs=32,
                             ctx=[2, 31, 64, 129], seed=4),
    lambda: workloads.custom("mqa", "f16", B=3, Hq=6, Hkv=1, D=64, bs=8,
                             ctx=[9, 40, 77], seed=5),
])
def test_paged_oracle_matches_library_attention(make):
    wl = make()
    st = run_script(wl)
    got = attention(wl, st)
    ref = _sdpa_reference(wl)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_paged_equals_contiguous_bitwise():
    wl = workloads.custom("pc", "f16", B=3, Hq=4, Hkv=2, D=64, bs=16, ctx=[5, 48, 70], seed=9)
    st = run_script(wl)
    paged = attention(wl, st)
    for b in range(wl.B):
        q = raw(wl.q()[b])
        k = raw(wl.contiguous_kv(int(wl.batch[b]), 0))
        v = raw(wl.contiguous_kv(int(wl.batch[b]), 1))
        assert np.array_equal(oracle.contiguous_attention(q, k, v, wl.scale, "f16"), paged[b])


def _one_seq_case(n, D=64, Hq=2, Hkv=1, k_rows=None, v_rows=None, q=None, bs=16, seed=0):
    rng = np.random.default_rng(seed)
    nblk = (n + bs - 1) // bs
    nb = nblk + 3
    perm = rng.permutation(nb)[:nblk].astype(np.int32)
    kc = np.zeros((nb, Hkv, bs, D), dtype=np.float32)
    vc = np.zeros((nb, Hkv, bs, D), dtype=np.float32)
    k_rows = rng.standard_normal((n, Hkv, D)).astype(np.float32) if k_rows is None else k_rows
    v_rows = rng.standard_normal((n, Hkv, D)).astype(np.float32) if v_rows is None else v_rows
    slots = perm[np.arange(n) // bs].astype(np.int64) * bs + np.arange(n) % bs
    oracle.reshape_and_cache(k_rows, v_rows, kc, vc, slots, bs, 4)
    q = rng.standard_normal((1, Hq, D)).astype(np.float32) if q is None else q
    table = np.full((1, nblk + 1), -1, dtype=np.int32)
    table[0, :nblk] = perm
    out = oracle.paged_decode_attention(q, kc, vc, table, np.array([n], np.int32),
                                        1 / np.sqrt(D), "f32")
    return out[0], k_rows, v_rows


def test_one_key_returns_its_value_exactly():
    out, _, v = _one_seq_case(1, Hq=3, Hkv=1)
    for h in range(3):
        assert np.array_equal(out[h], v[0, 0].astype(np.float64))


def test_equal_keys_and_zero_query_give_the_mean_of_values():
    n, D = 37, 64
    rng = np.random.default_rng(2)
    k = np.repeat(rng.standard_normal((1, 1, D)).astype(np.float32), n, axis=0)
    out, _, v = _one_seq_case(n, D=D, Hq=1, Hkv=1, k_rows=k)
    np.testing.assert_allclose(out[0], v[:, 0].astype(np.float64).mean(0), rtol=0, atol=1e-14)
    out, _, v = _one_seq_case(n, D=D, Hq=1, Hkv=1, q=np.zeros((1, 1, D), np.float32), seed=3)
    np.testing.assert_allclose(out[0], v[:, 0].astype(np.float64).mean(0), rtol=0, atol=1e-14)


def test_constant_values_are_returned():
    n, D = 50, 64
    row = np.random.default_rng(4).standard_normal(D).astype(np.float32)
    v = np.tile(row, (n, 1, 1))
    out, _, _ = _one_seq_case(n, D=D, Hq=2, Hkv=1, v_rows=v, seed=5)
    for h in range(2):
        np.testing.assert_allclose(out[h], row.astype(np.float64), rtol=1e-14, atol=1e-15)


def test_one_dominant_key_selects_its_value():
    n, D = 20, 64
    rng = np.random.default_rng(6)
    k = rng.standard_normal((n, 1, D)).astype(np.float32)
    q = np.zeros((1, 1, D), np.float32)
    q[0, 0, 0] = 1.0
    k[:, 0, 0] = 0.0
    k[13, 0, 0] = 2000.0  # score 2000/8 above the rest: every other weight underflows
    out, _, v = _one_seq_case(n, D=D, Hq=1, Hkv=1, k_rows=k, q=q, seed=6)
    assert np.array_equal(out[0], v[13, 0].astype(np.float64))


def test_physical_placement_does_not_matter():
    wl = workloads.custom("perm", "f16", B=3, Hq=4, Hkv=2, D=64, bs=16, ctx=[30, 64, 81],
                          seed=11)
    st = run_script(wl)
    base = attention(wl, st)
    rng = np.random.default_rng(12)
    perm = rng.permutation(wl.num_blocks)  # physical block b moves to perm[b]
    kc = np.empty_like(st["k_cache"])
    vc = np.empty_like(st["v_cache"])
    kc[perm] = st["k_cache"]
    vc[perm] = st["v_cache"]
    table = np.where(st["table"] >= 0, perm[np.maximum(st["table"], 0)], -1).astype(np.int32)
    moved = oracle.paged_decode_attention(raw(wl.q()), kc, vc, table, st["ctx"], wl.scale, "f16")
    assert np.array_equal(moved, base)


def test_block_size_does_not_matter():
    outs = []
    for bs in (8, 16, 32):
        wl = workloads.custom("bsz", "bf16", B=3, Hq=4, Hkv=2, D=64, bs=bs, ctx=[7, 40, 99],
                              seed=13)
        outs.append(attention(wl, run_script(wl)))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[1], outs[2])


def test_shared_prefix_equals_duplicated_prefix():
    shared = workloads.shared_prefix(n_groups=3, n_samples=4, prefix_len=64)
    st = run_script(shared)
    got = attention(shared, st)
    # the same logical rows with no sharing at all: each sequence's own copy
    for b in range(shared.B):
        q = raw(shared.q()[b])
        k = raw(shared.contiguous_kv(int(shared.batch[b]), 0))
        v = raw(shared.contiguous_kv(int(shared.batch[b]), 1))
        assert np.array_equal(oracle.contiguous_attention(q, k, v, shared.scale, "f16"), got[b])
    # and the sharing really happened: copies were made for partially filled blocks
    ncopies = sum(len(r[1]) for r in st["records"][shared.n_prefill_ops:] if r)
    groups = [int(s) for s in shared.batch[::4]]
    expected = sum(3 for s in groups if (shared.lengths[s] - 1) % shared.bs != 0)
    assert ncopies == expected and expected > 0


def test_cache_write_round_trip_and_skip():
    rng = np.random.default_rng(21)
    nb, Hkv, bs, D = 6, 2, 4, 8
    kc = np.zeros((nb, Hkv, bs, D), np.uint16)
    vc = np.zeros((nb, Hkv, bs, D), np.uint16)
    k = rng.integers(0, 65535, (5, Hkv, D)).astype(np.uint16)
    v = rng.integers(0, 65535, (5, Hkv, D)).astype(np.uint16)
    slots = np.array([7, -1, 0, 23, 12], np.int64)
    oracle.reshape_and_cache(k, v, kc, vc, slots, bs, 2)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        assert np.array_equal(kc[s // bs, :, s % bs], k[t])
        assert np.array_equal(vc[s // bs, :, s % bs], v[t])
    written = {int(s) for s in slots if s >= 0}
    for s in range(nb * bs):
        if s not in written:
            assert not kc[s // bs, :, s % bs].any() and not vc[s // bs, :, s % bs].any()


def test_copy_blocks_in_order():
    rng = np.random.default_rng(22)
    layers = [rng.integers(0, 60000, (5, 2, 4, 8)).astype(np.uint16) for _ in range(3)]
    vals = [rng.integers(0, 60000, (5, 2, 4, 8)).astype(np.uint16) for _ in range(3)]
    before_k = [x.copy() for x in layers]
    oracle.copy_blocks(layers, vals, np.array([[1, 3], [3, 4]]))
    for L in range(3):
        assert np.array_equal(layers[L][3], before_k[L][1])
        assert np.array_equal(layers[L][4], before_k[L][1])  # second pair sees the first
        assert np.array_equal(layers[L][0], before_k[L][0])


def test_empty_context_gives_zeros():
    wl = workloads.custom("z", "f16", B=2, Hq=2, Hkv=1, D=64, bs=16, ctx=[3, 5], seed=1)
    st = run_script(wl)
    ctx = st["ctx"].copy()
    ctx[0] = 0
    out = oracle.paged_decode_attention(raw(wl.q()), st["k_cache"], st["v_cache"], st["table"],
                                        ctx, wl.scale, "f16")
    assert not out[0].any()
