"""Swapping sequences between the device cache and a pinned host cache: the
copied bytes match the oracle's copy semantics exactly, and decode after a
round trip through host memory gives the same bits as before."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import paged_kv_cache_486_b200 as pa
from gpu_side import bits, build
from oracle_side import raw

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("make", [
    lambda: workloads.custom("sw16", "f16", B=6, Hq=32, Hkv=8, D=128, bs=16,
                             ctx=[1, 17, 300, 900, 2000, 64], seed=51),
    lambda: workloads.custom("swbf", "bf16", B=4, Hq=16, Hkv=2, D=64, bs=32,
                             ctx=[5, 64, 700, 33], seed=52),
])
def test_swap_round_trip(cuda_ok, make):
    wl = make()
    g = build(wl)
    eng, ref_out = g["eng"], g["out"].clone()
    nh = sum((int(c) + wl.bs - 1) // wl.bs for c in g["ctx"].cpu()) + 3
    hk = torch.zeros((nh,) + tuple(eng.k_cache.shape[1:]), dtype=eng.k_cache.dtype).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    host = pa.Pool(nh, wl.bs)
    seqs = [int(s) for s in wl.batch]
    for s in seqs[::2]:  # every other sequence goes to host memory
        pairs = pa.pa_swap(eng.pool, host, s)
        # the oracle's copy semantics, applied to copies of both pools taken before the copy
        ok_, ov_ = raw(hk).copy(), raw(hv).copy()
        oracle.copy_between([ok_], [ov_], [raw(eng.k_cache)], [raw(eng.v_cache)], pairs)
        pa.pa_swap_blocks([hk], [hv], [eng.k_cache], [eng.v_cache],
                          torch.from_numpy(pairs).cuda(), eng.dev_error)
        torch.cuda.synchronize()
        assert np.array_equal(raw(hk), ok_) and np.array_equal(raw(hv), ov_)
    # scribble over the freed device blocks, then bring the sequences back
    eng.k_cache.view(torch.int16).fill_(0x7E00)
    for s in seqs[::2]:
        pairs = pa.pa_swap(host, eng.pool, s)
        pa.pa_swap_blocks([eng.k_cache], [eng.v_cache], [hk], [hv],
                          torch.from_numpy(pairs).pin_memory(), eng.dev_error)
    torch.cuda.synchronize()
    # (the sequences that stayed on the device lost their keys to the scribble;
    # only the rows of the swapped sequences are compared)
    bt, ctx = eng.block_tables(wl.batch, wl.max_blocks)
    rows = list(range(0, wl.B, 2))
    out = eng.decode(g["q"], bt, ctx, wl.scale)
    torch.cuda.synchronize()
    for b in rows:
        assert torch.equal(bits(out[b]), bits(ref_out[b])), b
    assert eng.device_errors() == 0
