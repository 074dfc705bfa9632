"""Prefix caching end to end on the GPU: requests that share system prompts are
admitted through pa_alloc_tokens, only the tokens the cache does not supply are
written, and decode over the resulting (shared) blocks matches the oracle's
attention over each request's own logical rows.  Tables, slots and cached-token
counts are bit-exact against the oracle's pool."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_side import NAN_BITS, tol_ok
from oracle_side import raw
from paged_kv_cache_486_b200.engine import PagedKVCache

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


def _admit(ps, free_every, slack):
    """Admit every request in order on the GPU engine and on the oracle pool,
    freeing every `free_every`-th request after the next one is admitted (so
    cached blocks are released, found again and evicted)."""
    dt = workloads.TORCH_DTYPE[ps.dtype]
    eng = PagedKVCache(ps.num_blocks + slack, ps.bs, ps.Hkv, ps.D, dt, ps.Hq, ps.B, "cuda",
                       fill_bits=NAN_BITS[ps.dtype])
    eng.pool.pa_set_prefix_caching(True)
    orc = oracle.Pool(ps.num_blocks + slack, ps.bs)
    orc.set_prefix_caching(True)
    live, freed, cached = [], [], 0
    for i, ids in enumerate(ps.prompts):
        slots, cow, n_cached = eng.alloc_tokens(i, ids)
        st, slots_o, cow_o, n_cached_o = orc.alloc_tokens(i, ids)
        assert st == oracle.OK
        assert np.array_equal(slots, slots_o) and np.array_equal(cow, cow_o)
        assert n_cached == n_cached_o
        cached += n_cached
        eng.write(ps.rows(i, 0, "cuda"), ps.rows(i, 1, "cuda"), slots)
        live.append(i)
        if free_every and i % free_every == free_every - 1 and len(live) > 1:
            victim = live.pop(-2)
            eng.free(victim)
            assert orc.free(victim) == oracle.OK
            freed.append(victim)
    torch.cuda.synchronize()
    return eng, orc, live, cached


@pytest.mark.parametrize("dtype,bs,free_every,slack", [("f16", 16, 0, 0), ("bf16", 32, 3, 8),
                                                       ("f16", 16, 2, 4)])
def test_prefix_cached_prompts_decode_like_the_oracle(dtype, bs, free_every, slack):
    ps = workloads.prompt_set("pc", dtype, n_systems=3, system_lens=(100, 257, 64),
                              n_requests=24, user_len=(1, 300), vocab=50, bs=bs,
                              seed=77 + bs + free_every)
    eng, orc, live, cached = _admit(ps, free_every, slack)
    assert cached > 0
    bt, ctx = eng.block_tables(live, max(len(p) for p in ps.prompts) // ps.bs + 1)
    st, bt_o, ctx_o = orc.block_table(live, bt.shape[1])
    assert np.array_equal(bt.cpu().numpy(), bt_o) and np.array_equal(ctx.cpu().numpy(), ctx_o)
    q = ps.q("cuda")[live].contiguous()
    out = eng.decode(q, bt, ctx, ps.scale)
    torch.cuda.synchronize()
    got = out.double().cpu().numpy()
    for r, i in enumerate(live):
        ref = oracle.contiguous_attention(raw(ps.q()[i]), raw(ps.rows(i, 0)), raw(ps.rows(i, 1)),
                                          ps.scale, ps.dtype)
        ok, worst = tol_ok(got[r], ref, ps.dtype)
        assert ok, f"request {i}: worst error / bound = {worst:.3f}"
    assert eng.device_errors() == 0


def test_shared_blocks_are_written_once():
    """Requests behind one system prompt hold the same physical blocks for it, and
    the bytes there are those the first request wrote (no later write touched them)."""
    ps = workloads.prompt_set("pc1", "f16", n_systems=1, system_lens=(160,), n_requests=6,
                              user_len=(5, 40), vocab=50, seed=5)
    eng, orc, live, cached = _admit(ps, 0, 0)
    assert cached == 5 * 160  # every later request reuses the 10 full system blocks
    bt, _ = eng.block_tables(live, 16)
    bt = bt.cpu().numpy()
    assert (bt[1:, :10] == bt[0, :10]).all()
    first = ps.rows(0, 0, "cuda")[:160]
    blocks = torch.from_numpy(bt[0, :10]).long().cuda()
    cachek = eng.k_cache[blocks].permute(0, 2, 1, 3).reshape(160, ps.Hkv, ps.D)
    assert torch.equal(cachek.view(torch.int16), first.view(torch.int16))
