"""Parity on inputs whose scores span tens of base-2 units, with the largest ones
late in each context (the wide-range option of workloads.py: queries times a
power of two, keys doubled every few hundred positions).

The decode kernels keep a lazily updated running maximum and rescale their sums
only when a score passes it by more than 2^8; split contexts are merged from
pieces whose maxima here differ by tens of units; the prefill kernels rescale O
the same way.  With N(0, 1) inputs those branches hardly ever run after the
first tiles.  Here they run many times, and every output row is compared with
the oracle elementwise at the stated bound: 2e-3 + 1e-2 |o| for fp16 / bf16,
1e-5 + 1e-4 |o| for fp32 ("KV Cache for intermediates..." / "The precise
scientific definition": the new token attends to every cached key and value)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import paged_kv_cache_486_b200 as pa
from oracle_side import raw

LOG2E = 1.4426950408889634


def _spread(name, dtype, Hq, Hkv, D, bs, ctx, seed, q_mul, ramp, ramp_max):
    return workloads.spread(workloads.custom(name, dtype, B=len(ctx), Hq=Hq, Hkv=Hkv, D=D, bs=bs,
                                             ctx=ctx, seed=seed), q_mul, ramp, ramp_max)


DECODE = {
    "f16_g4_long": lambda: _spread("sa", "f16", 32, 8, 128, 16, [1, 300, 1000, 6000], 51,
                                   2, 512, 4),
    "bf16_g8": lambda: _spread("sb", "bf16", 64, 8, 128, 16, [2, 129, 700, 1500, 4000], 52,
                               2, 256, 4),
    "f16_g1_bs32": lambda: _spread("sc", "f16", 8, 8, 128, 32, [33, 900, 3000], 53, 4, 256, 3),
    "bf16_g2_d64": lambda: _spread("sd", "bf16", 4, 2, 64, 16, [48, 517, 2500], 54, 2, 128, 5),
    "f32_g4": lambda: _spread("se", "f32", 8, 2, 128, 16, [77, 2000], 55, 2, 256, 4),
    "f16_g16": lambda: _spread("sf", "f16", 32, 2, 128, 16, [90, 3000], 56, 2, 256, 4),
    "bf16_bs8": lambda: _spread("sg", "bf16", 8, 2, 64, 8, [9, 2000], 57, 2, 256, 4),
}

INT8 = {
    "f16_g4_long": DECODE["f16_g4_long"],
    "bf16_g8": DECODE["bf16_g8"],
    "f16_g1_bs32": DECODE["f16_g1_bs32"],
    "bf16_mqa_bs64": lambda: _spread("sh", "bf16", 4, 1, 128, 64, [5, 250, 2999], 58,
                                     2, 256, 4),
}

PREFILL = {
    "f16_g4": lambda: _prefill("pa", "f16", 32, 8, 128, 16, [300, 1500, 2100], [300, 700, 90],
                               61, 2, 256, 3),
    "bf16_g8": lambda: _prefill("pb", "bf16", 64, 8, 128, 16, [40, 1200, 2500], [40, 513, 300],
                                62, 2, 256, 4),
    "f16_g1_bs32": lambda: _prefill("pc", "f16", 8, 8, 128, 32, [97, 1600], [60, 900], 63,
                                    4, 256, 3),
    "bf16_g2_d64": lambda: _prefill("pd", "bf16", 4, 2, 64, 64, [300, 1777], [300, 400], 64,
                                    2, 128, 5),
}


def _prefill(name, dtype, Hq, Hkv, D, bs, ctx, n_new, seed, q_mul, ramp, ramp_max):
    wl = workloads.prefill(name, dtype, Hq, Hkv, D, bs, ctx, n_new, seed)
    return workloads.spread(wl, q_mul, ramp, ramp_max)


def _scores(wl, b, h):
    """Base-2 scores of query head h of batch row b over its logical keys (fp64)."""
    seq = int(wl.batch[b])
    k = wl.contiguous_kv(seq, 0, heads=[h // wl.G]).double()[:, 0, :]
    q = wl.q()[b, h].double()
    return (k @ q).numpy() * wl.scale * LOG2E


# ---------------------------------------------------------------- the inputs
def test_spread_inputs_reach_the_branches_they_are_for():
    """The cases do what they are for: the running maximum of a long context rises
    by more than 2^8 (the kernels' rescale threshold) many times after its first
    tiles, and its last tokens' maximum is at least 40 units above its first 512
    tokens' (a split context's pieces then have far-apart maxima)."""
    for make in (DECODE["f16_g4_long"], DECODE["bf16_g8"], INT8["bf16_mqa_bs64"]):
        wl = make()
        b = int(np.argmax(wl.context_lens()))
        for h in (0, wl.Hq - 1):
            s = _scores(wl, b, h)
            run = np.maximum.accumulate(s)
            ref, rises = run[15], 0           # reference after the first 16-token tile
            for x in run[16:]:
                if x > ref + 8:
                    ref, rises = x, rises + 1
            assert rises >= 3, (wl.name, h, rises)
            assert s[-512:].max() - s[:512].max() >= 40, (wl.name, h)
    # the generator stays exact: key rows of the ramp are power-of-two multiples
    wl = DECODE["f16_g1_bs32"]()
    k = wl.tokens(0, 0, 900, 0)
    base = workloads.custom("sc", "f16", B=3, Hq=8, Hkv=8, D=128, bs=32, ctx=[33, 900, 3000],
                            seed=53).tokens(0, 0, 900, 0)
    f = 2.0 ** np.minimum(np.arange(900) // 256, 3)
    assert torch.equal(k.double(), base.double() * torch.from_numpy(f)[:, None, None])


# ------------------------------------------------------------------- decode
@pytest.mark.gpu
@pytest.mark.parametrize("name", list(DECODE))
@pytest.mark.parametrize("path,workers", [(pa.PA_PATH_AUTO, 0), (pa.PA_PATH_AUTO, 1),
                                          (pa.PA_PATH_AUTO, 5), (pa.PA_PATH_AUTO, 64),
                                          (pa.PA_PATH_SIMT, 0), (pa.PA_PATH_SIMT, 64)])
def test_decode_with_wide_score_ranges_matches_the_oracle(cuda_ok, name, path, workers):
    from gpu_side import build, tol_ok
    from oracle_side import attention, run_script
    wl = DECODE[name]()
    g = build(wl, path=path, workers=workers)
    ref = attention(wl, run_script(wl))
    ok, worst = tol_ok(g["out"].double().cpu().numpy(), ref, wl.dtype)
    assert ok, f"worst error / bound = {worst:.3f}"
    assert g["eng"].device_errors() == 0


# --------------------------------------------------------------------- INT8
@pytest.mark.gpu
@pytest.mark.parametrize("name", list(INT8))
@pytest.mark.parametrize("workers", [0, 1, 5, 64])
def test_int8_decode_with_wide_score_ranges_matches_the_oracle(cuda_ok, name, workers):
    from gpu_side import build_int8, tol_ok
    from oracle_side import run_script_int8
    wl = INT8[name]()
    g = build_int8(wl, workers=workers)
    o = run_script_int8(wl)
    ref = oracle.paged_decode_attention_int8(raw(wl.q()), o["cache"], o["table"], o["ctx"],
                                             wl.scale, wl.dtype)
    ok, worst = tol_ok(g["out"].double().cpu().numpy(), ref, wl.dtype)
    assert ok, f"worst error / bound = {worst:.3f}"
    assert g["eng"].device_errors() == 0


# ------------------------------------------------------------------ prefill
@pytest.mark.gpu
@pytest.mark.parametrize("name", list(PREFILL))
@pytest.mark.parametrize("path", [pa.PA_PREFILL_AUTO, pa.PA_PREFILL_TCGEN05_PAIR,
                                  pa.PA_PREFILL_MMA_SYNC])
@pytest.mark.parametrize("persistent", [False, True])
def test_prefill_with_wide_score_ranges_matches_the_oracle(cuda_ok, name, path, persistent):
    from gpu_side import NAN_BITS, tol_ok
    from oracle_side import run_script
    from paged_kv_cache_486_b200.engine import PagedKVCache
    wl = PREFILL[name]()
    if path == pa.PA_PREFILL_TCGEN05_PAIR and wl.D != 128:
        pytest.skip("the tcgen05 pair kernel takes head_dim 128 only")
    dt = workloads.TORCH_DTYPE[wl.dtype]
    eng = PagedKVCache(wl.num_blocks, wl.bs, wl.Hkv, wl.D, dt, wl.Hq, wl.B, "cuda",
                       fill_bits=NAN_BITS[wl.dtype])
    eng.apply_ops(wl.ops, lambda s, p, n: (wl.tokens(s, p, n, 0, "cuda"),
                                           wl.tokens(s, p, n, 1, "cuda")))
    bt, ctx = eng.block_tables(wl.batch, wl.max_blocks)
    qs = torch.from_numpy(workloads.query_start(wl)).cuda()
    q = workloads.q_prefill(wl, "cuda")
    out = torch.empty_like(q)
    pa.pa_prefill_attention(out, q, eng.k_cache, eng.v_cache, bt, ctx, qs, int(wl.n_new.max()),
                            wl.scale, eng.dev_error, path,
                            eng.prefill_ws if persistent else None)
    torch.cuda.synchronize()
    o = run_script(wl)
    ref = oracle.paged_prefill_attention(raw(q), o["k_cache"], o["v_cache"], o["table"],
                                         o["ctx"], workloads.query_start(wl), wl.scale, wl.dtype)
    ok, worst = tol_ok(out.double().cpu().numpy(), ref, wl.dtype)
    assert ok, f"worst error / bound = {worst:.3f}"
    assert eng.device_errors() == 0
