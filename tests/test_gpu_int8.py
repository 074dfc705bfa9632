"""INT8 KV cache on the GPU against the oracle: codes and scales bit-exact (the
quantisation takes every decision in IEEE fp32 on both sides), attention over
the dequantised cache within the fp16/bf16 bound."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import paged_kv_cache_486_b200 as pa
from gpu_side import build_int8, gathered_int8, tol_ok
from oracle_side import int8_contiguous_row, raw, run_script_int8

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


def _cases():
    C = workloads.custom
    return {
        "f16_g4": lambda: C("i8a", "f16", B=7, Hq=32, Hkv=8, D=128, bs=16,
                            ctx=[1, 15, 16, 17, 33, 300, 1000], seed=21),
        "bf16_g8": lambda: C("i8b", "bf16", B=6, Hq=64, Hkv=8, D=128, bs=16,
                             ctx=[2, 31, 64, 129, 700, 1500], seed=22),
        "f16_g1_bs32": lambda: C("i8c", "f16", B=4, Hq=8, Hkv=8, D=128, bs=32,
                                 ctx=[1, 32, 33, 900], seed=23),
        "bf16_mqa_bs64": lambda: C("i8d", "bf16", B=3, Hq=4, Hkv=1, D=128, bs=64,
                                   ctx=[5, 250, 999], seed=24),
        "f16_g2_bs128": lambda: C("i8e", "f16", B=3, Hq=4, Hkv=2, D=128, bs=128,
                                  ctx=[1, 128, 700], seed=25),
        "shared_prefix": lambda: workloads.shared_prefix(n_groups=5, n_samples=4, prefix_len=80),
    }


CASES = _cases()


def _check_cache(wl, g, o):
    """Every cached row of every sequence: codes and scales equal the oracle's."""
    cache = o["cache"]
    for b in range(wl.B):
        n = int(o["ctx"][b])
        pos = np.arange(n)
        blk = o["table"][b][pos // wl.bs]
        off = pos % wl.bs
        for h in range(wl.Hkv):
            kc, vc, ks, vs = (t.cpu().numpy() for t in gathered_int8(g["eng"], g["bt"],
                                                                     g["ctx"], b, h))
            assert np.array_equal(kc, cache.k[blk, h, off, :])
            assert np.array_equal(vc, cache.v[blk, h, off, :])
            assert np.array_equal(ks.view(np.uint32), cache.ks[blk, h, off].view(np.uint32))
            assert np.array_equal(vs.view(np.uint32), cache.vs[blk, h, off].view(np.uint32))


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("workers", [0, 1, 5, 64])
def test_int8_small_configs_match_the_oracle(name, workers):
    wl = CASES[name]()
    g = build_int8(wl, workers=workers)
    o = run_script_int8(wl)
    assert np.array_equal(g["bt"].cpu().numpy(), o["table"])
    _check_cache(wl, g, o)
    ref = oracle.paged_decode_attention_int8(raw(wl.q()), o["cache"], o["table"], o["ctx"],
                                             wl.scale, wl.dtype)
    ok, worst = tol_ok(g["out"].double().cpu().numpy(), ref, wl.dtype)
    assert ok, f"worst error / bound = {worst:.3f}"
    assert g["eng"].device_errors() == 0


@pytest.mark.parametrize("dtype,bs", [("f32", 16), ("f16", 32), ("bf16", 64), ("f32", 128)])
def test_int8_cache_write_other_dtypes_and_block_sizes(dtype, bs):
    wl = workloads.custom("i8w", dtype, B=4, Hq=4, Hkv=2, D=128, bs=bs, ctx=[1, 17, 40, 300],
                          seed=26)
    from paged_kv_cache_486_b200.engine import PagedKVCacheInt8
    eng = PagedKVCacheInt8(wl.num_blocks, wl.bs, wl.Hkv, wl.D, workloads.TORCH_DTYPE[dtype],
                           wl.Hq, wl.B, "cuda", fill_bits=0x5A)
    eng.apply_ops(wl.ops, lambda s, p, n: (wl.tokens(s, p, n, 0, "cuda"),
                                           wl.tokens(s, p, n, 1, "cuda")))
    bt, ctx = eng.block_tables(wl.batch, wl.max_blocks)
    torch.cuda.synchronize()
    o = run_script_int8(wl)
    _check_cache(wl, dict(eng=eng, bt=bt, ctx=ctx), o)
    assert eng.device_errors() == 0


@pytest.mark.parametrize("name", ["llama3_8b", "llama3_70b"])
def test_int8_full_size_configs(name):
    wl = workloads.make(name)
    g = build_int8(wl)
    eng, bt, ctx, out = g["eng"], g["bt"], g["ctx"], g["out"]
    assert torch.isfinite(out.float()).all()
    rng = np.random.default_rng(4868)
    rows = sorted(set(int(x) for x in rng.choice(wl.B, size=min(wl.B, 5), replace=False))
                  | {int(np.argmax(ctx.cpu().numpy()))})
    for b in rows:
        seq = int(wl.batch[b])
        heads = sorted(set(int(x) for x in rng.choice(wl.Hq, size=3, replace=False)))
        for h in sorted({h // wl.G for h in heads}):
            # codes and scales read back through the table equal the oracle's
            # quantisation of the sequence's logical rows
            got = [t.cpu().numpy() for t in gathered_int8(eng, bt, ctx, b, h)]
            for kind in (0, 1):
                codes, scales = oracle.quantize_rows(
                    raw(wl.contiguous_kv(seq, kind, heads=[h]))[:, 0, :], wl.dtype)
                assert np.array_equal(got[kind], codes)
                assert np.array_equal(got[2 + kind].view(np.uint32), scales.view(np.uint32))
        ref = int8_contiguous_row(wl, b, heads)
        ok, worst = tol_ok(out[b].double().cpu().numpy()[heads], ref[heads], wl.dtype)
        assert ok, f"row {b}: worst error / bound = {worst:.3f}"
    assert eng.device_errors() == 0


@pytest.mark.parametrize("name", ["llama3_8b", "llama3_70b"])
def test_int8_full_size_every_row(name):
    """Every output row of the full-size INT8 decode workloads against the oracle,
    elementwise at the fp16 / bf16 bound.  Values enter the products as biased
    codes whose offset (1152 times the summed weights) is taken out at the end,
    so the longest contexts are where its cancellation in fp32 would show."""
    from oracle_side import int8_all_rows
    wl = workloads.make(name)
    g = build_int8(wl)
    ref = int8_all_rows(wl)
    ok, worst = tol_ok(g["out"].double().cpu().numpy(), ref, wl.dtype)
    assert ok, f"worst error / bound = {worst:.3f}"
    assert g["eng"].device_errors() == 0


def test_int8_value_scales_of_very_different_magnitudes():
    """Token rows scaled by 2^-24 .. 2^12 (fp16 keys and values stay finite):
    the running value-scale normaliser keeps P' in [0, 1], so tiny and huge
    value rows mix without underflow or overflow."""
    wl = workloads.custom("i8m", "f16", B=3, Hq=8, Hkv=2, D=128, bs=16, ctx=[40, 300, 777],
                          seed=27)
    expo = torch.arange(2048, dtype=torch.float64)
    mag = torch.pow(2.0, (expo * 7919 % 37) - 24)  # a fixed spread of 37 binades per position

    class Scaled:
        def __getattr__(self, k):
            return getattr(wl, k)

        def tokens(self, seq, pos0, n, kind, device=None):
            t = wl.tokens(seq, pos0, n, kind)
            if kind == 1:
                t = (t.double() * mag[pos0:pos0 + n, None, None]).to(t.dtype)
            else:
                t = (t.double() * 0.25).to(t.dtype)
            return t if device is None else t.to(device)

    sw = Scaled()
    g = build_int8(sw)
    o = run_script_int8(sw)
    _check_cache(wl, g, o)
    ref = oracle.paged_decode_attention_int8(raw(wl.q()), o["cache"], o["table"], o["ctx"],
                                             wl.scale, wl.dtype)
    got = g["out"].double().cpu().numpy()
    # bound relative to each row's largest output (outputs span many binades)
    scale = np.abs(ref).max(axis=2, keepdims=True)
    err = np.abs(got - ref) / scale
    assert np.all(np.isfinite(got))
    assert err.max() <= 5e-3, err.max()


def test_int8_empty_contexts_and_bad_block_ids():
    wl = workloads.custom("i8z", "bf16", B=4, Hq=16, Hkv=2, D=128, bs=16, ctx=[3, 50, 1, 17],
                          seed=28)
    g = build_int8(wl)
    o = run_script_int8(wl)
    ctx = o["ctx"].copy()
    ctx[[0, 2]] = 0
    eng = g["eng"]
    out = eng.decode(g["q"], g["bt"], torch.from_numpy(ctx).cuda(), wl.scale)
    torch.cuda.synchronize()
    assert not out[0].float().any() and not out[2].float().any()
    ref = oracle.paged_decode_attention_int8(raw(wl.q()), o["cache"], o["table"], ctx,
                                             wl.scale, wl.dtype, rows=[wl.Hq + h for h in
                                                                       range(wl.Hq)]
                                             + [3 * wl.Hq + h for h in range(wl.Hq)])
    ok, worst = tol_ok(out.double().cpu().numpy()[[1, 3]], ref[[1, 3]], wl.dtype)
    assert ok, worst
    allzero = eng.decode(g["q"], g["bt"], torch.zeros_like(g["ctx"]), wl.scale)
    torch.cuda.synchronize()
    assert not allzero.float().any()
    assert eng.device_errors() == 0
    # an out-of-range block id is reported and skipped, never dereferenced
    bt = g["bt"].clone()
    bt[1, 1] = wl.num_blocks + 5
    eng.decode(g["q"], bt, g["ctx"], wl.scale)
    torch.cuda.synchronize()
    assert eng.device_errors() & pa.PA_DEVERR_BAD_BLOCK


def test_int8_overlapped_prologue_gives_the_same_bits():
    wl = CASES["bf16_g8"]()
    g = build_int8(wl, workers=64)
    eng = g["eng"]
    again = eng.decode(g["q"], g["bt"], g["ctx"], wl.scale, num_workers=64,
                       flags=pa.PA_DECODE_OVERLAP_PROLOGUE)
    torch.cuda.synchronize()
    assert torch.equal(again.view(torch.int16), g["out"].view(torch.int16))
