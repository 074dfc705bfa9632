"""CUDA path against the oracle: block tables and cache writes bit-exact,
attention within the stated tolerance, on every configuration and edge case."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import paged_kv_cache_486_b200 as pa
from gpu_side import bits, build, gathered, tol_ok
from oracle_side import all_rows, attention, contiguous_row, raw, run_script

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


def _small_cases():
    C = workloads.custom
    return {
        "tiny": workloads.tiny,
        "f16_g4_d128": lambda: C("a", "f16", B=7, Hq=32, Hkv=8, D=128, bs=16,
                                 ctx=[1, 15, 16, 17, 33, 300, 1000], seed=11),
        "bf16_g8_d128": lambda: C("b", "bf16", B=6, Hq=64, Hkv=8, D=128, bs=16,
                                  ctx=[2, 31, 64, 129, 700, 1500], seed=12),
        "f16_g1_bs32": lambda: C("c", "f16", B=4, Hq=8, Hkv=8, D=128, bs=32,
                                 ctx=[1, 32, 33, 900], seed=13),
        "bf16_g2_d64": lambda: C("d", "bf16", B=5, Hq=4, Hkv=2, D=64, bs=16,
                                 ctx=[3, 16, 48, 200, 517], seed=14),
        "f16_mqa_g4": lambda: C("e", "f16", B=3, Hq=4, Hkv=1, D=128, bs=16,
                                ctx=[5, 250, 999], seed=15),
        "f16_g16_simt": lambda: C("f", "f16", B=3, Hq=32, Hkv=2, D=128, bs=16,
                                  ctx=[7, 90, 400], seed=16),
        "bf16_bs8_simt": lambda: C("g", "bf16", B=4, Hq=8, Hkv=2, D=64, bs=8,
                                   ctx=[1, 8, 9, 333], seed=17),
        "f32_d128": lambda: C("h", "f32", B=3, Hq=8, Hkv=2, D=128, bs=16, ctx=[4, 77, 300],
                              seed=18),
        "f16_bs64": lambda: C("i", "f16", B=3, Hq=16, Hkv=4, D=128, bs=64, ctx=[1, 64, 650],
                              seed=19),
    }


SMALL = _small_cases()


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("path,workers", [(pa.PA_PATH_AUTO, 0), (pa.PA_PATH_AUTO, 1),
                                          (pa.PA_PATH_AUTO, 5), (pa.PA_PATH_SIMT, 0)])
def test_small_configs_match_the_oracle(name, path, workers):
    wl = SMALL[name]()
    g = build(wl, path=path, workers=workers)
    o = run_script(wl)
    # block tables and context lengths: bit-exact
    assert np.array_equal(g["bt"].cpu().numpy(), o["table"])
    assert np.array_equal(g["ctx"].cpu().numpy(), o["ctx"])
    # every cached row of every sequence: bit-exact against the oracle's cache
    for b in range(wl.B):
        n = int(o["ctx"][b])
        pos = np.arange(n)
        slots = o["table"][b][pos // wl.bs] * wl.bs + pos % wl.bs
        for kind, cache in ((0, o["k_cache"]), (1, o["v_cache"])):
            ref = cache[slots // wl.bs, :, slots % wl.bs, :]
            got = raw(gathered(g["eng"], g["bt"], g["ctx"], b, kind))
            assert np.array_equal(got, ref)
    ref = attention(wl, o)
    got = g["out"].double().cpu().numpy()
    ok, worst = tol_ok(got, ref, wl.dtype)
    assert ok, f"worst error / bound = {worst:.3f}"
    assert g["eng"].device_errors() == 0


def test_tensor_core_path_is_used_and_forced_paths_agree():
    wl = SMALL["bf16_g8_d128"]()
    o = attention(wl, run_script(wl))
    outs = {}
    for path in (pa.PA_PATH_TC, pa.PA_PATH_SIMT):
        for workers in (1, 3, 64, 2048):
            g = build(wl, path=path, workers=workers)
            ok, worst = tol_ok(g["out"].double().cpu().numpy(), o, wl.dtype)
            assert ok, (path, workers, worst)
            outs[(path, workers)] = g["out"]
    # the same path with the same split is deterministic
    again = build(wl, path=pa.PA_PATH_TC, workers=64)["out"]
    assert torch.equal(bits(again), bits(outs[(pa.PA_PATH_TC, 64)]))


@pytest.mark.parametrize("name", ["llama3_8b", "llama3_70b", "shared_prefix", "long_mha",
                                  "long_mha_bs32"])
def test_full_size_configs(name):
    """Every output row of the full-size workload against the oracle, and every cached
    row of every sequence bit-exact against the sequence's logical rows."""
    wl = workloads.make(name)
    g = build(wl)
    eng, bt, ctx, out = g["eng"], g["bt"], g["ctx"], g["out"]
    # block tables bit-exact against the oracle's pool model (host ints only)
    o = run_script(wl, with_cache=False)
    assert np.array_equal(bt.cpu().numpy(), o["table"])
    assert np.array_equal(ctx.cpu().numpy(), o["ctx"])
    copies = [r[1] for r in g["records"] if r is not None and len(r[1])]
    copies_o = [r[1] for r in o["records"] if r is not None and len(r[1])]
    assert len(copies) == len(copies_o)
    assert all(np.array_equal(a, b) for a, b in zip(copies, copies_o))
    got = out.double().cpu().numpy()
    assert np.all(np.isfinite(got))

    def exact(b, k, v):
        # the cache read back through the table equals the logical rows, exactly
        return all(torch.equal(bits(gathered(eng, bt, ctx, b, kind)), bits(ref))
                   for kind, ref in ((0, k), (1, v)))

    # long contexts hold 1 GB of logical rows per sequence, so fewer rows at once
    ref, same = all_rows(wl, threads=2 if name.startswith("long") else None, visit=exact)
    assert all(same), [b for b, x in enumerate(same) if not x][:10]
    ok, worst = tol_ok(got, ref, wl.dtype)
    assert ok, f"worst error / bound = {worst:.3f}"
    assert eng.device_errors() == 0


def test_split_and_single_pass_agree_at_full_size():
    """Other splits of the 8B-shaped batch (37 workers, one worker) against the
    oracle on every row: the result does not depend on how the work is cut."""
    wl = workloads.make("llama3_8b")
    ref, _ = all_rows(wl)
    for workers in (37, 1):
        x = build(wl, workers=workers)
        ok, worst = tol_ok(x["out"].double().cpu().numpy(), ref, "f16")
        assert ok, (workers, worst)


def test_block_size_and_sharing_do_not_change_the_result():
    base = workloads.custom("s16", "f16", B=4, Hq=16, Hkv=4, D=128, bs=16, ctx=[40, 129, 300, 5],
                            seed=21)
    other = workloads.custom("s32", "f16", B=4, Hq=16, Hkv=4, D=128, bs=32, ctx=[40, 129, 300, 5],
                             seed=21)
    x = build(base)["out"].double().cpu().numpy()
    y = build(other)["out"].double().cpu().numpy()
    ok, worst = tol_ok(x, y, "f16")
    assert ok, worst
    # shared prefix with copy-on-write equals the unshared logical rows (oracle, contiguous)
    wl = workloads.shared_prefix(n_groups=5, n_samples=4, prefix_len=80)
    g = build(wl)
    for b in range(wl.B):
        ref = contiguous_row(wl, b)
        ok, worst = tol_ok(g["out"][b].double().cpu().numpy(), ref, "f16")
        assert ok, (b, worst)


def test_copy_blocks_is_byte_exact_over_layers():
    torch.manual_seed(0)
    L, NB, Hkv, bs, D = 3, 12, 2, 16, 64
    ks = [torch.randn(NB, Hkv, bs, D, device="cuda").half() for _ in range(L)]
    vs = [torch.randn(NB, Hkv, bs, D, device="cuda").half() for _ in range(L)]
    pairs = np.array([[1, 4], [2, 7], [1, 9]], np.int32)
    kh = [raw(k) for k in ks]
    vh = [raw(v) for v in vs]
    oracle.copy_blocks(kh, vh, pairs)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks(ks, vs, torch.from_numpy(pairs).cuda(), err)
    torch.cuda.synchronize()
    for i in range(L):
        assert np.array_equal(raw(ks[i]), kh[i]) and np.array_equal(raw(vs[i]), vh[i])
    assert pa.pa_check_device_error(err) == 0


def test_empty_contexts_give_zero_rows():
    wl = workloads.custom("z", "bf16", B=4, Hq=16, Hkv=4, D=128, bs=16, ctx=[3, 50, 1, 70], seed=5)
    g = build(wl)
    ctx = g["ctx"].clone()
    ctx[1] = 0
    ctx[3] = 0
    out = g["eng"].decode(g["q"], g["bt"], ctx, wl.scale)
    torch.cuda.synchronize()
    assert not out[1].float().any() and not out[3].float().any()
    assert torch.equal(bits(out[0]), bits(g["out"][0])) or tol_ok(
        out[0].double().cpu().numpy(), g["out"][0].double().cpu().numpy(), "bf16")[0]
    allzero = torch.zeros_like(ctx)
    out2 = g["eng"].decode(g["q"], g["bt"], allzero, wl.scale)
    torch.cuda.synchronize()
    assert not out2.float().any()


def test_device_guards_report_instead_of_faulting():
    wl = workloads.custom("guard", "f16", B=3, Hq=8, Hkv=2, D=128, bs=16, ctx=[20, 40, 60],
                          seed=6)
    g = build(wl)
    eng = g["eng"]
    assert eng.device_errors() == 0
    bt = g["bt"].clone()
    bt[1, 0] = wl.num_blocks + 5          # block id outside the pool
    eng.decode(g["q"], bt, g["ctx"], wl.scale)
    assert eng.device_errors() & pa.PA_DEVERR_BAD_BLOCK
    eng.decode(g["q"], bt, g["ctx"], wl.scale, path=pa.PA_PATH_SIMT)
    assert eng.device_errors() & pa.PA_DEVERR_BAD_BLOCK
    ctx = g["ctx"].clone()
    ctx[2] = wl.max_blocks * wl.bs + 1    # longer than the table row
    eng.decode(g["q"], g["bt"], ctx, wl.scale)
    assert eng.device_errors() & pa.PA_DEVERR_BAD_CTX
    k = torch.zeros(2, wl.Hkv, wl.D, dtype=torch.float16, device="cuda")
    slots = torch.tensor([wl.num_blocks * wl.bs, -1], dtype=torch.int64, device="cuda")
    before = eng.k_cache.clone()
    pa.pa_reshape_and_cache(k, k, eng.k_cache, eng.v_cache, slots, eng.dev_error)
    assert eng.device_errors() & pa.PA_DEVERR_BAD_SLOT
    assert torch.equal(bits(before), bits(eng.k_cache))
    pairs = torch.tensor([[0, wl.num_blocks]], dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks([eng.k_cache], [eng.v_cache], pairs, eng.dev_error)
    assert eng.device_errors() & pa.PA_DEVERR_BAD_BLOCK
    # the context stays usable
    out = eng.decode(g["q"], g["bt"], g["ctx"], wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(bits(out), bits(g["out"]))


def test_overlapped_prologue_gives_the_same_bits():
    wl = workloads.custom("ovl", "bf16", B=5, Hq=64, Hkv=8, D=128, bs=16,
                          ctx=[3, 100, 700, 1600, 2500], seed=41)
    g = build(wl)
    eng = g["eng"]
    k = wl.tokens(7, 0, wl.B, 0, "cuda")
    v = wl.tokens(7, 0, wl.B, 1, "cuda")
    # rewrite each sequence's last token, then decode right behind the cache write
    last = []
    for b in range(wl.B):
        n = int(g["ctx"][b])
        blk = int(g["bt"][b, (n - 1) // wl.bs])
        last.append(blk * wl.bs + (n - 1) % wl.bs)
    slots = torch.tensor(last, dtype=torch.int64, device="cuda")
    outs = []
    for flags in (0, pa.PA_DECODE_OVERLAP_PROLOGUE, pa.PA_DECODE_OVERLAP_PROLOGUE):
        pa.pa_reshape_and_cache(k, v, eng.k_cache, eng.v_cache, slots, eng.dev_error)
        outs.append(eng.decode(g["q"], g["bt"], g["ctx"], wl.scale, flags=flags))
    torch.cuda.synchronize()
    assert torch.equal(bits(outs[0]), bits(outs[1])) and torch.equal(bits(outs[1]), bits(outs[2]))
    assert not torch.equal(bits(outs[0]), bits(g["out"]))  # the rewritten tokens were seen
    assert eng.device_errors() == 0


@pytest.mark.parametrize("B,Hq,Hkv,D,dtype", [(4096, 64, 64, 64, "f16"),   # B * Hkv = 262144
                                              (4096, 32, 8, 128, "bf16")])  # the largest batch
def test_maximum_batch_and_pair_counts(B, Hq, Hkv, D, dtype):
    """The largest shapes the decode accepts: batch 4096 (the context scan's limit) and
    batch x kv heads = 262144 (the workspace's arrival counts), with short contexts of
    1..40 tokens; every row against the oracle, on both paths."""
    rng = np.random.default_rng(90 + Hkv)
    wl = workloads.custom("maxsz", dtype, B=B, Hq=Hq, Hkv=Hkv, D=D, bs=16,
                          ctx=rng.integers(1, 41, size=B), seed=91, shuffle=False)
    ref, _ = all_rows(wl)
    for path in (pa.PA_PATH_AUTO, pa.PA_PATH_SIMT):
        g = build(wl, path=path)
        ok, worst = tol_ok(g["out"].double().cpu().numpy(), ref, wl.dtype)
        assert ok, (path, worst)
        assert g["eng"].device_errors() == 0
