"""Paged prefill / chunked-prefill attention on the GPU against the oracle: every
row within the fp16/bf16 bound on small cases (whole prompts, chunks after
earlier context, single new tokens, ragged tiles), sampled rows at full size,
and the guards (empty chunks, lengths the launch does not cover, bad block ids)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import paged_kv_cache_486_b200 as pa
from gpu_side import NAN_BITS, tol_ok
from oracle_side import raw, run_script
from paged_kv_cache_486_b200.engine import PagedKVCache

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


def _build(wl):
    dt = workloads.TORCH_DTYPE[wl.dtype]
    eng = PagedKVCache(wl.num_blocks, wl.bs, wl.Hkv, wl.D, dt, wl.Hq, wl.B, "cuda",
                       fill_bits=NAN_BITS[wl.dtype])
    eng.apply_ops(wl.ops, lambda s, p, n: (wl.tokens(s, p, n, 0, "cuda"),
                                           wl.tokens(s, p, n, 1, "cuda")))
    bt, ctx = eng.block_tables(wl.batch, wl.max_blocks)
    qs = torch.from_numpy(workloads.query_start(wl)).cuda()
    q = workloads.q_prefill(wl, "cuda")
    torch.cuda.synchronize()
    return eng, bt, ctx, qs, q


def _cases():
    P = workloads.prefill
    return {
        "f16_g4_d128": lambda: P("a", "f16", 32, 8, 128, 16, [1, 17, 64, 300, 700, 90],
                                 [1, 17, 30, 120, 700, 90], 31),
        "bf16_g8_d128": lambda: P("b", "bf16", 64, 8, 128, 16, [40, 129, 513, 1000],
                                  [40, 1, 200, 513], 32),
        "f16_g1_bs32": lambda: P("c", "f16", 8, 8, 128, 32, [33, 97, 400], [33, 60, 5], 33),
        "bf16_g2_d64_bs64": lambda: P("d", "bf16", 4, 2, 64, 64, [65, 300, 777], [64, 300, 100],
                                      34),
        "f16_mqa_g16": lambda: P("e", "f16", 16, 1, 128, 16, [5, 250, 999], [5, 250, 31], 35),
        "f16_g64_d64": lambda: P("f", "f16", 64, 1, 64, 16, [7, 90], [7, 45], 36),
        # large groups at head_dim 128: the tcgen05 kernel's query boxes of 4 and 2 tokens
        "bf16_g32_d128": lambda: P("g", "bf16", 64, 2, 128, 16, [3, 70, 260], [3, 37, 260], 37),
        "f16_g64_d128": lambda: P("h", "f16", 64, 1, 128, 32, [130, 9], [66, 9], 38),
    }


CASES = _cases()


# the automatic choice (the one-SM tcgen05 kernel where it applies), the tcgen05
# kernel on pairs of SMs where it applies, and mma.sync
PATHS = [pa.PA_PREFILL_AUTO, pa.PA_PREFILL_TCGEN05_PAIR, pa.PA_PREFILL_MMA_SYNC]


def _path_applies(wl, path):
    return path != pa.PA_PREFILL_TCGEN05_PAIR or (wl.D == 128 and 128 % wl.G == 0)


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("path", PATHS)
def test_prefill_small_configs_match_the_oracle(name, path):
    wl = CASES[name]()
    if not _path_applies(wl, path):
        pytest.skip("the tcgen05 pair kernel takes head_dim 128 only")
    eng, bt, ctx, qs, q = _build(wl)
    out = eng.prefill(q, bt, ctx, qs, int(wl.n_new.max()), wl.scale, path=path)
    torch.cuda.synchronize()
    o = run_script(wl)
    ref = oracle.paged_prefill_attention(raw(q), o["k_cache"], o["v_cache"], o["table"],
                                         o["ctx"], workloads.query_start(wl), wl.scale, wl.dtype)
    ok, worst = tol_ok(out.double().cpu().numpy(), ref, wl.dtype)
    assert ok, f"worst error / bound = {worst:.3f}"
    assert eng.device_errors() == 0
    # a larger max_q only launches more (empty) tiles
    again = eng.prefill(q, bt, ctx, qs, int(wl.n_new.max()) + 100, wl.scale, path=path)
    torch.cuda.synchronize()
    assert torch.equal(again.view(torch.int16), out.view(torch.int16))


@pytest.mark.parametrize("name", ["prefill_8b", "chunked_8b"])
@pytest.mark.parametrize("path", PATHS)
def test_prefill_full_size_sampled_rows(name, path):
    wl = {"prefill_8b": workloads.prefill_8b, "chunked_8b": workloads.chunked_8b}[name]()
    eng, bt, ctx, qs, q = _build(wl)
    out = eng.prefill(q, bt, ctx, qs, int(wl.n_new.max()), wl.scale, path=path)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    o = run_script(wl, with_cache=False)
    assert np.array_equal(bt.cpu().numpy(), o["table"])
    # sampled rows: first, last and random new tokens of a few sequences, the oracle
    # reading the same cache rows (built from the script on the CPU)
    rng = np.random.default_rng(4869)
    qsn = workloads.query_start(wl)
    rows = []
    for b in sorted(rng.choice(wl.B, size=3, replace=False)):
        toks = {int(qsn[b]), int(qsn[b + 1]) - 1} | set(
            int(x) for x in rng.integers(qsn[b], qsn[b + 1], size=3))
        for t in sorted(toks):
            for h in rng.choice(wl.Hq, size=2, replace=False):
                rows.append(t * wl.Hq + int(h))
    full = run_script(wl)
    ref = oracle.paged_prefill_attention(raw(q), full["k_cache"], full["v_cache"],
                                         full["table"], full["ctx"], qsn, wl.scale, wl.dtype,
                                         rows=rows)
    got = out.double().cpu().numpy().reshape(-1, wl.D)[rows]
    ok, worst = tol_ok(got, ref.reshape(-1, wl.D)[rows], wl.dtype)
    assert ok, f"worst error / bound = {worst:.3f}"
    assert eng.device_errors() == 0


@pytest.mark.parametrize("path", PATHS)
def test_prefill_guards(path):
    wl = CASES["f16_g4_d128"]()
    eng, bt, ctx, qs, q = _build(wl)
    ref = eng.prefill(q, bt, ctx, qs, int(wl.n_new.max()), wl.scale, path=path).clone()
    torch.cuda.synchronize()
    # a chunk longer than max_q: that sequence is skipped and reported; others unchanged
    out = torch.zeros_like(q)
    eng.prefill(q, bt, ctx, qs, 200, wl.scale, out=out, path=path)
    torch.cuda.synchronize()
    assert eng.device_errors() & pa.PA_DEVERR_BAD_CTX
    qsn = workloads.query_start(wl)
    for b in range(wl.B):
        seg = slice(int(qsn[b]), int(qsn[b + 1]))
        if wl.n_new[b] <= 200:
            assert torch.equal(out[seg].view(torch.int16), ref[seg].view(torch.int16))
        else:
            assert not out[seg].float().any()
    # an out-of-range block id: reported, its keys skipped, nothing faults
    bt2 = bt.clone()
    bt2[3, 2] = wl.num_blocks + 7
    eng.prefill(q, bt2, ctx, qs, int(wl.n_new.max()), wl.scale, path=path)
    torch.cuda.synchronize()
    assert eng.device_errors() & pa.PA_DEVERR_BAD_BLOCK
    # no new tokens anywhere
    empty = torch.zeros_like(qs)
    eng.prefill(q[:0], bt, ctx, empty, 0, wl.scale, path=path)
    torch.cuda.synchronize()
    assert eng.device_errors() == 0


@pytest.mark.parametrize("name", ["f16_g4_d128", "bf16_g8_d128", "f16_g1_bs32"])
@pytest.mark.parametrize("path", [pa.PA_PREFILL_TCGEN05, pa.PA_PREFILL_TCGEN05_PAIR])
def test_prefill_persistent_and_per_item_launches_agree(name, path):
    """Each tcgen05 kernel with a scheduling workspace (persistent, items handed
    out by a counter) and without (one item per CTA or CTA pair) computes every
    item the same way: identical bits, and the workspace is left zero for the
    next call."""
    wl = CASES[name]()
    eng, bt, ctx, qs, q = _build(wl)
    max_q = int(wl.n_new.max())
    ws = torch.zeros(2, dtype=torch.int64, device="cuda")
    outs = []
    for workspace in (ws, None, ws):
        out = torch.full_like(q, float("nan"))
        pa.pa_prefill_attention(out, q, eng.k_cache, eng.v_cache, bt, ctx, qs, max_q, wl.scale,
                                eng.dev_error, path, workspace)
        torch.cuda.synchronize()
        outs.append(out)
        assert not ws.any(), "the scheduling counter was not returned to zero"
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    assert torch.equal(outs[0].view(torch.int16), outs[2].view(torch.int16))
    assert eng.device_errors() == 0


@pytest.mark.parametrize("width", [1024, 2000, 6000])
def test_prefill_item_order_blocks_of_pairs(width):
    """The one-SM tcgen05 kernel hands out its items longest first within blocks
    of (sequence, kv head) pairs sized from the table's width (the pairs whose
    keys and values fit in part of L2).  A wider table with the same contents
    gives blocks of 5, 2 and 1 of these 48 pairs (the last block partial for 5):
    every row still matches the oracle, persistent or one item per CTA, with the
    same bits as the narrow table."""
    wl = workloads.prefill("w", "f16", 32, 8, 128, 16, [40, 129, 513, 1000, 700, 260],
                           [40, 1, 200, 513, 700, 77], 39)
    eng, bt, ctx, qs, q = _build(wl)
    wide, ctx_w = eng.block_tables(wl.batch, width)
    assert torch.equal(ctx, ctx_w) and torch.equal(wide[:, :bt.shape[1]], bt)
    max_q = int(wl.n_new.max())
    o = run_script(wl)
    ref = oracle.paged_prefill_attention(raw(q), o["k_cache"], o["v_cache"], o["table"],
                                         o["ctx"], workloads.query_start(wl), wl.scale, wl.dtype)
    narrow = torch.empty_like(q)
    pa.pa_prefill_attention(narrow, q, eng.k_cache, eng.v_cache, bt, ctx, qs, max_q, wl.scale,
                            eng.dev_error, pa.PA_PREFILL_TCGEN05, eng.prefill_ws)
    for workspace in (eng.prefill_ws, None):
        out = torch.full_like(q, float("nan"))
        pa.pa_prefill_attention(out, q, eng.k_cache, eng.v_cache, wide, ctx, qs, max_q,
                                wl.scale, eng.dev_error, pa.PA_PREFILL_TCGEN05, workspace)
        torch.cuda.synchronize()
        ok, worst = tol_ok(out.double().cpu().numpy(), ref, wl.dtype)
        assert ok, f"worst error / bound = {worst:.3f}"
        assert torch.equal(out.view(torch.int16), narrow.view(torch.int16))
    assert eng.device_errors() == 0
