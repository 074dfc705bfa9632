"""The decode entry point for callers that cannot allocate device memory.

Such callers (an embedding host that hands out no device memory, a serving loop
that must not call cudaMalloc while requests run) use
pa_decode_attention_static_ws, which works in the library's own fixed 28 MiB
device scratch instead of a caller workspace.  This file is collected last on
purpose.  The GPU tests call the new entry point through the C ABI, twice in a
row and across shapes whose batch and head counts differ, and check each result
against the ordinary entry point's and against the oracle, within the tolerance
the other parity tests use.  The host tests check that every argument, and the
size limit of the fixed area, is checked before the device is touched."""
import ctypes as C

import numpy as np
import pytest
import torch

import workloads
import paged_kv_cache_486_b200 as pa

STATIC_BYTES = 28 << 20  # the area's size as include/pa.h states it


def _static_call(wl, g, out):
    q, eng = g["q"], g["eng"]
    NB, Hkv, bs, D = eng.k_cache.shape
    st = pa.lib.pa_decode_attention_static_ws(
        C.c_void_p(out.data_ptr()), C.c_void_p(q.data_ptr()), C.c_void_p(eng.k_cache.data_ptr()),
        C.c_void_p(eng.v_cache.data_ptr()), C.c_void_p(g["bt"].data_ptr()),
        C.c_void_p(g["ctx"].data_ptr()), wl.B, wl.Hq, Hkv, D, bs, NB, g["bt"].shape[1],
        wl.scale, pa.DTYPE_CODE[q.dtype], C.c_void_p(eng.dev_error.data_ptr()),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == pa.PA_OK, pa.pa_last_error()


def _host_call(B=4, Hq=8, Hkv=2, D=128, bs=16, NB=10, MB=4, scale=0.1, dtype=pa.PA_F16,
               ptr=C.c_void_p(16)):
    return pa.lib.pa_decode_attention_static_ws(ptr, ptr, ptr, ptr, ptr, ptr, B, Hq, Hkv, D, bs,
                                                NB, MB, scale, dtype, None, None)


# ------------------------------------------------------------------ host only
def test_every_group_up_to_2048_fits_the_area_and_the_layout_ignores_the_batch():
    for G in list(range(1, 65)) + [96, 128, 255, 256, 512, 1000, 1024, 2047, 2048]:
        for D in (64, 128):
            need = pa.pa_decode_workspace_size(1, G, 1, D)
            assert 0 < need <= STATIC_BYTES, (G, D, need)
            # one workspace serves calls of any batch: its size does not depend on it
            assert pa.pa_decode_workspace_size(4096, G, 1, D) == need
    assert pa.pa_decode_workspace_size(8, 8192, 1, 128) > STATIC_BYTES


@pytest.mark.parametrize("bad", [
    dict(Hq=8192, Hkv=1),            # needs more scratch than the fixed area holds
    dict(Hq=16384, Hkv=2),
    dict(D=96), dict(Hq=7), dict(Hkv=0), dict(bs=12), dict(B=-1), dict(B=5000), dict(dtype=7),
    dict(scale=float("nan")), dict(NB=1 << 24, Hkv=16, Hq=16), dict(B=4096, Hkv=128, Hq=128),
    dict(ptr=None),
])
def test_static_entry_rejects_on_the_host_before_touching_the_device(bad):
    # no GPU is needed: a check that reached the device would fail with PA_ERR_CUDA
    st = _host_call(**bad)
    assert st == pa.PA_ERR_INVALID, pa.pa_last_error()
    assert pa.pa_last_error()


def test_static_entry_with_an_empty_batch_is_a_no_op():
    assert _host_call(B=0, ptr=None) == pa.PA_OK


# ----------------------------------------------------------------------- GPU
def _check_against_workspace_and_oracle(wl, g, with_oracle=True):
    from gpu_side import tol_ok
    from oracle_side import attention, run_script
    ref_ws = g["out"].double().cpu().numpy()
    ref_o = attention(wl, run_script(wl)) if with_oracle else None
    for _ in range(2):  # two calls in a row share (and reuse) the same scratch
        out = torch.full_like(g["q"], float("nan"))
        _static_call(wl, g, out)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        ok, worst = tol_ok(got, ref_ws, wl.dtype)
        assert ok, f"{wl.name} vs workspace entry: worst error / bound = {worst:.3f}"
        if with_oracle:
            ok, worst = tol_ok(got, ref_o, wl.dtype)
            assert ok, f"{wl.name} vs oracle: worst error / bound = {worst:.3f}"
    assert g["eng"].device_errors() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("make", [
    lambda: workloads.custom("na16", "f16", B=6, Hq=32, Hkv=8, D=128, bs=16,
                             ctx=[1, 17, 300, 900, 2000, 4000], seed=31),
    lambda: workloads.custom("nabf", "bf16", B=5, Hq=64, Hkv=8, D=128, bs=32,
                             ctx=[5, 64, 700, 1500, 3000], seed=32),
    workloads.tiny,
])
def test_static_scratch_entry_matches_the_workspace_entry_and_the_oracle(cuda_ok, make):
    from gpu_side import build
    wl = make()
    _check_against_workspace_and_oracle(wl, build(wl))


@pytest.mark.gpu
def test_calls_of_changing_batch_and_head_counts_share_the_area(cuda_ok):
    """B * Hkv goes 16 -> 2048 -> 16 -> 320 over calls on the one area, with contexts
    long enough that sequences are split over workers and merged from partial
    results: each call's counters sit where an earlier call of another shape kept
    partial results, and each call must still match the workspace entry point."""
    from gpu_side import build
    rng = np.random.default_rng(77)
    shapes = [
        workloads.custom("grow0", "f16", B=2, Hq=64, Hkv=8, D=128, bs=16, ctx=[12000, 9000],
                         seed=71),
        workloads.custom("grow1", "f16", B=256, Hq=16, Hkv=8, D=128, bs=16,
                         ctx=rng.integers(1, 1500, size=256), seed=72),
        workloads.custom("grow2", "bf16", B=4, Hq=16, Hkv=4, D=64, bs=16,
                         ctx=[7000, 3, 5000, 800], seed=73),
        workloads.custom("grow3", "bf16", B=40, Hq=64, Hkv=8, D=128, bs=32,
                         ctx=rng.integers(100, 4000, size=40), seed=74),
    ]
    for i, wl in enumerate(shapes):
        _check_against_workspace_and_oracle(wl, build(wl), with_oracle=(i != 1))
