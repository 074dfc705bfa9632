"""The decode entry point for callers that cannot allocate device memory.

Such callers (an embedding host that hands out no device memory, a serving loop
that must not call cudaMalloc while requests run) use
pa_decode_attention_static_ws, which works in the library's own fixed device
scratch instead of a caller workspace.  This file is collected last on purpose.
The test calls the new entry point through the C ABI twice in a row and checks
each result against the ordinary entry point's on the same inputs, within the
tolerance the other parity tests use."""
import ctypes as C

import pytest
import torch

import workloads
import paged_kv_cache_486_b200 as pa
from gpu_side import build, tol_ok

pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("make", [
    lambda: workloads.custom("na16", "f16", B=6, Hq=32, Hkv=8, D=128, bs=16,
                             ctx=[1, 17, 300, 900, 2000, 4000], seed=31),
    lambda: workloads.custom("nabf", "bf16", B=5, Hq=64, Hkv=8, D=128, bs=32,
                             ctx=[5, 64, 700, 1500, 3000], seed=32),
    workloads.tiny,
])
def test_static_scratch_entry_matches_the_workspace_entry(cuda_ok, make):
    wl = make()
    g = build(wl)  # ordinary entry point, caller workspace
    ref = g["out"].double().cpu().numpy()
    for _ in range(2):  # two calls in a row share (and reuse) the same scratch
        out = torch.full_like(g["q"], float("nan"))
        _static_call(wl, g, out)
        torch.cuda.synchronize()
        ok, worst = tol_ok(out.double().cpu().numpy(), ref, wl.dtype)
        assert ok, f"worst error / bound = {worst:.3f}"
    assert g["eng"].device_errors() == 0
