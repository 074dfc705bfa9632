"""A bounded device wait that runs out, in the form that neither faults nor hangs a
GPU: with PA_DECODE_TEST_WAIT_EXPIRY every worker of the tensor-core decode treats
its first tile wait as run out, and the warp feeding it then waits for a slot
release that never comes until that wait's own limit (about a second) ends it.
The call must come back with PA_DEVERR_TIMEOUT set, the context must stay usable,
and, once the workspace counters are zeroed again (the documented recovery), the
next call must match the oracle."""
import time

import pytest
import torch

import oracle
import workloads
import paged_kv_cache_486_b200 as pa
from gpu_side import build, build_int8, tol_ok
from oracle_side import attention, raw, run_script, run_script_int8

pytestmark = pytest.mark.gpu


def _case():
    return workloads.custom("expiry", "f16", B=4, Hq=32, Hkv=8, D=128, bs=16,
                            ctx=[300, 700, 1200, 2000], seed=81)


def test_decode_wait_expiry_reports_and_the_next_call_is_correct(cuda_ok):
    wl = _case()
    g = build(wl)
    eng = g["eng"]
    assert eng.device_errors() == 0
    out = torch.full_like(g["q"], float("nan"))
    t0 = time.perf_counter()
    # four workers, each with far more stages than its ring holds, so every
    # worker gives up with copies of its own in flight
    eng.decode(g["q"], g["bt"], g["ctx"], wl.scale, out=out, num_workers=4,
               flags=pa.PA_DECODE_TEST_WAIT_EXPIRY)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert eng.device_errors() & pa.PA_DEVERR_TIMEOUT
    assert elapsed < 30.0
    assert torch.isnan(out.float()).all()  # no row was written
    eng.workspace.zero_()
    for workers in (4, 0):
        again = eng.decode(g["q"], g["bt"], g["ctx"], wl.scale, num_workers=workers)
        torch.cuda.synchronize()
        ref = attention(wl, run_script(wl))
        ok, worst = tol_ok(again.double().cpu().numpy(), ref, wl.dtype)
        assert ok, f"worst error / bound = {worst:.3f}"
    assert eng.device_errors() == 0


def test_int8_decode_wait_expiry_reports_and_the_next_call_is_correct(cuda_ok):
    wl = _case()
    g = build_int8(wl)
    eng = g["eng"]
    assert eng.device_errors() == 0
    eng.decode(g["q"], g["bt"], g["ctx"], wl.scale, num_workers=4,
               flags=pa.PA_DECODE_TEST_WAIT_EXPIRY)
    torch.cuda.synchronize()
    assert eng.device_errors() & pa.PA_DEVERR_TIMEOUT
    eng.workspace.zero_()
    again = eng.decode(g["q"], g["bt"], g["ctx"], wl.scale)
    torch.cuda.synchronize()
    o = run_script_int8(wl)
    ref = oracle.paged_decode_attention_int8(raw(wl.q()), o["cache"], o["table"], o["ctx"],
                                             wl.scale, wl.dtype)
    ok, worst = tol_ok(again.double().cpu().numpy(), ref, wl.dtype)
    assert ok, f"worst error / bound = {worst:.3f}"
    assert eng.device_errors() == 0
