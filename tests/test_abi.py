"""The C ABI library loads without a GPU, exports every function include/*.h
declares, and rejects bad arguments on the host before any device work."""
import ctypes as C
import glob
import os
import re

import pytest

import paged_kv_cache_486_b200 as pa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(pa_[a-z0-9_]+)\s*\(", text):
            names.add(m.group(1))
    return names


def test_every_declared_symbol_is_exported_and_bound():
    declared = _declared()
    assert len(declared) >= 20
    raw = C.CDLL(pa.LIB_PATH)
    for name in declared:
        assert hasattr(raw, name), name
        assert name in pa.SIGNATURES, f"binding lacks {name}"


def test_loaded_library_is_the_in_tree_build():
    assert os.path.dirname(pa.LIB_PATH) == os.path.join(ROOT, "paged_kv_cache_486_b200")
    assert os.path.exists(pa.LIB_PATH)


def test_kv_bytes():
    assert pa.pa_kv_bytes(80, 1, 8, 128, 2) == 327680
    assert pa.pa_kv_bytes(32, 4096, 8, 128, 2) == 2 * 32 * 4096 * 8 * 128 * 2


def _decode_args(**kw):
    args = dict(out=C.c_void_p(16), q=C.c_void_p(16), k=C.c_void_p(16), v=C.c_void_p(16),
                bt=C.c_void_p(16), ctx=C.c_void_p(16), B=4, Hq=8, Hkv=2, D=128, bs=16, NB=10,
                MB=4, scale=0.1, dtype=pa.PA_F16, ws=C.c_void_p(16), ws_bytes=1 << 30, err=None,
                path=0, workers=0, flags=0, stream=None)
    args.update(kw)
    return args


def _call_decode(a):
    return pa.lib.pa_decode_attention_ex(a["out"], a["q"], a["k"], a["v"], a["bt"], a["ctx"],
                                         a["B"], a["Hq"], a["Hkv"], a["D"], a["bs"], a["NB"],
                                         a["MB"], a["scale"], a["dtype"], a["ws"], a["ws_bytes"],
                                         a["err"], a["path"], a["workers"], a["flags"],
                                         a["stream"])


@pytest.mark.parametrize("bad", [
    dict(D=96), dict(Hq=7), dict(Hkv=0), dict(bs=12), dict(B=-1), dict(B=5000), dict(dtype=7),
    dict(ws_bytes=16), dict(q=None), dict(k=C.c_void_p(8)), dict(path=9),
    dict(path=pa.PA_PATH_TC, dtype=pa.PA_F32), dict(path=pa.PA_PATH_TC, Hq=32, Hkv=2),
    dict(path=pa.PA_PATH_TC, bs=8), dict(NB=1 << 24, Hkv=16, Hq=16), dict(scale=float("nan")),
    dict(flags=2), dict(B=4096, Hkv=128, Hq=128),
    # the test-only wait-expiry flag exists on the tensor-core path only
    dict(flags=pa.PA_DECODE_TEST_WAIT_EXPIRY, path=pa.PA_PATH_SIMT),
    dict(flags=pa.PA_DECODE_TEST_WAIT_EXPIRY, dtype=pa.PA_F32),
])
def test_decode_rejects_bad_arguments_on_host(bad):
    st = _call_decode(_decode_args(**bad))
    assert st == pa.PA_ERR_INVALID, pa.pa_last_error()
    assert pa.pa_last_error()


def test_empty_batch_is_a_no_op():
    assert _call_decode(_decode_args(B=0, q=None, out=None)) == pa.PA_OK


def test_cache_write_and_copy_reject_bad_arguments():
    p = C.c_void_p(16)
    assert pa.lib.pa_reshape_and_cache(p, p, p, p, p, 4, 8, 100, 16, 10, pa.PA_F16, None,
                                       None) == pa.PA_ERR_INVALID  # 200-byte rows
    assert pa.lib.pa_reshape_and_cache(p, p, p, p, p, -1, 8, 128, 16, 10, pa.PA_F16, None,
                                       None) == pa.PA_ERR_INVALID
    assert pa.lib.pa_reshape_and_cache(C.c_void_p(8), p, p, p, p, 4, 8, 128, 16, 10, pa.PA_F16,
                                       None, None) == pa.PA_ERR_INVALID
    assert pa.lib.pa_reshape_and_cache(p, p, p, p, p, 0, 8, 128, 16, 10, pa.PA_F16, None,
                                       None) == pa.PA_OK
    arr = (C.c_void_p * 1)(16)
    assert pa.lib.pa_copy_blocks(arr, arr, 0, p, 1, 10, 4096, None, None) == pa.PA_ERR_INVALID
    assert pa.lib.pa_copy_blocks(arr, arr, 129, p, 1, 10, 4096, None, None) == pa.PA_ERR_INVALID
    assert pa.lib.pa_copy_blocks(arr, arr, 1, p, 1, 10, 4100, None, None) == pa.PA_ERR_INVALID
    assert pa.lib.pa_copy_blocks(arr, arr, 1, p, 0, 10, 4096, None, None) == pa.PA_OK


def test_workspace_size_is_independent_of_context_and_grows_with_group():
    a = pa.pa_decode_workspace_size(64, 32, 8, 128)
    b = pa.pa_decode_workspace_size(256, 64, 8, 128)
    assert 0 < a < b < (64 << 20)
    assert pa.pa_decode_workspace_size(4, 7, 2, 128) == 0


def test_plan_chooses_tensor_cores_where_they_apply():
    import torch
    assert pa.pa_decode_plan(64, 32, 8, 128, 16, torch.float16)[0] == pa.PA_PATH_TC
    assert pa.pa_decode_plan(64, 64, 8, 128, 16, torch.bfloat16)[0] == pa.PA_PATH_TC
    assert pa.pa_decode_plan(64, 64, 64, 128, 32, torch.float16)[0] == pa.PA_PATH_TC
    assert pa.pa_decode_plan(4, 4, 2, 64, 16, torch.float32)[0] == pa.PA_PATH_SIMT
    assert pa.pa_decode_plan(4, 32, 2, 128, 16, torch.float16)[0] == pa.PA_PATH_SIMT
    assert pa.pa_decode_plan(4, 8, 2, 128, 8, torch.float16)[0] == pa.PA_PATH_SIMT


def _int8_args(**kw):
    p = C.c_void_p(16)
    args = dict(out=p, q=p, kp=p, vp=p, bt=p, ctx=p, B=4, Hq=8, Hkv=2, D=128, bs=16, NB=10, MB=4,
                scale=0.1, dtype=pa.PA_F16, ws=p, ws_bytes=1 << 30, err=None, workers=0, flags=0,
                stream=None)
    args.update(kw)
    return args


def _call_decode_int8(a):
    return pa.lib.pa_decode_attention_int8(
        a["out"], a["q"], a["kp"], a["vp"], a["bt"], a["ctx"], a["B"], a["Hq"], a["Hkv"], a["D"],
        a["bs"], a["NB"], a["MB"], a["scale"], a["dtype"], a["ws"], a["ws_bytes"], a["err"],
        a["workers"], a["flags"], a["stream"])


@pytest.mark.parametrize("bad", [
    dict(D=64), dict(dtype=pa.PA_F32), dict(Hq=32, Hkv=2), dict(bs=8), dict(bs=48),
    dict(Hq=7), dict(B=-1), dict(B=5000), dict(ws_bytes=16), dict(kp=None),
    dict(vp=C.c_void_p(8)), dict(flags=4), dict(scale=float("nan")),
    dict(NB=1 << 24, Hkv=8, Hq=8), dict(Hkv=5000, Hq=5000), dict(MB=1 << 30, Hkv=4, Hq=8),
])
def test_int8_decode_rejects_bad_arguments_on_host(bad):
    st = _call_decode_int8(_int8_args(**bad))
    assert st == pa.PA_ERR_INVALID, pa.pa_last_error()
    assert pa.pa_last_error()


def test_int8_cache_write_rejects_bad_arguments():
    p = C.c_void_p(16)

    def call(key=p, kp=p, T=4, Hkv=2, D=128, bs=16, NB=10, dt=pa.PA_F16):
        return pa.lib.pa_reshape_and_cache_int8(key, p, kp, p, p, T, Hkv, D, bs, NB, dt, None,
                                                None)

    assert call(D=64) == pa.PA_ERR_INVALID
    assert call(bs=8) == pa.PA_ERR_INVALID
    assert call(bs=24) == pa.PA_ERR_INVALID
    assert call(T=-1) == pa.PA_ERR_INVALID
    assert call(dt=9) == pa.PA_ERR_INVALID
    assert call(key=C.c_void_p(8)) == pa.PA_ERR_INVALID
    assert call(kp=None) == pa.PA_ERR_INVALID
    assert call(T=0) == pa.PA_OK
    assert _call_decode_int8(_int8_args(B=0, q=None, out=None)) == pa.PA_OK


def test_int8_block_bytes():
    assert pa.pa_int8_block_bytes(8, 128, 16) == 8 * 2112
    assert pa.pa_int8_block_bytes(8, 128, 64) == 8 * 4 * 2112
    assert pa.pa_int8_block_bytes(8, 64, 16) == 0
    assert pa.pa_int8_block_bytes(8, 128, 8) == 0


def _prefill_args(**kw):
    p = C.c_void_p(16)
    args = dict(out=p, q=p, kc=p, vc=p, bt=p, ctx=p, qs=p, B=4, Hq=8, Hkv=2, D=128, bs=16, NB=10,
                MB=4, T=8, max_q=4, scale=0.1, dtype=pa.PA_F16, err=None, ws=None,
                path=pa.PA_PREFILL_AUTO, stream=None)
    args.update(kw)
    return args


def _call_prefill(a):
    return pa.lib.pa_prefill_attention_ex(
        a["out"], a["q"], a["kc"], a["vc"], a["bt"], a["ctx"], a["qs"], a["B"], a["Hq"], a["Hkv"],
        a["D"], a["bs"], a["NB"], a["MB"], a["T"], a["max_q"], a["scale"], a["dtype"], a["err"],
        a["ws"], a["path"], a["stream"])


@pytest.mark.parametrize("bad", [
    dict(path=4), dict(path=-1), dict(dtype=pa.PA_F32), dict(T=-1), dict(B=-1), dict(B=70000),
    dict(Hkv=0), dict(Hq=7), dict(Hq=256, Hkv=2), dict(D=96), dict(bs=8), dict(bs=24),
    dict(NB=-1), dict(max_q=1 << 30), dict(scale=float("nan")), dict(kc=None),
    dict(q=C.c_void_p(2)), dict(kc=C.c_void_p(8)), dict(ws=C.c_void_p(4)),
    # the tcgen05 kernel asked for where it does not apply
    dict(path=pa.PA_PREFILL_TCGEN05, D=64), dict(path=pa.PA_PREFILL_TCGEN05, scale=-1.0),
    dict(path=pa.PA_PREFILL_TCGEN05, q=C.c_void_p(20)),
    dict(path=pa.PA_PREFILL_TCGEN05, out=C.c_void_p(36)),
    dict(path=pa.PA_PREFILL_TCGEN05_PAIR, D=64), dict(path=pa.PA_PREFILL_TCGEN05_PAIR, Hq=256,
                                                       Hkv=1),
])
def test_prefill_rejects_bad_arguments_on_host(bad):
    """Every limit pa.h states for pa_prefill_attention_ex is checked before anything
    reaches the device: PA_ERR_INVALID with a message, nothing launched."""
    st = _call_prefill(_prefill_args(**bad))
    assert st == pa.PA_ERR_INVALID, pa.pa_last_error()
    assert pa.pa_last_error()


def test_prefill_empty_calls_are_no_ops():
    assert _call_prefill(_prefill_args(B=0, q=None, out=None)) == pa.PA_OK
    assert _call_prefill(_prefill_args(max_q=0)) == pa.PA_OK
    assert _call_prefill(_prefill_args(T=0)) == pa.PA_OK
