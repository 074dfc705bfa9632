"""Pins the oracle's number-format conversions to library routines (numpy fp16,
torch bf16) and to exact midpoint cases."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def test_f16_decode_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(b) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_decode_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_to_f64(b) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def _f16_cases(rng):
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0,
        rng.standard_normal(5000) * 1e-5,              # subnormal range
        rng.uniform(6.0e4, 7.0e4, 2000),               # around the overflow threshold
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 2.0 ** -24, 2.0 ** -25,
                  2.0 ** -25 * 1.0000001, 3 * 2.0 ** -26]),
    ])
    # exact midpoints between neighbouring fp16 values: ties must go to even
    h = rng.integers(0, 0x7bff, 5000).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    return np.concatenate([x, (lo + hi) / 2, -(lo + hi) / 2])


def test_f64_to_f16_matches_numpy_rounding():
    x = _f16_cases(np.random.default_rng(0))
    ref = x.astype(np.float16).view(np.uint16)
    got = oracle.round_to(x, "f16")
    assert np.array_equal(got, ref)


def test_f64_to_bf16_matches_torch_rounding_on_fp32_values():
    rng = np.random.default_rng(1)
    x32 = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 7,
        rng.standard_normal(2000).astype(np.float32) * np.float32(1e-39),  # subnormals
        np.array([3.3895314e38, 3.39e38, 1e-45, 0.0], dtype=np.float32),
    ])
    # exact midpoints between neighbouring bf16 values (representable in fp32)
    b = rng.integers(0, 0x7f7f, 5000).astype(np.uint16)
    lo = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).float()
    hi = torch.from_numpy((b + 1).view(np.int16)).view(torch.bfloat16).float()
    mid = ((lo.double() + hi.double()) / 2).float().numpy()
    x32 = np.concatenate([x32, mid, -mid])
    ref = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.round_to(x32.astype(np.float64), "bf16")
    assert np.array_equal(got, ref)


def test_round_trip_is_identity():
    bits = np.arange(0, 0x7c00, dtype=np.uint16)  # every finite non-negative fp16
    vals = bits.view(np.float16).astype(np.float64)
    assert np.array_equal(oracle.round_to(vals, "f16"), bits)
    bb = np.arange(0, 0x7f80, dtype=np.uint16)
    bvals = torch.from_numpy(bb.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.round_to(bvals, "bf16"), bb)
