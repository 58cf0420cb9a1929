"""Pins of the oracle's e4m3 rounding and per-row quantisation (CPU only).

The serving benchmark runs DeepSeek-V3.2 W8A8 (vLLM AFD Plugin, 效能基準測試); the format
reading (e4m3 "fn", round to nearest even, saturating) is pinned here against two
independent library implementations (ml_dtypes and torch) and against hand-checked codes.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import fp8

ALL_CODES = np.arange(256, dtype=np.uint8)


def test_all_codes_match_ml_dtypes_and_torch():
    mine = fp8.e4m3_decode(ALL_CODES)
    lib = ALL_CODES.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    tch = torch.from_numpy(ALL_CODES.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2
    assert np.array_equal(mine[~nan], lib[~nan])
    assert np.array_equal(mine[~nan], tch[~nan])


def test_hand_checked_codes():
    assert fp8.e4m3_decode([0x38])[0] == 1.0            # exponent field 7 = bias, mantissa 0
    assert fp8.e4m3_decode([0x7E])[0] == 448.0          # 2^8 * 1.75, the largest finite
    assert fp8.e4m3_decode([0x08])[0] == 2.0 ** -6      # smallest normal
    assert fp8.e4m3_decode([0x01])[0] == 2.0 ** -9      # smallest subnormal
    assert fp8.e4m3_decode([0xC0])[0] == -2.0
    assert np.isnan(fp8.e4m3_decode([0x7F])[0])


def test_every_code_round_trips():
    vals = fp8.e4m3_decode(ALL_CODES)
    ok = ~np.isnan(vals)
    codes = fp8.e4m3_encode(vals[ok])
    # +0 and -0 keep their sign bit
    assert np.array_equal(codes, ALL_CODES[ok])
    assert np.array_equal(fp8.e4m3_round(vals[ok]), vals[ok])


def test_ties_to_even_and_saturation():
    # between 1.0 (mantissa 0) and 1.125 (mantissa 1): the midpoint goes to the even code
    assert fp8.e4m3_round(1.0625) == 1.0
    # between 1.125 (m=1) and 1.25 (m=2): midpoint 1.1875 goes to 1.25
    assert fp8.e4m3_round(1.1875) == 1.25
    # just above the midpoint rounds up
    assert fp8.e4m3_round(np.nextafter(1.0625, 2.0)) == 1.125
    # subnormal midpoint between 0 and 2^-9 goes to 0, between 2^-9 and 2^-8 to 2^-8
    assert fp8.e4m3_round(2.0 ** -10) == 0.0
    assert fp8.e4m3_round(3 * 2.0 ** -10) == 2.0 ** -8
    # saturating: past 448 stays 448 (no NaN, no inf)
    for v in [448.0, 463.9, 464.0, 500.0, 1e30, np.inf]:
        assert fp8.e4m3_round(v) == 448.0
        assert fp8.e4m3_round(-v) == -448.0


def test_random_values_match_ml_dtypes_in_range():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * rng.choice([1e-3, 1e-1, 1, 30, 200], 200000)).astype(np.float32)
    x = x[np.abs(x) <= 448]
    lib = x.astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(fp8.e4m3_round(x), lib)


def test_quantize_rows_properties():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((50, 300)).astype(np.float32)
    x[3] = 0.0
    q, s = fp8.quantize_rows(x)
    amax = np.abs(x).max(axis=1)
    assert s.dtype == np.float32
    assert np.array_equal(s[amax > 0], (amax[amax > 0] / np.float32(448)).astype(np.float32))
    assert s[3] == 1.0 and np.all(q[3] == 0)
    assert np.all(np.abs(q) <= 448)
    # the largest element of each row lands on (or next to) the largest code
    assert np.all(np.abs(q[amax > 0]).max(axis=1) >= 416)
    # dequantised rows are within half an e4m3 step (relative 2^-4) of the input
    deq = q * s[:, None].astype(np.float64)
    err = np.abs(deq - x)
    assert np.all(err <= np.maximum(np.abs(x) * 2.0 ** -4, s[:, None] * 2.0 ** -10) + 1e-12)
