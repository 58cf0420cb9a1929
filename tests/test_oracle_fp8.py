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


def _torch_fp32_quantize(x32):
    """The same per-row quantisation evaluated by torch: fp32 amax, fp32 quotient amax / 448,
    fp32 quotient x / scale, then torch's own float8_e4m3fn conversion (round to nearest even)."""
    x = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32))
    amax = x.abs().amax(dim=1)
    s = torch.where(amax > 0, amax / torch.tensor(448.0, dtype=torch.float32), torch.ones_like(amax))
    q = (x / s[:, None]).to(torch.float8_e4m3fn).to(torch.float64)
    return q.numpy(), s.numpy()


def test_quantize_rows_matches_torch_fp32_path():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((64, 257)) * rng.choice([1e-4, 1e-2, 1.0, 50.0, 3e4], (64, 1))).astype(np.float32)
    x[5] = 0.0                                          # zero row: scale 1, codes 0
    x[9] = 0.0
    x[9, 100] = -3.0                                    # one non-zero: it maps to -448
    q, s = fp8.quantize_rows(x)
    qt, st = _torch_fp32_quantize(x)
    assert np.array_equal(s, st)
    assert np.array_equal(q, qt)


# Rows whose fp32 quotient x / scale lands exactly on an e4m3 rounding midpoint, so that the
# precision of the scale decides the code (the W8A8 reading: scale and quotient are fp32):
#   amax = 0x1.143802p-1, scale = fp32(amax / 448) = 0x1.3badbap-10 (above the exact quotient),
#   x = 0x1.4f6896p-6: fp32(x / scale) = 17.0 exactly, the midpoint of 16 and 18; ties to even
#   give 16.  With an fp64 scale and quotient, x / (amax / 448) = 17.000000994..., which gives 18.
#   amax = 0x1.9e97e4p+2, x = 0x1.f76f4ep-1: fp32(x / scale) = 68.0 exactly, the midpoint of 64
#   and 72 -> 64 (an fp64 scale gives 68.0000047... -> 72).
FP32_TIE_ROWS = [
    (float.fromhex("0x1.143802p-1"), float.fromhex("0x1.4f6896p-6"), 16.0),
    (float.fromhex("0x1.9e97e4p+2"), float.fromhex("0x1.f76f4ep-1"), 64.0),
]


def test_quantize_rows_scale_and_quotient_are_fp32():
    x = np.array([[a, v] for a, v, _ in FP32_TIE_ROWS], dtype=np.float32)
    q, s = fp8.quantize_rows(x)
    assert s[0] == np.float32(float.fromhex("0x1.3badbap-10"))
    for r, (_, _, code) in enumerate(FP32_TIE_ROWS):
        assert q[r, 0] == 448.0
        assert q[r, 1] == code
    qt, st = _torch_fp32_quantize(x)
    assert np.array_equal(q, qt) and np.array_equal(s, st)
