"""e4m3 ("fn" variant) rounding and the per-row activation quantisation of the W8A8 path.

Test infrastructure only (see the package docstring).

Source: the FFN service of the vLLM AFD plugin is benchmarked on DeepSeek-V3.2 W8A8
(vLLM AFD Plugin page, section 效能基準測試 / 同步 Decode 吞吐量).  The pages fix no
format details; the reading used here is e4m3 "fn" (bias 7, no infinities, largest finite
magnitude 448, NaN only for the all-ones exponent-and-mantissa code), round to nearest even,
saturating to +-448, with one fp32 scale per row equal to amax/448 (1 when the row is zero).

Where these roundings decide a stored code, the decision is taken in fp32 -- the precision
of the GPU kernel: the scale is an fp32 quotient and each element is the fp32 quotient
x / scale before it is rounded to e4m3.

Pins (tests/test_oracle_fp8.py): every one of the 256 codes decodes to the value two
independent implementations give (ml_dtypes.float8_e4m3fn and torch.float8_e4m3fn) and
re-encodes to itself; a few codes are checked by hand (1, 448, the smallest normal and
subnormal, -2, NaN); exact midpoints round to the even code; values past 448 saturate;
random fp32 values match ml_dtypes wherever it is in range.  quantize_rows is checked against
torch's own fp32 quotients and e4m3 conversion, and on rows whose fp32 quotient lands exactly
on a rounding midpoint, so that an fp64 scale would give a different code.  The quantisation
points of the W8A8 layer (hidden row, SwiGLU row) are pinned by a hand-worked expert and a
scalar-loop layer (tests/test_oracle_expert.py::test_w8a8_worked_example and
::test_w8a8_forward_against_scalar_loops).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
_MIN_NORMAL_EXP = -6          # smallest normal: 2**-6
_SUBNORMAL_STEP = 2.0 ** -9   # spacing of the subnormals (mantissa 3 bits)


def e4m3_decode(codes) -> np.ndarray:
    """Value of each 8-bit code as float64 (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * (1.0 + m / 8.0) * np.exp2(ef.astype(np.float64) - 7.0)
    sub = sign * (m / 8.0) * 2.0 ** _MIN_NORMAL_EXP
    v = np.where(ef == 0, sub, normal)
    return np.where((ef == 0xF) & (m == 0x7), np.nan, v)


def e4m3_round(x) -> np.ndarray:
    """Round values to the nearest e4m3 value (ties to even), saturating at +-448.

    Works in float64, where every fp32 input and every scaling by a power of two is exact,
    so the result is the correctly rounded e4m3 value of the input.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    out = np.empty_like(a)
    # normal range: a = s * 2**e with s in [1, 2)
    with np.errstate(divide="ignore", invalid="ignore"):
        frac, ex = np.frexp(a)                       # a = frac * 2**ex, frac in [0.5, 1)
    e = ex.astype(np.int64) - 1
    is_normal = a >= 2.0 ** _MIN_NORMAL_EXP
    s = np.where(is_normal, frac * 2.0, 0.0)          # significand in [1, 2)
    q = np.rint(s * 8.0) / 8.0                        # 3 mantissa bits, half to even
    normal_val = q * np.exp2(e.astype(np.float64))
    # subnormal range: multiples of 2**-9 (rounding up may reach 2**-6, the smallest normal)
    sub_val = np.rint(a / _SUBNORMAL_STEP) * _SUBNORMAL_STEP
    out = np.where(is_normal, normal_val, sub_val)
    out = np.minimum(out, E4M3_MAX)                   # satfinite
    out = np.where(np.isnan(x), np.nan, out)
    return np.copysign(out, x)


def e4m3_encode(x) -> np.ndarray:
    """8-bit code of the e4m3 rounding of each value (NaN -> 0x7F)."""
    v = e4m3_round(x)
    a = np.abs(v)
    sign = np.signbit(v).astype(np.int64) << 7
    code = np.zeros(a.shape, dtype=np.int64)
    sub = a < 2.0 ** _MIN_NORMAL_EXP
    code = np.where(sub, np.rint(a / _SUBNORMAL_STEP).astype(np.int64), code)
    with np.errstate(divide="ignore", invalid="ignore"):
        frac, ex = np.frexp(np.where(sub, 1.0, a))
    ef = ex.astype(np.int64) - 1 + 7
    m = np.rint((frac * 2.0 - 1.0) * 8.0).astype(np.int64)
    code = np.where(sub, code, (ef << 3) | m)
    code = np.where(np.isnan(v), 0x7F, code | sign)
    return code.astype(np.uint8)


def quantize_rows(x32):
    """Per-row e4m3 quantisation of an fp32 matrix, decisions taken in fp32.

    scale_r = fp32(amax_r / 448) (1 when the row is all zero); q = e4m3(fp32(x / scale_r)).
    Returns (q values as float64, scale as float32); the dequantised row is q * scale.
    """
    x32 = np.asarray(x32, dtype=np.float32)
    amax = np.abs(x32).max(axis=1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    y32 = (x32 / scale[:, None]).astype(np.float32)   # IEEE fp32 quotient
    return e4m3_round(y32), scale
