"""Software rounding to bf16, fp32, FP8 e4m3, FP4 e2m1 and ue4m3 (oracle).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

All rounding is round-to-nearest-even on fp64 values.  A value is rounded to a
format by finding its quantum (the spacing of the format's grid in the binade
of the value, or the subnormal spacing below the smallest normal), dividing by
it (exact: the quantum is a power of two), rounding to the nearest integer with
ties to even (``np.rint``) and multiplying back (exact).  "satfinite" clamps
the magnitude to the largest finite value of the format.

Formats, as used for NVFP4 and FP8 attention in "Triage" (zhuanzhiai paper
page, abstract: NVFP4 tiles on FP4 tensor cores):

* e4m3 (OCP FP8 E4M3FN): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits,
  no infinities, NaN only at S.1111.111; max finite 448, min normal 2^-6,
  subnormal spacing 2^-9.
* e2m1 (FP4): 1 sign, 2 exponent bits (bias 1), 1 mantissa bit; values
  {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
* ue4m3: the e4m3 grid restricted to non-negative values (NVFP4 block scale).
* bf16: 8 exponent bits, 7 mantissa bits; fp32: IEEE binary32.

Codes are returned as uint8 (an FP4 code in the low nibble, sign in bit 3).  A
negative value that rounds to zero keeps its sign bit (IEEE signed zero).
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0
_E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _floor_log2(a: np.ndarray) -> np.ndarray:
    """floor(log2(a)) for a > 0, exactly (from the binary exponent)."""
    _, e = np.frexp(a)
    return e.astype(np.int64) - 1


def _round_grid(x, min_exp: int, mant_bits: int, max_val: float):
    """RNE onto a binary grid with ``mant_bits`` explicit mantissa bits whose
    smallest normal exponent is ``min_exp``; magnitudes clamp to ``max_val``."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.maximum(_floor_log2(np.where(a > 0, a, 1.0)), min_exp)
    q = np.ldexp(1.0, (e - mant_bits).astype(np.int64))
    r = np.rint(a / q) * q
    r = np.minimum(r, max_val)
    return np.copysign(r, x)


def bf16_rne(x):
    """Round fp64 values to the nearest bf16 value (ties to even), returned as fp64."""
    return _round_grid(x, -126, 7, np.inf)


def fp32_rne(x):
    """Round fp64 values to the nearest IEEE binary32 value, returned as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def e4m3_round(x):
    """Value of e4m3 RNE satfinite rounding."""
    return _round_grid(x, -6, 3, E4M3_MAX)


def e4m3_encode(x) -> np.ndarray:
    """e4m3 code (uint8) of RNE satfinite rounding of x."""
    x = np.asarray(x, dtype=np.float64)
    r = np.abs(e4m3_round(x))
    sub = r < 2.0 ** -6
    with np.errstate(divide="ignore"):
        e = _floor_log2(np.where(sub, 1.0, r))
    mant_n = (r / np.ldexp(1.0, e) - 1.0) * 8.0
    code_n = ((e + 7) << 3) + np.rint(mant_n).astype(np.int64)
    code_s = np.rint(r / 2.0 ** -9).astype(np.int64)
    code = np.where(sub, code_s, code_n)
    code = code | (np.signbit(x).astype(np.int64) << 7)
    return code.astype(np.uint8)


def e4m3_decode(code) -> np.ndarray:
    """fp64 value of e4m3 codes (NaN codes S.1111.111 decode to NaN)."""
    c = np.asarray(code, dtype=np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(ef == 0, m * 2.0 ** -9, np.ldexp(1.0 + m / 8.0, ef - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return s * val


def e2m1_round(x):
    """Value of e2m1 RNE satfinite rounding."""
    return _round_grid(x, 0, 1, E2M1_MAX)


def e2m1_encode(x) -> np.ndarray:
    """e2m1 code (uint8, low nibble) of RNE satfinite rounding of x."""
    x = np.asarray(x, dtype=np.float64)
    r = np.abs(e2m1_round(x))
    mag = np.searchsorted(_E2M1_GRID, r)
    return (mag | (np.signbit(x).astype(np.int64) << 3)).astype(np.uint8)


def e2m1_decode(code) -> np.ndarray:
    c = np.asarray(code, dtype=np.int64)
    return np.where(c & 0x8, -1.0, 1.0) * _E2M1_GRID[c & 0x7]


def ue4m3_encode(x) -> np.ndarray:
    """Unsigned e4m3 code of x >= 0 (RNE satfinite)."""
    x = np.asarray(x, dtype=np.float64)
    if np.any(x < 0):
        raise ValueError("ue4m3 takes non-negative values")
    return e4m3_encode(x)


def ue4m3_decode(code) -> np.ndarray:
    return e4m3_decode(np.asarray(code, dtype=np.int64) & 0x7F)
