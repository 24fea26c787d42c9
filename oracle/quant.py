"""Oracle KV quantisation: per-row absmax integer codes.

Test infrastructure only (see the package header).  Restates the KV
quantisation experiment of "vladkulikov.com modern-llms module 9 notebook"
(``fake_quantize_rows``): for a row x and ``bits`` bits, limit = 2^(bits-1) - 1,
scale = max|x| / limit (a zero row takes scale 1), code = round-half-even of
x / scale clipped to [-limit, limit], value = code * scale.  Everything is
float64, as on the page.

Reading taken for a stored pool (the page dequantises in float64 and counts
4-byte scales in its byte model): the codes are decided in float64 exactly as
above; the pool stores each row's scale as float32 (round to nearest), and a
row is read back as code * float64(float32(scale)).
"""
from __future__ import annotations

import numpy as np


def quantize_rows(x, bits=8):
    """Codes (int8) and float64 scales (one per row of the last axis), as
    "vladkulikov.com modern-llms module 9 notebook"'s ``fake_quantize_rows`` decides them."""
    limit = float(2 ** (bits - 1) - 1)
    x = np.asarray(x, dtype=np.float64)
    scale = np.abs(x).max(axis=-1) / limit
    scale = np.where(scale == 0.0, 1.0, scale)
    q = np.rint(x / scale[..., None])
    codes = np.minimum(np.maximum(q, -limit), limit).astype(np.int8)
    return codes, scale


def dequantize_rows(codes, scale):
    """code * scale, float64 ("vladkulikov.com modern-llms module 9 notebook", ``fake_quantize_rows``)."""
    return np.asarray(codes, dtype=np.float64) * np.asarray(scale, dtype=np.float64)[..., None]


def fake_quantize_rows(x, bits=8):
    """The page's round trip, float64 scales."""
    codes, scale = quantize_rows(x, bits)
    return dequantize_rows(codes, scale)


def stored_rows(x):
    """A row as an int8 pool holds it: (codes, float32 scale, value read back);
    the float32 scale is the reading stated in the module header."""
    codes, scale = quantize_rows(x, 8)
    s32 = scale.astype(np.float32)
    return codes, s32, dequantize_rows(codes, s32.astype(np.float64))


# ---------------------------------------------------------------- FP8 E4M3 --
# The KV rows may also be stored as 8-bit floats instead of integers.  The
# pages quantise to an integer grid only; the reading taken here keeps the
# page's per-row absmax recipe and swaps the grid for the E4M3 format of the
# OCP 8-bit floating point specification: 1 sign bit, 4 exponent bits with
# bias 7, 3 mantissa bits, subnormals, no infinities, and S.1111.111 as NaN,
# so the largest finite magnitude is 448.  For a row x: scale = max|x| / 448
# (a zero row takes scale 1), each code is the E4M3 value nearest to
# x / scale (ties to the even code, i.e. the even mantissa), decided in
# float64.  A result of magnitude zero is stored as +0 (code 0x00).  As for
# the integer codes, the pool keeps the scale as float32.

E4M3_MAX = 448.0


def e4m3_values():
    """Value of each of the 256 codes (NaN for 0x7F and 0xFF), float64,
    straight from the format definition (the E4M3 format of the OCP 8-bit floating point specification)."""
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        s, e, m = code >> 7, (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            v = np.nan
        elif e == 0:
            v = (m / 8.0) * 2.0 ** (1 - 7)        # subnormal: 0.m x 2^(1 - bias)
        else:
            v = (1.0 + m / 8.0) * 2.0 ** (e - 7)
        vals[code] = -v if s else v
    return vals


def e4m3_round(y):
    """Codes (uint8) of the E4M3 values nearest to y (|y| <= 448), ties to the
    even code; magnitude zero gives 0x00 (round to nearest even on the E4M3 format of the OCP 8-bit floating point specification)."""
    y = np.asarray(y, dtype=np.float64)
    if np.any(np.abs(y) > E4M3_MAX) or np.any(np.isnan(y)):
        raise ValueError("e4m3_round: |y| must be <= 448")
    grid = e4m3_values()[:127]                 # codes 0x00 .. 0x7E, increasing
    a = np.abs(y).ravel()
    hi = np.searchsorted(grid, a, side="left")  # first grid value >= a
    hi = np.minimum(hi, 126)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - grid[lo], grid[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag = np.where(pick_hi, hi, lo).astype(np.uint8)
    neg = (y.ravel() < 0) & (mag != 0)
    return (mag | np.where(neg, 0x80, 0).astype(np.uint8)).reshape(y.shape)


def quantize_rows_fp8(x):
    """E4M3 codes (uint8 bit patterns) and float64 scales, one per row: the
    per-row recipe of "vladkulikov.com modern-llms module 9 notebook"'s ``fake_quantize_rows`` on the E4M3 format of the OCP 8-bit floating point specification (a reading)."""
    x = np.asarray(x, dtype=np.float64)
    scale = np.abs(x).max(axis=-1) / E4M3_MAX
    scale = np.where(scale == 0.0, 1.0, scale)
    y = np.clip(x / scale[..., None], -E4M3_MAX, E4M3_MAX)
    return e4m3_round(y), scale


def dequantize_rows_fp8(codes, scale):
    """value(code) * scale, float64 (the E4M3 format of the OCP 8-bit floating point specification)."""
    return e4m3_values()[np.asarray(codes, dtype=np.uint8)] * \
        np.asarray(scale, dtype=np.float64)[..., None]


def stored_rows_fp8(x):
    """A row as an FP8 pool holds it: (codes, float32 scale, value read back);
    the float32 scale as for the int8 pool."""
    codes, scale = quantize_rows_fp8(x)
    s32 = scale.astype(np.float32)
    return codes, s32, dequantize_rows_fp8(codes, s32.astype(np.float64))
