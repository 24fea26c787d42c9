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
    """Codes (int8) and float64 scales (one per row of the last axis)."""
    limit = float(2 ** (bits - 1) - 1)
    x = np.asarray(x, dtype=np.float64)
    scale = np.abs(x).max(axis=-1) / limit
    scale = np.where(scale == 0.0, 1.0, scale)
    q = np.rint(x / scale[..., None])
    codes = np.minimum(np.maximum(q, -limit), limit).astype(np.int8)
    return codes, scale


def dequantize_rows(codes, scale):
    """code * scale, float64."""
    return np.asarray(codes, dtype=np.float64) * np.asarray(scale, dtype=np.float64)[..., None]


def fake_quantize_rows(x, bits=8):
    """The page's round trip, float64 scales."""
    codes, scale = quantize_rows(x, bits)
    return dequantize_rows(codes, scale)


def stored_rows(x):
    """A row as an int8 pool holds it: (codes, float32 scale, value read back)."""
    codes, scale = quantize_rows(x, 8)
    s32 = scale.astype(np.float32)
    return codes, s32, dequantize_rows(codes, s32.astype(np.float64))
