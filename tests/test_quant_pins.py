"""Pins of the oracle's KV quantisation ("vladkulikov.com modern-llms module 9
notebook", KV quantisation experiment): the page's own checks (int8 keeps the
attention output within 3 % relative error; an all-zero row stays zero), a
worked row with round-half-even ties, exact rational arithmetic on small rows,
and the bounds that any per-row absmax code must meet."""
from fractions import Fraction

import numpy as np

from oracle import attention_two_pass, dequantize_rows, fake_quantize_rows, quantize_rows, stored_rows


def _attn(q, k, v):
    # each query as one decode step (q_tokens = 1, one head) over all n keys
    return np.stack([attention_two_pass(qi[None, None, :], k[:, None, :], v[:, None, :])[0, 0]
                     for qi in q])


def test_page_relative_error_bound_int8():
    rng = np.random.default_rng(20260810)
    n, d = 128, 32
    keys, values = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    queries = rng.normal(size=(12, d))
    ref = _attn(queries, keys, values)
    err = {}
    for bits in (8, 3):
        out = _attn(queries, fake_quantize_rows(keys, bits), fake_quantize_rows(values, bits))
        err[bits] = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert err[8] < 0.03
    assert err[3] > err[8]                      # fewer bits, larger error


def test_page_zero_rows_stay_zero():
    assert np.array_equal(fake_quantize_rows(np.zeros((2, 4)), 3), np.zeros((2, 4)))
    codes, scale = quantize_rows(np.zeros((3, 5)))
    assert np.all(codes == 0) and np.all(scale == 1.0)


def test_worked_row_half_even():
    codes, scale = quantize_rows(np.array([[127.0, 2.5, -3.5, 0.5, -0.5, 1.5, -127.0]]))
    assert scale.tolist() == [1.0]
    assert codes.tolist() == [[127, 2, -4, 0, 0, 2, -127]]
    codes3, scale3 = quantize_rows(np.array([[6.0, 1.0, -4.5]]), bits=3)   # limit 3
    assert scale3.tolist() == [2.0] and codes3.tolist() == [[3, 0, -2]]


def _exact_codes(row, limit):
    amax = max(abs(Fraction(float(x))) for x in row)
    scale = amax / limit if amax else Fraction(1)
    out = []
    for x in row:
        t = Fraction(float(x)) / scale
        f = t.numerator // t.denominator
        r = t - f
        k = f + (1 if r > Fraction(1, 2) or (r == Fraction(1, 2) and f % 2) else 0)
        out.append(max(-limit, min(limit, k)))
    return out, scale


def test_codes_equal_exact_rational_arithmetic():
    rng = np.random.default_rng(5)
    for bits in (8, 4, 3):
        limit = 2 ** (bits - 1) - 1
        x = rng.normal(size=(200, 16)) * rng.choice([1e-3, 1.0, 300.0], size=(200, 1))
        codes, scale = quantize_rows(x, bits)
        for i in range(x.shape[0]):
            want, s = _exact_codes(x[i], limit)
            assert codes[i].tolist() == want
            assert abs(scale[i] - float(s)) <= 1e-15 * float(s)


def test_bounds_of_absmax_codes():
    rng = np.random.default_rng(6)
    x = rng.normal(size=(500, 128)) * rng.uniform(0.01, 50, size=(500, 1))
    codes, scale = quantize_rows(x)
    assert np.all(np.abs(codes).max(axis=1) == 127)          # the absmax element hits the limit
    am = np.abs(x).argmax(axis=1)
    assert np.all(np.sign(codes[np.arange(500), am]) == np.sign(x[np.arange(500), am]))
    err = np.abs(dequantize_rows(codes, scale) - x)
    assert np.all(err <= scale[:, None] / 2 * (1 + 1e-12))   # half a step at most


def test_stored_rows_use_float32_scale():
    rng = np.random.default_rng(7)
    x = rng.normal(size=(10, 128)).astype(np.float32).astype(np.float64)
    codes, s32, back = stored_rows(x)
    c64, s64 = quantize_rows(x)
    assert np.array_equal(codes, c64)
    assert s32.dtype == np.float32 and np.array_equal(s32, s64.astype(np.float32))
    assert np.array_equal(back, codes.astype(np.float64) * s32.astype(np.float64)[:, None])


# ------------------------------------------------------------- FP8 E4M3 ----
# The pages quantise to integers; the FP8 pool keeps their per-row absmax
# recipe on the E4M3 grid of the OCP 8-bit floating point specification.  The
# grid is pinned by the format's closed forms, the rounding by torch's own
# float8_e4m3fn cast (a library routine) and by exact rational arithmetic.
import torch  # noqa: E402

from oracle.quant import (  # noqa: E402
    E4M3_MAX, dequantize_rows_fp8, e4m3_round, e4m3_values, quantize_rows_fp8, stored_rows_fp8)


def test_e4m3_table_closed_forms():
    v = e4m3_values()
    want = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
            0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}
    for code, val in want.items():
        assert v[code] == val, hex(code)
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and np.signbit(v[0x80]) and v[0x80] == 0
    assert np.count_nonzero(np.isfinite(v)) == 254
    assert np.all(np.diff(v[:127]) > 0)                      # codes 0x00 .. 0x7E increase
    assert np.array_equal(v[0x80:0xFF], -v[:127])             # sign bit only flips the sign


def test_e4m3_round_matches_torch_cast():
    rng = np.random.default_rng(7)
    grid = e4m3_values()[:127]
    mids = (grid[1:] + grid[:-1]) / 2                       # every exact tie
    y = np.concatenate([rng.uniform(-E4M3_MAX, E4M3_MAX, 20000),
                        rng.normal(size=20000) * rng.choice([1e-3, 1e-2, 1.0, 30.0], 20000),
                        mids, -mids, grid, -grid]).astype(np.float32)
    y = np.clip(y, -E4M3_MAX, E4M3_MAX)
    assert np.array_equal(mids.astype(np.float32).astype(np.float64), mids)   # ties exact
    lib = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    lib = np.where((lib & 0x7F) == 0, 0, lib)                # zero is stored as +0
    assert np.array_equal(e4m3_round(y.astype(np.float64)), lib)


def test_e4m3_worked_ties_go_to_even():
    ties = {1.0625: 0x38, 1.1875: 0x3A, 2.0 ** -10: 0x00, 3 * 2.0 ** -10: 0x02,
            432.0: 0x7E, 400.0: 0x7C, -1.0625: 0xB8, -(2.0 ** -11): 0x00}
    for y, code in ties.items():
        assert int(e4m3_round(np.array(y))) == code, y
    codes = np.arange(127, dtype=np.uint8)
    assert np.array_equal(e4m3_round(e4m3_values()[:127]), codes)       # round trip


def _exact_e4m3(t):
    """Nearest E4M3 value to the rational t (|t| <= 448), ties to the even code."""
    grid = [Fraction(float(g)) for g in e4m3_values()[:127]]
    a = abs(t)
    best = min(range(127), key=lambda c: (abs(grid[c] - a), c % 2))
    return 0 if best == 0 else (best | (0x80 if t < 0 else 0))


def test_fp8_codes_equal_exact_rational_arithmetic():
    rng = np.random.default_rng(11)
    for _ in range(40):
        row = (rng.normal(size=16) * rng.choice([1e-3, 1.0, 50.0])).astype(np.float32)
        row[rng.integers(16)] = 0.0
        codes, scale = quantize_rows_fp8(row[None].astype(np.float64))
        amax = max(abs(Fraction(float(x))) for x in row)
        for x, c in zip(row, codes[0]):
            assert int(c) == _exact_e4m3(Fraction(float(x)) * E4M3_MAX / amax)


def test_fp8_rows_bounds_and_special_rows():
    rng = np.random.default_rng(12)
    x = rng.normal(size=(200, 128)) * rng.uniform(1e-3, 1e3, size=(200, 1))
    codes, scale = quantize_rows_fp8(x)
    assert np.all(np.abs(codes[np.arange(200), np.abs(x).argmax(axis=1)].astype(int) & 0x7F) == 0x7E)
    y = dequantize_rows_fp8(codes, scale)
    t = np.abs(x / scale[:, None])
    normal = t >= 2.0 ** -6
    assert np.all(np.abs(y - x)[normal] <= 2.0 ** -4 * np.abs(x)[normal] * (1 + 1e-12))
    sub = ~normal
    assert np.all(np.abs(y - x)[sub] <= 2.0 ** -10 * np.broadcast_to(scale[:, None], x.shape)[sub]
                  * (1 + 1e-12))
    z, zs = quantize_rows_fp8(np.zeros((3, 8)))
    assert np.all(z == 0) and np.all(zs == 1.0)
    neg = quantize_rows_fp8(-np.abs(x))[0]
    assert np.array_equal(neg, np.where(codes & 0x7F, (codes & 0x7F) | 0x80, 0))


def test_fp8_stored_rows_use_float32_scales():
    rng = np.random.default_rng(13)
    x = rng.normal(size=(5, 128)) * 3.3
    codes, s32, val = stored_rows_fp8(x)
    assert s32.dtype == np.float32
    assert np.array_equal(codes, quantize_rows_fp8(x)[0])
    assert np.array_equal(val, e4m3_values()[codes] * s32.astype(np.float64)[:, None])


def test_page_experiment_fp8_between_int8_and_int3():
    # the page's experiment with the E4M3 grid: 3 mantissa bits put FP8 between
    # the 8-bit and 3-bit integer codes (it does not meet the 3 % int8 bound)
    rng = np.random.default_rng(20260810)
    n, d = 128, 32
    keys, values = rng.normal(size=(n, d)), rng.normal(size=(n, d))
    queries = rng.normal(size=(12, d))
    ref = _attn(queries, keys, values)
    rel = lambda out: np.linalg.norm(out - ref) / np.linalg.norm(ref)   # noqa: E731
    fq = lambda x: dequantize_rows_fp8(*quantize_rows_fp8(x))           # noqa: E731
    e8 = rel(_attn(queries, fake_quantize_rows(keys, 8), fake_quantize_rows(values, 8)))
    e3 = rel(_attn(queries, fake_quantize_rows(keys, 3), fake_quantize_rows(values, 3)))
    ef = rel(_attn(queries, fq(keys), fq(values)))
    assert e8 < ef < e3 and ef < 2.0 ** -4
