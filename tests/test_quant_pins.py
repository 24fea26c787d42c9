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
