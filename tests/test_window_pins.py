"""Pins of the oracle's sink + recent window ("vladkulikov.com modern-llms
module 9 notebook": ``streaming_keep_indices`` and its reference value for
16 tokens, budget 8, 4 sinks; the window-3 sliding cache) and of windowed
decode attention against attention over the explicit slice."""
import json
import os

import numpy as np
import pytest

from oracle import attention_two_pass, attention_window, visible_positions

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "p2_streaming.json")


def test_page_streaming_reference_value():
    g = json.load(open(GOLDEN))
    n, budget, sinks = g["length"], g["budget"], g["sink_tokens"]
    assert visible_positions(n, budget - sinks, sinks) == g["streaming"]


def test_page_window3_cache_keeps_last_three():
    # five appends into a window-3 cache leave positions 2, 3, 4 (start 2, next 5)
    assert visible_positions(5, 3) == [2, 3, 4]
    assert visible_positions(2, 3) == [0, 1]


def test_short_sequences_keep_everything():
    for n in range(0, 9):
        assert visible_positions(n, 5, 3) == list(range(n))


def test_overlap_and_bounds():
    assert visible_positions(10, 4, 8) == list(range(10))        # sinks reach the window
    assert visible_positions(20, 1, 0) == [19]
    assert visible_positions(20, 1, 2) == [0, 1, 19]
    for n in (0, 7, 100):
        assert len(visible_positions(n, 6, 2)) == min(n, 8)
    with pytest.raises(ValueError):
        visible_positions(10, 0, 2)


def test_window_attention_equals_explicit_slice():
    # the page's check: window-3 attention at step s equals full attention
    # over keys[max(0, s - 2) .. s]
    rng = np.random.default_rng(17)
    k = rng.standard_normal((40, 2, 8))
    v = rng.standard_normal((40, 2, 8))
    q = rng.standard_normal((1, 4, 8))
    for n in (1, 3, 7, 40):
        for window, sinks in ((3, 0), (5, 2), (64, 0), (1, 4)):
            got = attention_window(q, k[:n], v[:n], window, sinks)
            lo = max(0, n - window)
            head = min(sinks, lo)
            kk = np.concatenate([k[:head], k[lo:n]])
            vv = np.concatenate([v[:head], v[lo:n]])
            assert np.allclose(got, attention_two_pass(q, kk, vv), atol=1e-14)
