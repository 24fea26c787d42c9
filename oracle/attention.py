"""Oracle attention over a paged KV cache, float64 -- TEST INFRASTRUCTURE ONLY.

Restates:
  * "docs.rs ferrum-kv 0.4.0 src/attention.rs", ``paged_attention``: query
    [q_tokens, num_heads, head_dim]; K/V gathered [kv_len, num_kv_heads,
    head_dim]; heads_per_kv = num_heads / num_kv_heads and kv_h = h /
    heads_per_kv (GQA); scores q.k * scale with scale = 1/sqrt(head_dim);
    query qt may see positions 0..max_visible, max_visible = kv_len - q_tokens
    + qt; max-subtracted softmax; weighted sum of V.
  * "abhik.ai examples/pagedattention.py", ``KVPool.attention`` (Eq. 3): the
    same softmax for one decode query; an empty cache gives zeros.
  * "semidirectx cmu11-667 lecture19 infer_world.py", section 3: one-pass
    statistics m' = max(m, max block), l' = l e^(m - m') + sum e^(block - m')
    (``online_softmax_stats``) and the tiled (m, l, acc) recurrence with the
    -inf guard (``tiled_attention``).

Readings (where the pages are silent): the scale is computed in float64 as
1/sqrt(head_dim); a split of the key range into partitions keeps, per
partition, (m_p, l_p, o_p = acc_p / l_p) and merges them with weights
w_p = l_p e^(m_p - M), M = max_p m_p -- the same algebra as the tiled
recurrence applied once across partitions; an empty partition has m = -inf,
l = 0 and weight 0.
"""
from __future__ import annotations

import math

import numpy as np


def _check(q, k, v):
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    if q.ndim != 3 or k.ndim != 3 or v.shape != k.shape:
        raise ValueError("q [q_tokens, H, d], k/v [kv_len, Hkv, d] expected")
    if q.shape[2] != k.shape[2]:
        raise ValueError("head_dim mismatch")
    H, Hkv = q.shape[1], k.shape[1]
    if Hkv == 0 or H % Hkv:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    return q, k, v


def attention_two_pass(q, k, v, scale=None):
    """Gathered (contiguous, logical-order) attention with the causal offset rule.

    q: [q_tokens, H, d]; k, v: [kv_len, Hkv, d]  ->  out [q_tokens, H, d].
    kv_len == 0 gives zeros (first page's authored empty-cache result).
    """
    q, k, v = _check(q, k, v)
    q_tokens, H, d = q.shape
    kv_len, Hkv = k.shape[0], k.shape[1]
    if kv_len and q_tokens > kv_len:
        raise ValueError("q_tokens exceeds kv_len")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    group = H // Hkv
    out = np.zeros((q_tokens, H, d))
    if kv_len == 0:
        return out
    for qt in range(q_tokens):
        max_visible = kv_len - q_tokens + qt
        for h in range(H):
            kv_h = h // group
            scores = (k[:, kv_h, :] @ q[qt, h]) * scale
            scores[max_visible + 1:] = -np.inf
            weights = np.exp(scores - scores.max())
            weights /= weights.sum()
            out[qt, h] = weights @ v[:, kv_h, :]
    return out


def paged_attention(pool, seq, q, kv_len=None, scale=None):
    """Attention of ``q`` [q_tokens, H, d] over sequence ``seq`` of an oracle
    ``KVPool``: gather through the block table, then ``attention_two_pass``
    ("docs.rs ferrum-kv 0.4.0 src/attention.rs", ``paged_attention``; "abhik.ai examples/pagedattention.py", ``KVPool.attention``).

    The pool must store every KV head (``store_heads='all'``) unless H equals
    the number of stored heads times the group size of those heads; for a pool
    storing a subset of KV heads, pass q restricted to the matching query heads.
    """
    k, v = pool.gather(seq, kv_len)
    return attention_two_pass(q, k, v, scale)


def online_softmax_stats(score_blocks):
    """(m, l) of a score vector seen block by block; softmax_i = e^(x_i - m) / l
    ("semidirectx cmu11-667 lecture19 infer_world.py", section 3, ``online_softmax_stats``)."""
    m, l = -math.inf, 0.0
    for blk in score_blocks:
        blk = np.asarray(blk, np.float64)
        if blk.size == 0:
            continue
        m_new = max(m, float(blk.max()))
        l = (l * math.exp(m - m_new) if l else 0.0) + float(np.exp(blk - m_new).sum())
        m = m_new
    return m, l


def attention_tiled(q, k, v, tile=16, scale=None):
    """The one-pass (m, l, acc) recurrence over key tiles, causal offset rule
    ("semidirectx cmu11-667 lecture19 infer_world.py", section 3, ``tiled_attention``).

    Same contract as ``attention_two_pass``; each query keeps running
    max m, sum l and unnormalised accumulator acc, rescaled by e^(m - m') when a
    tile raises the max; a fully masked tile leaves the state unchanged.
    """
    q, k, v = _check(q, k, v)
    q_tokens, H, d = q.shape
    kv_len, Hkv = k.shape[0], k.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    group = H // Hkv
    out = np.zeros((q_tokens, H, d))
    for qt in range(q_tokens):
        max_visible = kv_len - q_tokens + qt
        for h in range(H):
            kv_h = h // group
            m, l, acc = -math.inf, 0.0, np.zeros(d)
            for s0 in range(0, kv_len, tile):
                s1 = min(s0 + tile, kv_len)
                s = (k[s0:s1, kv_h, :] @ q[qt, h]) * scale
                s[np.arange(s0, s1) > max_visible] = -np.inf
                tile_max = s.max()
                if tile_max == -np.inf:
                    continue
                m_new = max(m, tile_max)
                correction = math.exp(m - m_new) if m != -math.inf else 0.0
                p = np.exp(s - m_new)
                acc = acc * correction + p @ v[s0:s1, kv_h, :]
                l = l * correction + p.sum()
                m = m_new
            if l > 0:
                out[qt, h] = acc / l
    return out


def partition_stats(q, k, v, start, stop, scale=None):
    """Reading (split-K is not on the pages): the recurrence of "semidirectx cmu11-667 lecture19 infer_world.py",
    section 3, over one key range.  Per (qt, h): (m, l, o) over keys [start, stop) with the causal rule of
    the whole sequence; o = acc / l, or zeros with m = -inf, l = 0 when no key
    of the partition is visible."""
    q, k, v = _check(q, k, v)
    q_tokens, H, d = q.shape
    kv_len, Hkv = k.shape[0], k.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    group = H // Hkv
    m = np.full((q_tokens, H), -np.inf)
    l = np.zeros((q_tokens, H))
    o = np.zeros((q_tokens, H, d))
    stop = min(stop, kv_len)
    for qt in range(q_tokens):
        max_visible = kv_len - q_tokens + qt
        hi = min(stop, max_visible + 1)
        if hi <= start:
            continue
        for h in range(H):
            kv_h = h // group
            s = (k[start:hi, kv_h, :] @ q[qt, h]) * scale
            m[qt, h] = s.max()
            p = np.exp(s - m[qt, h])
            l[qt, h] = p.sum()
            o[qt, h] = (p @ v[start:hi, kv_h, :]) / l[qt, h]
    return m, l, o


def combine_partitions(ms, ls, os):
    """Reading: the rescale of "semidirectx cmu11-667 lecture19 infer_world.py", section 3, applied once
    across partitions.  Merge partition statistics: M = max_p m_p, w_p = l_p e^(m_p - M),
    o = sum_p w_p o_p / sum_p w_p.  ms, ls: [P, ...]; os: [P, ..., d]."""
    ms = np.asarray(ms, np.float64)
    ls = np.asarray(ls, np.float64)
    os = np.asarray(os, np.float64)
    M = ms.max(axis=0)
    finite = np.isfinite(M)
    safe_M = np.where(finite, M, 0.0)
    w = np.where(np.isfinite(ms), ls * np.exp(np.where(np.isfinite(ms), ms, 0.0) - safe_M), 0.0)
    den = w.sum(axis=0)
    num = (w[..., None] * os).sum(axis=0)
    out = np.zeros(num.shape)
    ok = den > 0
    out[ok] = num[ok] / den[ok][..., None]
    return out


def attention_split_kv(q, k, v, partition, scale=None):
    """Attention computed as partitions of ``partition`` keys plus the merge
    (``partition_stats`` and ``combine_partitions``, readings of "semidirectx cmu11-667 lecture19 infer_world.py", section 3)."""
    kv_len = np.asarray(k).shape[0]
    parts = max(1, -(-kv_len // partition))
    stats = [partition_stats(q, k, v, p * partition, (p + 1) * partition, scale)
             for p in range(parts)]
    return combine_partitions([s[0] for s in stats], [s[1] for s in stats],
                              [s[2] for s in stats])


def visible_positions(kv_len, window, sinks=0):
    """Key positions one decode step sees under a sink + recent window.

    "vladkulikov.com modern-llms module 9 notebook", ``streaming_keep_indices``
    with budget = sinks + window: the first ``sinks`` positions and the most
    recent ``window``; everything when kv_len <= budget.  With sinks = 0 this
    is the sliding-window cache of the same page (``NumpyKVCacheExplicit``:
    the last ``window`` positions survive)."""
    kv_len, window, sinks = int(kv_len), int(window), int(sinks)
    if window < 1 or sinks < 0:
        raise ValueError("window must be >= 1 and sinks >= 0")
    head = list(range(min(sinks, kv_len)))
    start = max(len(head), kv_len - window)
    return head + list(range(start, kv_len))


def attention_window(q, k, v, window, sinks=0, scale=None):
    """Decode attention (q_tokens = 1) over the visible positions only
    ("vladkulikov.com modern-llms module 9 notebook", ``streaming_keep_indices``; see ``visible_positions``)."""
    idx = visible_positions(np.asarray(k).shape[0], window, sinks)
    return attention_two_pass(q, np.asarray(k)[idx], np.asarray(v)[idx], scale)
