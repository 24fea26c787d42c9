"""Pins of the float64 oracle against what the pages and the mathematics fix.

Each test names the passage or the mathematical fact it relies on.  None of
them re-derives the oracle's own formula: expected values come from the
pages' printed traces (tests/golden/p2_paged_trace.json), traces derived by
hand from the pages' code (tests/golden/p1_ownership_trace.json), closed forms
evaluated in 40-digit decimal arithmetic (tests/golden/p3_closed_forms.json),
invariants (paging and tiling must not change results), special cases that
reduce to textbook forms, and brute force in decimal arithmetic.
"""
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest

from oracle import (KVPool, PoolError, PoolExhausted, attention_two_pass,
                    attention_tiled, attention_split_kv, combine_partitions,
                    online_softmax_stats, paged_attention, partition_stats)


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# Allocator: "vladkulikov.com modern-llms module 9 notebook", embedded contract
# key paged.trace (printed snapshots, asserted by the notebook).
# ---------------------------------------------------------------------------
def test_p2_printed_sharing_trace(golden_dir):
    g = _load(golden_dir, "p2_paged_trace.json")
    pool = KVPool(8, 4, store_heads=None)
    for op in g["_ops"]:
        if op[0] == "create":
            pool.create(op[1])
        elif op[0] == "append":
            pool.append(op[1], op[2])
        elif op[0] == "share":
            pool.share_prefix(op[1], op[2], op[3])
        elif op[0] == "release":
            pool.release(op[1])
        else:
            assert pool.snapshot() == g["trace"][op[1]], op[1]
        pool.validate()


def test_p2_cow_gives_distinct_tails(golden_dir):
    # the notebook asserts A's last block differs from B's second block
    pool = KVPool(8, 4, store_heads=None)
    pool.create("A"); pool.append("A", 6)
    pool.share_prefix("A", "B", 6); pool.append("B", 3)
    assert pool.tables["A"][-1] != pool.tables["B"][1]
    assert pool.refs[pool.tables["A"][0]] == 2      # full shared block stays shared


def test_p2_negative_contract():
    # the notebook's negative tests on PagedKVPool(total_blocks=2, block_size=4)
    pool = KVPool(2, 4, store_heads=None)
    with pytest.raises(PoolError):
        pool.append("missing", 1)
    pool.create("x")
    with pytest.raises(PoolError):
        pool.create("x")
    pool.append("x", 6)
    before = pool.snapshot()
    with pytest.raises(PoolExhausted):
        pool.append("x", 3)                 # needs 1 more block than remain
    assert pool.snapshot() == before          # preflight: nothing changed
    with pytest.raises(PoolError):
        pool.share_prefix("x", "y", 7)
    pool.validate()


def test_payload_takes_the_largest_fill_among_sharers():
    # both pages count a shared block's live slots as the largest fill any
    # sharer gives it ("abhik.ai examples/pagedattention.py", the ownership
    # snapshot's occupied slots; "vladkulikov.com modern-llms module 9
    # notebook", PagedKVPool._refresh_fills, unequal prefixes sharing a block)
    pool = KVPool(4, 4, store_heads=None)
    pool.create("parent")
    pool.append("parent", 6)                  # blocks [b0: 4, b1: 2]
    pool.share_prefix("parent", "child", 5)   # child sees b1 with 1 slot
    assert pool.fills()[pool.tables["parent"][1]] == 2
    snap = pool.snapshot()
    assert snap["physical_payload_tokens"] == 6
    assert snap["logical_tokens"] == 11
    assert snap["internal_waste_tokens"] == 8 - 6
    assert snap["sharing_savings_tokens"] == 11 - 6
    pool.validate()


def test_preflight_counts_the_copy_of_a_shared_partial_tail():
    # the notebook's preflight (PagedKVPool._blocks_needed_for_append): a
    # partial tail block with more than one reference needs one extra block,
    # for its copy, before the room left in it can be used
    pool = KVPool(3, 4, store_heads=None)
    pool.create("a")
    pool.append("a", 6)                       # 2 blocks, tail 2 of 4 used; 1 free
    pool.share_prefix("a", "b", 6)            # both blocks shared, tail partial
    assert pool.blocks_needed("b", 1) == 1    # the copy; the token fits its room
    assert pool.blocks_needed("b", 2) == 1
    assert pool.blocks_needed("b", 3) == 2    # the copy and one new block
    assert pool.blocks_needed("a", 0) == 0
    # one free block covers the new block but not the copy: all or nothing
    before = pool.snapshot()
    with pytest.raises(PoolExhausted):
        pool.append("b", 3)
    assert pool.snapshot() == before
    pool.release("a")                          # now b's tail is private
    assert pool.blocks_needed("b", 3) == 1
    pool.validate()


@pytest.mark.parametrize("action,payload", [("release", 1), ("append", 5)])
def test_p2_short_child_survives_parent(action, payload):
    pool = KVPool(4, 4, store_heads=None)
    pool.create("parent"); pool.append("parent", 3)
    pool.share_prefix("parent", "child", 1)
    if action == "release":
        pool.release("parent")
    else:
        pool.append("parent", 1)
    assert pool.snapshot()["physical_payload_tokens"] == payload
    pool.append("child", 2)
    pool.validate()


def test_p2_exact_2048_has_no_waste(golden_dir):
    g = _load(golden_dir, "p2_paged_trace.json")
    pool = KVPool(128, 16, store_heads=None)
    pool.create("fixed"); pool.append("fixed", 2048)
    s = pool.snapshot()
    assert s["internal_waste_tokens"] == 0 == g["paged_waste"]["exact_2048_waste_fraction"]
    assert s["free_blocks"] == 0 and len(pool.tables["fixed"]) == 128


# ---------------------------------------------------------------------------
# Allocator with data: "abhik.ai examples/pagedattention.py", ownership_trace
# (allocation order [5,2,7,0,3,6,1,4]); expected tables derived by hand.
# ---------------------------------------------------------------------------
def test_p1_ownership_trace(golden_dir):
    g = _load(golden_dir, "p1_ownership_trace.json")
    rng = np.random.default_rng(7)
    keys = rng.normal(size=(10, 1, 3))
    values = rng.normal(size=(10, 1, 3))
    pool = KVPool(g["num_blocks"], g["block_size"], 1, 3, g["order"])
    events = iter(g["events"])

    def check():
        want = next(events)
        got = pool.ownership()
        for key in ("tables", "refs", "free", "unique_blocks", "tail_waste_slots",
                    "logical_live_slots", "unique_live_slots"):
            assert got[key] == want[key], (want["event"], key, got[key])
        pool.validate()

    check()
    pool.create("A")
    for i in range(7):
        pool.append("A", 1, keys[i:i + 1], values[i:i + 1])
    check()
    pool.fork("A", "B"); check()
    pool.append("B", 1, keys[7:8], values[7:8]); check()
    pool.append("A", 1, keys[8:9], values[8:9]); check()
    pool.append("B", 1, keys[9:10], values[9:10])
    check()
    for seq in ("A", "B"):
        k, v = pool.gather(seq)
        idx = g["gather"][seq]
        assert np.array_equal(k, keys[idx]) and np.array_equal(v, values[idx])
    pool.release("A"); check()
    pool.release("B"); check()
    assert pool.ownership()["free"] == list(range(8))      # full_pool_recovered


def test_multi_token_append_equals_single_token_appends():
    # the second page's block-wise append and the first page's token-wise
    # append must leave identical tables, refcounts and slot mappings
    rng = np.random.default_rng(11)
    for trial in range(20):
        nb, bs = 64, int(rng.integers(1, 6))
        order = rng.permutation(nb)
        a, b = KVPool(nb, bs, allocation_order=order, store_heads=None), \
            KVPool(nb, bs, allocation_order=order, store_heads=None)
        a.create(0); b.create(0)
        n0 = int(rng.integers(0, 12)); a.append(0, n0); b.append(0, n0)
        p = int(rng.integers(0, n0 + 1))
        a.share_prefix(0, 1, p); b.share_prefix(0, 1, p)
        n1 = int(rng.integers(0, 12))
        slots_a, cow_a = a.append(1, n1)
        slots_b, cow_b = [], []
        for _ in range(n1):
            s, c = b.append(1, 1)
            slots_b += s; cow_b += c
        assert slots_a == slots_b and cow_a == cow_b
        assert a.tables == b.tables and a.refs == b.refs
        a.validate(); b.validate()


def test_cow_copies_whole_block_and_only_partial_shared_tails():
    pool = KVPool(16, 4, 1, 2, allocation_order=list(range(16)))
    kv = np.arange(6 * 2, dtype=float).reshape(6, 1, 2)
    pool.create(0); pool.append(0, 6, kv, -kv)
    pool.share_prefix(0, 1, 6)
    _, cow = pool.append(1, 1, kv[:1] + 100, kv[:1] + 100)
    assert cow == [(1, 2)]                             # partial shared tail copied
    assert np.array_equal(pool.keys[2, :2], pool.keys[1, :2])
    pool.share_prefix(1, 2, 4)                         # full block 0 shared 3 ways
    _, cow = pool.append(2, 1, kv[:1], kv[:1])
    assert cow == [] and pool.tables[2] == [0, 3]      # full block: no copy


def _rename(pool, old, new):
    pool.tables[new] = pool.tables.pop(old)
    pool.lengths[new] = pool.lengths.pop(old)


def test_truncate_equals_share_prefix_then_release():
    # truncate(s, n) is the pages' share_prefix of the first n tokens into a
    # new sequence followed by release of s: same tables, refcounts, free
    # blocks, statistics and next allocations, on random traces with sharing
    rng = np.random.default_rng(23)
    for trial in range(60):
        nb, bs = 48, int(rng.integers(1, 7))
        order = rng.permutation(nb)
        a, b = (KVPool(nb, bs, allocation_order=order, store_heads=None) for _ in range(2))
        for p in (a, b):
            p.create(0)
        n0 = int(rng.integers(1, 30))
        a.append(0, n0); b.append(0, n0)
        for child in (1, 2):                       # sharers of various prefixes
            src = int(rng.integers(0, child))
            pre = int(rng.integers(0, a.lengths[src] + 1))
            a.share_prefix(src, child, pre); b.share_prefix(src, child, pre)
            k = int(rng.integers(0, 9))
            a.append(child, k); b.append(child, k)
        victim = int(rng.integers(0, 3))
        n = int(rng.integers(0, a.lengths[victim] + 1))
        a.truncate(victim, n)
        b.share_prefix(victim, "tmp", n)
        b.release(victim)
        _rename(b, "tmp", victim)
        assert a.tables == b.tables and a.lengths == b.lengths and a.refs == b.refs
        assert a.free_blocks == b.free_blocks and a.snapshot() == b.snapshot()
        a.validate(); b.validate()
        grow = int(rng.integers(0, 2 * bs + 1))   # the next allocations agree too
        if a.blocks_needed(victim, grow) <= a.free_blocks:
            assert a.append(victim, grow) == b.append(victim, grow)
            assert a.tables == b.tables and a.refs == b.refs


def test_truncate_special_cases():
    pool = KVPool(8, 4, store_heads=None)
    pool.create(0); pool.append(0, 10)             # blocks 0, 1, 2 (2 tokens in 2)
    pool.truncate(0, 10)                           # to its own length: nothing changes
    assert pool.tables[0] == [0, 1, 2] and pool.free_blocks == 5
    pool.truncate(0, 8)                            # a whole block dropped, freed
    assert pool.tables[0] == [0, 1] and pool.refs[2] == 0 and pool.free_blocks == 6
    pool.truncate(0, 5)                            # partial block kept
    assert pool.tables[0] == [0, 1] and pool.lengths[0] == 5
    pool.share_prefix(0, 1, 5)
    pool.truncate(0, 0)                            # shared blocks survive their sharer
    assert pool.tables[0] == [] and pool.refs[:2] == [1, 1] and pool.free_blocks == 6
    slots, cow = pool.append(1, 1)                 # sole holder now: no copy-on-write
    assert cow == [] and slots == [1 * 4 + 1]
    with pytest.raises(PoolError):
        pool.truncate(1, 7)                        # beyond the length
    with pytest.raises(PoolError):
        pool.truncate(1, -1)
    with pytest.raises(PoolError):
        pool.truncate(5, 0)                        # unknown sequence
    pool.validate()


# ---------------------------------------------------------------------------
# Attention: "docs.rs ferrum-kv 0.4.0 src/attention.rs" unit tests, closed forms
# ---------------------------------------------------------------------------
def _pool_with(keys, values, block_size, order=None):
    kv_len, hkv, d = keys.shape
    nb = max(1, -(-kv_len // block_size))
    pool = KVPool(nb, block_size, hkv, d, order)
    pool.create("s")
    pool.append("s", kv_len, keys, values)
    return pool


def test_p3_single_token_decode(golden_dir):
    c = _load(golden_dir, "p3_closed_forms.json")["single_token_decode"]
    H, d, n = c["num_heads"], c["head_dim"], c["kv_len"]
    keys = np.ones((n, H, d))
    values = np.stack([np.full((H, d), p + 1.0) for p in range(n)])
    pool = _pool_with(keys, values, 16)
    out = paged_attention(pool, "s", np.ones((1, H, d)))
    assert np.allclose(out, c["expected"], atol=1e-14, rtol=0)


def test_p3_prefill_causal_masking(golden_dir):
    c = _load(golden_dir, "p3_closed_forms.json")["prefill_causal_masking"]
    k = np.array(c["keys"], float)[:, None, :]
    v = np.array(c["values"], float)[:, None, :]
    q = np.array(c["queries"], float)[:, None, :]
    out = paged_attention(_pool_with(k, v, 16), "s", q)[:, 0, :]
    assert np.allclose(out, np.array(c["expected"], float), atol=1e-15, rtol=0)
    assert out[1, 0] < 0.5 < out[1, 1]                # the page's own assertion


def test_p3_attention_across_blocks(golden_dir):
    c = _load(golden_dir, "p3_closed_forms.json")["attention_across_blocks"]
    n = c["kv_len"]
    k = np.array([[[p + 1.0] * 2] for p in range(n)])
    v = 10.0 * k
    pool = _pool_with(k, v, c["block_size"], order=[1, 0])
    assert pool.tables["s"] == [1, 0]                 # physically out of order
    out = paged_attention(pool, "s", np.ones((1, 1, 2)))
    assert np.allclose(out, c["expected"], atol=1e-12, rtol=0)
    assert 10 < out[0, 0, 0] < 40                     # the page's own assertion


# ---------------------------------------------------------------------------
# Invariants and special cases
# ---------------------------------------------------------------------------
def _random_case(rng, q_tokens, H, Hkv, d, kv_len):
    q = rng.normal(size=(q_tokens, H, d))
    k = rng.normal(size=(kv_len, Hkv, d))
    v = rng.normal(size=(kv_len, Hkv, d))
    return q, k, v


def test_paged_equals_contiguous_under_any_permutation():
    rng = np.random.default_rng(3)
    q, k, v = _random_case(rng, 2, 4, 2, 8, 37)
    ref = attention_two_pass(q, k, v)
    for trial in range(10):
        order = rng.permutation(10) if trial else None
        pool = _pool_with(k, v, 4, order)
        assert np.array_equal(paged_attention(pool, "s", q), ref)


def test_uniform_keys_give_mean_of_values():
    rng = np.random.default_rng(5)
    kv_len, d = 23, 16
    k = np.tile(rng.normal(size=(1, 2, d)), (kv_len, 1, 1))
    v = rng.normal(size=(kv_len, 2, d))
    out = attention_two_pass(rng.normal(size=(1, 4, d)), k, v)
    mean = v.mean(axis=0)
    assert np.allclose(out[0, :2], mean[0], atol=1e-14)
    assert np.allclose(out[0, 2:], mean[1], atol=1e-14)


def test_single_key_returns_its_value_exactly():
    rng = np.random.default_rng(6)
    q, k, v = _random_case(rng, 1, 3, 1, 8, 1)
    out = attention_two_pass(q, k, v)
    for h in range(3):
        assert np.array_equal(out[0, h], v[0, 0])


def test_one_hot_limit():
    # a dominant score selects its value: the page's query-shift control
    # ("vladkulikov.com ... controlled query shift", error < .03 when kept)
    n, d = 128, 32
    k = np.zeros((n, 1, d)); k[0, 0, 0] = 12; k[90, 0, 1] = 12
    v = np.zeros((n, 1, d)); v[0, 0, 0] = 1; v[90, 0, 1] = 1
    q = np.zeros((1, 1, d)); q[0, 0, 1] = 4
    out = attention_two_pass(q, k, v)
    target = np.zeros(d); target[1] = 1
    assert np.linalg.norm(out[0, 0] - target) < 0.03


def test_empty_cache_gives_zeros():
    out = attention_two_pass(np.ones((1, 2, 4)), np.zeros((0, 1, 4)), np.zeros((0, 1, 4)))
    assert np.array_equal(out, np.zeros((1, 2, 4)))


def test_decode_sees_everything_and_full_chunk_is_square_causal():
    # q_tokens = 1: no mask (plain softmax); q_tokens = kv_len: the square
    # lower-triangular mask of the lecture's reference_attention (numpy tril)
    rng = np.random.default_rng(8)
    q, k, v = _random_case(rng, 9, 1, 1, 8, 9)
    s = q[:, 0] @ k[:, 0].T / math.sqrt(8)
    s = np.where(np.tril(np.ones((9, 9), bool)), s, -np.inf)
    p = np.exp(s - s.max(1, keepdims=True)); p /= p.sum(1, keepdims=True)
    assert np.allclose(attention_two_pass(q, k, v)[:, 0], p @ v[:, 0], atol=1e-14)
    s1 = k[:, 0] @ q[3, 0] / math.sqrt(8)
    p1 = np.exp(s1 - s1.max()); p1 /= p1.sum()
    assert np.allclose(attention_two_pass(q[3:4], k, v)[0, 0], p1 @ v[:, 0], atol=1e-14)


def test_causal_offset_rule_matches_cached_decoder_mask():
    # "semidirectx ... CachedDecoder._block_step": new queries are positions
    # Tk-T..Tk-1 and see keys j <= i + Tk - T.  Changing a key that query i may
    # not see must not change row i; changing one it may see must change it.
    rng = np.random.default_rng(9)
    T, Tk = 4, 10
    q, k, v = _random_case(rng, T, 1, 1, 8, Tk)
    base = attention_two_pass(q, k, v)
    for i in range(T):
        for j in range(Tk):
            k2 = k.copy(); k2[j] += 3.0
            changed = not np.allclose(attention_two_pass(q, k2, v)[i], base[i], atol=1e-15)
            assert changed == (j <= i + Tk - T), (i, j)


def test_gqa_equals_mha_with_repeated_kv_heads():
    rng = np.random.default_rng(10)
    H, Hkv = 8, 2
    q, k, v = _random_case(rng, 3, H, Hkv, 16, 20)
    kr, vr = np.repeat(k, H // Hkv, axis=1), np.repeat(v, H // Hkv, axis=1)
    assert np.array_equal(attention_two_pass(q, k, v), attention_two_pass(q, kr, vr))
    # contiguous grouping: query head h uses KV head h // (H/Hkv), not h % Hkv
    out = attention_two_pass(q, k, v)
    alt = attention_two_pass(q, k[:, ::-1], v[:, ::-1])
    assert not np.allclose(out, alt)


@pytest.mark.parametrize("tile", [1, 3, 16, 64])
def test_online_tiled_equals_two_pass(tile):
    rng = np.random.default_rng(12)
    q, k, v = _random_case(rng, 5, 4, 2, 16, 50)
    assert np.allclose(attention_tiled(q, k, v, tile), attention_two_pass(q, k, v),
                       atol=1e-12, rtol=0)


def test_online_softmax_stats_closed_form():
    rng = np.random.default_rng(13)
    x = rng.normal(size=41) * 5
    m, l = online_softmax_stats([x[:7], x[7:8], x[8:30], x[30:]])
    assert m == x.max()
    assert math.isclose(l, float(np.exp(x - x.max()).sum()), rel_tol=1e-13)


@pytest.mark.parametrize("part", [1, 4, 7, 64, 4096])
def test_split_kv_equals_unsplit(part):
    rng = np.random.default_rng(14)
    q, k, v = _random_case(rng, 3, 4, 2, 16, 64)
    assert np.allclose(attention_split_kv(q, k, v, part), attention_two_pass(q, k, v),
                       atol=1e-12, rtol=0)


def test_combine_ignores_empty_partitions():
    rng = np.random.default_rng(15)
    q, k, v = _random_case(rng, 1, 2, 1, 8, 10)
    m0, l0, o0 = partition_stats(q, k, v, 0, 10)
    m1, l1, o1 = partition_stats(q, k, v, 10, 20)      # beyond kv_len: empty
    assert np.all(np.isneginf(m1)) and np.all(l1 == 0)
    assert np.allclose(combine_partitions([m0, m1], [l0, l1], [o0, o1]),
                       attention_two_pass(q, k, v), atol=1e-14)


def _decimal_attention(q, k, v):
    """Brute force in 40-digit decimal: p_j = e^(s_j) / sum e^(s_i) over the
    visible keys, no max shift, plain Python loops."""
    getcontext().prec = 40
    q_tokens, H, d = q.shape
    kv_len, Hkv, _ = k.shape
    G = H // Hkv
    root = Decimal(d).sqrt()
    out = np.zeros((q_tokens, H, d))
    for t in range(q_tokens):
        for h in range(H):
            e = []
            for j in range(kv_len):
                if j > kv_len - q_tokens + t:
                    break
                s = sum(Decimal(float(q[t, h, i])) * Decimal(float(k[j, h // G, i]))
                        for i in range(d)) / root
                e.append(s.exp())
            tot = sum(e)
            for i in range(d):
                out[t, h, i] = float(sum(e[j] * Decimal(float(v[j, h // G, i]))
                                         for j in range(len(e))) / tot)
    return out


@pytest.mark.parametrize("shape", [(1, 2, 1, 4, 5), (3, 4, 2, 8, 12), (2, 1, 1, 3, 2)])
def test_brute_force_decimal(shape):
    qt, H, Hkv, d, n = shape
    rng = np.random.default_rng(sum(shape))
    q, k, v = _random_case(rng, qt, H, Hkv, d, n)
    ref = _decimal_attention(q, k, v)
    assert np.allclose(attention_two_pass(q, k, v), ref, atol=1e-13, rtol=0)
    assert np.allclose(attention_tiled(q, k, v, 3), ref, atol=1e-13, rtol=0)


def test_validate_catches_corruption():
    pool = KVPool(4, 2, store_heads=None)
    pool.create(0); pool.append(0, 3)
    pool.refs[pool.tables[0][0]] += 1
    with pytest.raises(AssertionError):
        pool.validate()


def test_random_op_fuzz_keeps_invariants():
    rng = np.random.default_rng(16)
    pool = KVPool(40, 4, allocation_order=rng.permutation(40), store_heads=None)
    live, nxt = [], 0
    for _ in range(400):
        r = rng.random()
        try:
            if r < 0.2 or not live:
                pool.create(nxt); live.append(nxt); nxt += 1
            elif r < 0.6:
                pool.append(live[rng.integers(len(live))], int(rng.integers(0, 9)))
            elif r < 0.8:
                src = live[rng.integers(len(live))]
                pool.share_prefix(src, nxt, int(rng.integers(0, pool.lengths[src] + 1)))
                live.append(nxt); nxt += 1
            elif r < 0.9:
                s = live.pop(rng.integers(len(live)))
                pool.release(s)
            else:
                s = live[rng.integers(len(live))]
                pool.truncate(s, int(rng.integers(0, pool.lengths[s] + 1)))
        except PoolExhausted:
            pass
        pool.validate()
