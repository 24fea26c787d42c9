"""Prefix cache (content-keyed reuse of full blocks): oracle pins, the
library against the page's trace numbers, and the library against the
oracle on random traces, bit for bit (tables, refcounts, statistics).

The page ("vladkulikov.com modern-llms module 9 notebook", prefix-hash
trace) states for its 100-user x 5-turn trace: 98 % of requests reuse a
block and 490 x 32 / (500 x 48) of the input tokens come from the cache
with one shared scope; 80 % of requests reuse a block with per-user scopes;
a block with the same tokens but different preceding context, or another
model revision, is a different key.
"""
import numpy as np
import pytest

import paged_kv_cache_483_b200 as pa
from oracle import KVPool, PoolError, PrefixCache, prefix_key, run_prefix_trace, trace_tokens


# ---------------------------------------------------------------- oracle pins
def test_oracle_trace_matches_page_numbers():
    shared = run_prefix_trace(isolated=False)
    isolated = run_prefix_trace(isolated=True)
    assert np.isclose(shared[0], 0.98)
    assert np.isclose(isolated[0], 0.8)
    assert np.isclose(shared[1], 490 * 32 / (500 * 48))


def test_oracle_key_identity():
    a = list(range(32))
    b = list(a)
    b[0] = 999
    assert a[16:32] == b[16:32]                    # same block content
    assert prefix_key(a, 32, "s", "r1") != prefix_key(b, 32, "s", "r1")   # other context
    assert prefix_key(a, 32, "s", "r1") != prefix_key(a, 32, "s", "r2")   # other revision
    assert prefix_key(a, 32, "s", "r1") != prefix_key(a, 32, "t", "r1")   # other scope
    assert prefix_key(a, 32, "s", "r1") == prefix_key(list(a), 32, "s", "r1")


def _oracle_trace_through_pool(isolated, bs=16):
    """The trace driven through the block-level PrefixCache: its hit counts
    must be the key-level trace's, and the pool stays valid throughout."""
    pool = KVPool(1024, bs)
    cache = PrefixCache(pool)
    n_hit = reused = total = 0
    seq = 0
    for user in range(100):
        for turn in range(5):
            toks = trace_tokens(user, turn)
            scope = ("user", user) if isolated else "shared"
            hit = cache.create_cached(seq, toks, scope, "model-r1")
            pool.append(seq, len(toks) - hit)
            cache.publish(seq, toks, scope, "model-r1")
            pool.release(seq)
            pool.validate()
            n_hit += hit > 0
            reused += hit
            total += len(toks)
            seq += 1
    return n_hit / 500, reused / total, pool, cache


@pytest.mark.parametrize("isolated", [False, True])
def test_oracle_block_cache_equals_key_trace(isolated):
    hits, frac, pool, cache = _oracle_trace_through_pool(isolated)
    assert (hits, frac) == run_prefix_trace(isolated)
    # keys: 10 first blocks, 10 second blocks, 500 third blocks (shared);
    # per user: 1 + 1 + 5 (isolated)
    assert len(cache.blocks) == (520 if not isolated else 700)
    held = pool.num_blocks - pool.free_blocks
    assert held == len(set(cache.blocks.values()))
    assert cache.clear() == held and pool.free_blocks == pool.num_blocks
    pool.validate()


def test_oracle_publish_rejects_tokens_beyond_length():
    pool = KVPool(8, 4)
    cache = PrefixCache(pool)
    pool.create(0)
    pool.append(0, 5)
    with pytest.raises(PoolError):
        cache.publish(0, list(range(6)), "s", "r")
    assert cache.publish(0, list(range(5)), "s", "r") == 1      # one full block


# ----------------------------------------------------- library vs the page
@pytest.mark.parametrize("isolated", [False, True])
def test_library_trace_matches_page_numbers(isolated):
    pool = pa.Pool(1024, 16, 1, 1, "f32")
    n_hit = reused = total = 0
    for seq in range(500):
        user, turn = divmod(seq, 5)
        toks = trace_tokens(user, turn)
        scope = 1000 + user if isolated else 7
        hit = pool.create_cached(seq, toks, scope=scope, revision=1)
        pool.plan_append([seq], [len(toks) - hit])
        pool.publish(seq, toks, scope=scope, revision=1)
        pool.release(seq)
        n_hit += hit > 0
        reused += hit
        total += len(toks)
    assert pool.validate()
    want = run_prefix_trace(isolated)
    assert np.isclose(n_hit / 500, want[0]) and np.isclose(reused / total, want[1])
    assert pool.prefix_entries() == (520 if not isolated else 700)
    held = pool.stats()["allocated_blocks"]
    assert pool.prefix_clear() == held
    assert pool.stats()["allocated_blocks"] == 0 and pool.validate()


def test_library_key_identity():
    pool = pa.Pool(16, 16, 1, 1, "f32")
    a = list(range(32))
    b = list(a)
    b[0] = 999
    pool.create(0)
    pool.plan_append([0], [32])
    assert pool.publish(0, a, scope=1, revision=1) == 2
    assert pool.create_cached(1, a, scope=1, revision=1) == 32
    assert pool.create_cached(2, b, scope=1, revision=1) == 0    # other context
    assert pool.create_cached(3, a, scope=1, revision=2) == 0    # other revision
    assert pool.create_cached(4, a, scope=2, revision=1) == 0    # other scope
    assert pool.create_cached(5, a[:31], scope=1, revision=1) == 16   # full blocks only
    assert pool.table(1)[0] == pool.table(0)[0]
    assert pool.validate()


def test_library_prefix_errors():
    pool = pa.Pool(8, 4, 1, 1, "f32")
    pool.create(0)
    pool.plan_append([0], [5])
    with pytest.raises(pa.PAError):
        pool.publish(0, list(range(6)))                  # beyond the length
    with pytest.raises(pa.PAError):
        pool.publish(9, list(range(4)))                  # unknown sequence
    with pytest.raises(pa.PAError):
        pool.create_cached(0, list(range(4)))            # duplicate sequence
    assert pool.validate()


# --------------------------------------------- library vs oracle, bit-exact
def _compare(pool, ref, live):
    assert pool.refcounts() == ref.refs
    snap = ref.snapshot()
    st = pool.stats()
    for k in ("allocated_blocks", "free_blocks", "physical_capacity_tokens",
              "physical_payload_tokens", "logical_tokens", "internal_waste_tokens",
              "sharing_savings_tokens"):
        assert st[k] == snap[k], k
    for s in live:
        assert pool.table(s) == (ref.tables[s], ref.lengths[s])
    assert pool.validate()
    ref.validate()


@pytest.mark.parametrize("seed", [1, 2, 3, 4])
def test_library_equals_oracle_random_trace(seed):
    rng = np.random.default_rng(seed)
    bs, nb = 4, 96
    order = rng.permutation(nb).tolist()
    pool = pa.Pool(nb, bs, 1, 1, "f32", alloc_order=order)
    ref = KVPool(nb, bs, allocation_order=order)
    cache = PrefixCache(ref)
    stems = [rng.integers(0, 5, size=24).tolist() for _ in range(3)]
    live, tokens_of, nxt = [], {}, 0
    reused = 0
    for step in range(300):
        r = rng.random()
        if r < 0.45:                                    # a request with a known stem
            stem = stems[rng.integers(0, 3)]
            cut = int(rng.integers(0, 25))
            toks = stem[:cut] + rng.integers(0, 3, size=int(rng.integers(0, 9))).tolist()
            scope, rev = int(rng.integers(0, 2)), int(rng.integers(0, 2))
            hit_ref = cache.hit_tokens(toks, scope, rev)
            try:
                ref_hit = cache.create_cached(nxt, toks, scope, rev)
            except PoolError:
                continue
            hit = pool.create_cached(nxt, toks, scope=scope, revision=rev)
            assert hit == ref_hit == hit_ref
            reused += hit
            rest = len(toks) - hit
            try:
                ref.append(nxt, rest)
                ok = True
            except MemoryError:
                ok = False
            if ok:
                pool.plan_append([nxt], [rest])
                added_ref = cache.publish(nxt, toks, scope, rev)
                assert pool.publish(nxt, toks, scope=scope, revision=rev) == added_ref
            else:
                with pytest.raises(pa.PAError):
                    pool.plan_append([nxt], [rest])
            live.append(nxt)
            tokens_of[nxt] = toks
            nxt += 1
        elif r < 0.75 and live:                         # release
            s = live.pop(int(rng.integers(0, len(live))))
            ref.release(s)
            pool.release(s)
        elif r < 0.9 and live:                          # decode-style growth
            s = live[int(rng.integers(0, len(live)))]
            try:
                ref.append(s, 1)
            except MemoryError:
                with pytest.raises(pa.PAError):
                    pool.plan_append([s], [1])
                continue
            pool.plan_append([s], [1])
        elif r < 0.93:                                  # drop the cache
            assert pool.prefix_clear() == cache.clear()
        _compare(pool, ref, live)
    assert pool.prefix_entries() == len(cache.blocks)
    assert reused > 0                                   # the trace did reuse blocks
