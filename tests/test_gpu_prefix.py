"""Decode over blocks reached through the prefix cache (needs a B200).

The prefix-hash trace of "vladkulikov.com modern-llms module 9 notebook"
(complete block boundaries) keys full blocks by (scope, revision, every token
id before the block's end); a new request starts with its longest run of
cached leading blocks.  Here that reuse drives real K/V: sequences start
through pa_seq_create_cached, append past the cached run, one of them forks a
partial prefix and appends (a copy-on-write of a shared partial tail), the
writer of the cached blocks is released before later requests reuse them, and
the cache is cleared so freed blocks are reallocated.  The library and an
oracle KVPool + PrefixCache run the same script on the same bf16 rows.

Bars: slot mappings, tables, refcounts and every live slot's bytes
bit-exact; decode outputs within 2e-3 max-abs (the bf16 decode bar) on every
head of every sequence.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_483_b200 as pa
import workloads
from oracle import KVPool, PrefixCache, attention_two_pass

pytestmark = pytest.mark.gpu

TOL_DECODE = 2e-3
NB, BS, HKV, H, D = 96, 16, 8, 32, 128
SCOPE, REV = 0x5EED, 3


class Both:
    """The library pool and the oracle pool, driven by the same calls."""

    def __init__(self, seed):
        self.order = workloads.permutation(NB, seed)
        self.kc = torch.empty((NB, BS, HKV, D), dtype=torch.bfloat16, device="cuda")
        self.vc = torch.empty_like(self.kc)
        self.kc.fill_(float("nan"))          # never-written slots must not leak
        self.vc.fill_(float("nan"))
        self.lib = pa.Pool(NB, BS, HKV, D, "bf16", self.kc, self.vc, alloc_order=self.order)
        self.ref = KVPool(NB, BS, HKV, D, self.order, dtype=np.float32)
        self.cache = PrefixCache(self.ref)
        self.seed = seed
        self.n_appends = 0

    def create_cached(self, seq, tokens):
        got = self.lib.create_cached(seq, tokens, SCOPE, REV)
        want = self.cache.create_cached(seq, tokens, SCOPE, REV)
        assert got == want
        return got

    def publish(self, seq, tokens):
        assert self.lib.publish(seq, tokens, SCOPE, REV) == self.cache.publish(seq, tokens,
                                                                               SCOPE, REV)

    def fork(self, parent, child, prefix):
        self.lib.fork(parent, child, prefix)
        self.ref.share_prefix(parent, child, prefix)

    def release(self, seq):
        self.lib.release(seq)
        self.ref.release(seq)

    def clear(self):
        assert self.lib.prefix_clear() == self.cache.clear()

    def append(self, seq, n):
        self.n_appends += 1
        base = 2 * (self.seed * 1_000_003 + self.n_appends)
        k = workloads.normal((n, HKV, D), base)
        v = workloads.normal((n, HKV, D), base + 1)
        got = self.lib.append_kv([seq], [n], k.cuda(), v.cuda(), return_slots=True)
        want, _ = self.ref.append(seq, n, k.float().numpy(), v.float().numpy())
        assert got == want                                  # bit-exact plan
        return want

    def check_state(self, seqs):
        assert self.lib.refcounts() == self.ref.refs
        assert self.lib.validate()
        self.ref.validate()
        for s in seqs:
            assert self.lib.table(s) == (self.ref.tables[s], self.ref.lengths[s])
        torch.cuda.synchronize()
        kc, vc = self.kc.float().cpu().numpy(), self.vc.float().cpu().numpy()
        for s in seqs:
            for t in range(self.ref.lengths[s]):
                blk, off = self.ref.address(s, t)
                assert np.array_equal(kc[blk, off], self.ref.keys[blk, off])
                assert np.array_equal(vc[blk, off], self.ref.values[blk, off])

    def decode(self, seqs, q):
        tables, lens = self.lib.block_tables(seqs, max(len(self.ref.tables[s]) for s in seqs))
        assert np.array_equal(tables, self.ref.block_table(seqs, tables.shape[1]))
        out = self.lib.decode(q.cuda(), torch.from_numpy(tables).cuda(),
                              torch.from_numpy(lens).cuda())
        torch.cuda.synchronize()
        out = out.cpu().numpy()
        worst = 0.0
        for i, s in enumerate(seqs):
            k, v = self.ref.gather(s)
            ref = attention_two_pass(q[i:i + 1].double().numpy(), k.astype(np.float64),
                                     v.astype(np.float64))
            worst = max(worst, float(np.abs(out[i] - ref[0]).max()))
        assert np.isfinite(out).all()
        return worst


def _prompt(head, tail_id, n_tail):
    """A shared system prompt followed by a request-specific tail."""
    return list(range(head)) + [tail_id * 1000 + i for i in range(n_tail)]


def test_decode_over_prefix_cached_blocks():
    x = Both(seed=20261203)
    p0 = _prompt(40, 1, 10)                  # 50 tokens: 3 full blocks + 2
    assert x.create_cached(0, p0) == 0       # cold cache
    x.append(0, len(p0))
    x.publish(0, p0)                         # keys of 3 full blocks
    p1 = _prompt(40, 2, 20)                  # same first 40 ids: 2 full blocks match
    assert x.create_cached(1, p1) == 32
    x.append(1, len(p1) - 32)
    x.fork(1, 2, 37)                         # shares block 2 of seq 1 with 5 of its 16 slots
    x.append(2, 3)                           # copy-on-write of that shared partial tail
    x.release(0)                             # the writer goes; the cache keeps its blocks
    assert x.create_cached(3, p0 + [7, 8]) == 48
    x.append(3, 4)
    x.check_state([1, 2, 3])
    # one decode step: every sequence appends its next token, then attends
    seqs = [1, 2, 3]
    for s in seqs:
        x.append(s, 1)
    x.check_state(seqs)
    q = workloads.normal((len(seqs), H, D), 4242)
    assert x.decode(seqs, q) <= TOL_DECODE

    # clear the cache: blocks only it held return to the free list and are
    # reallocated (stale bytes) by the next sequences
    x.clear()
    p4 = _prompt(40, 4, 30)
    assert x.create_cached(4, p4) == 0
    x.append(4, len(p4))
    x.publish(4, p4)
    assert x.create_cached(5, p4) == 64      # 4 full blocks of the 70 tokens
    x.append(5, len(p4) - 64 + 1)
    seqs = [1, 2, 3, 4, 5]
    x.check_state(seqs)
    q = workloads.normal((len(seqs), H, D), 4243)
    assert x.decode(seqs, q) <= TOL_DECODE
    assert x.lib.get_error() == 0
    x.lib.close()
