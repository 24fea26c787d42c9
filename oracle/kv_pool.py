"""Oracle block manager: a refcounted physical KV pool with copy-on-write.

Test infrastructure only (see the package header).  Restates:
  * "abhik.ai examples/pagedattention.py", ``KVPool``: a fixed pool of
    ``num_blocks`` blocks of ``block_size`` slots; allocation claims the first
    free id in a fixed permutation (region physical_pool / ``_allocate``);
    address = divmod(token, block_size) through the table (region
    logical_address); a write into a shared partial tail first copies the whole
    block into a freshly allocated one (region copy_on_write); release returns
    blocks whose refcount reaches zero (region release_sequence).
  * "vladkulikov.com modern-llms module 9 notebook", ``PagedKVPool``: a
    multi-token append is preflighted (blocks needed = [shared partial tail] +
    ceil(tokens beyond the tail's room / block_size)) so exhaustion changes
    nothing; ``share_prefix`` shares ceil(prefix / block_size) blocks; the fill
    of a physical block is the maximum over its sharers; ``snapshot`` and
    ``validate`` as on that page.

Reading taken where the two pages differ: allocation follows the first page
(first free id in ``allocation_order``); with the identity order this gives
the ids printed by the second page's trace.  Data, when stored, is float64
(or float32 holding bf16-exact values) laid out [block, slot, kv_head, dim].
"""
from __future__ import annotations

import heapq
import math

import numpy as np


class PoolError(ValueError):
    """Invalid request: unknown or duplicate sequence, bad prefix, bad shape."""


class PoolExhausted(MemoryError):
    """Not enough free blocks; raised before any state changes."""


class KVPool:
    """The physical pool, its tables and refcounts ("abhik.ai examples/pagedattention.py", ``KVPool``; the
    multi-token append, sharing and accounting of "vladkulikov.com modern-llms module 9 notebook",
    ``PagedKVPool``)."""

    def __init__(self, num_blocks, block_size, num_kv_heads=1, head_dim=1,
                 allocation_order=None, store_heads="all", dtype=np.float64):
        for name, v in (("num_blocks", num_blocks), ("block_size", block_size),
                        ("num_kv_heads", num_kv_heads), ("head_dim", head_dim)):
            if int(v) != v or v <= 0:
                raise PoolError(f"{name} must be a positive integer")
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        self.num_kv_heads, self.head_dim = int(num_kv_heads), int(head_dim)
        order = list(range(self.num_blocks)) if allocation_order is None \
            else [int(x) for x in allocation_order]
        if sorted(order) != list(range(self.num_blocks)):
            raise PoolError("allocation_order must be a permutation of the block ids")
        self.order = order
        self._rank = {blk: r for r, blk in enumerate(order)}
        # free ids kept as a heap of their positions in the allocation order:
        # popping the smallest position is "first free id in the order".
        self._free_heap = list(range(self.num_blocks))
        self._free = set(range(self.num_blocks))
        self.refs = [0] * self.num_blocks
        # references held outside the sequence tables (a prefix cache), per block
        self.external: dict = {}
        self.tables: dict = {}
        self.lengths: dict = {}
        if store_heads is None:
            self.heads = []
        elif store_heads == "all":
            self.heads = list(range(self.num_kv_heads))
        else:
            self.heads = [int(h) for h in store_heads]
        self._hidx = {h: i for i, h in enumerate(self.heads)}
        shape = (self.num_blocks, self.block_size, len(self.heads), self.head_dim)
        self.keys = np.zeros(shape, dtype) if self.heads else None
        self.values = np.zeros(shape, dtype) if self.heads else None

    # -- allocation ("abhik.ai ... KVPool._allocate") -----------------------
    def _allocate(self):
        if not self._free:
            raise PoolExhausted("physical KV pool exhausted")
        blk = self.order[heapq.heappop(self._free_heap)]
        self._free.remove(blk)
        self.refs[blk] = 1
        if self.keys is not None:          # the first page zero-fills on claim
            self.keys[blk] = 0
            self.values[blk] = 0
        return blk

    def _give_back(self, blk):
        self._free.add(blk)
        heapq.heappush(self._free_heap, self._rank[blk])
        if self.keys is not None:          # and on release
            self.keys[blk] = 0
            self.values[blk] = 0

    def _require(self, seq):
        if seq not in self.tables:
            raise PoolError(f"unknown or released sequence {seq!r}")

    # -- sequences ----------------------------------------------------------
    def create(self, seq):
        """Empty table; no block reserved ("abhik.ai ... KVPool.create")."""
        if seq in self.tables:
            raise PoolError(f"duplicate sequence {seq!r}")
        self.tables[seq] = []
        self.lengths[seq] = 0

    def blocks_needed(self, seq, n):
        """Preflight count ("vladkulikov.com ... _blocks_needed_for_append")."""
        self._require(seq)
        if n == 0:
            return 0
        length, table = self.lengths[seq], self.tables[seq]
        used = length % self.block_size
        room, need = 0, 0
        if table and used:
            room = self.block_size - used
            if self.refs[table[-1]] > 1:
                need += 1
        beyond = max(0, n - room)
        return need + math.ceil(beyond / self.block_size)

    def append(self, seq, n, keys=None, values=None):
        """Append ``n`` tokens; returns (slot_mapping, cow_pairs).

        Preflight first (second page); then a shared partial tail is made
        private by copying the whole block (first page, copy_on_write); then
        tokens are written one by one at divmod(position, block_size), a fresh
        block being claimed at every block boundary (first page, append).
        ``keys``/``values``: arrays [n, num_kv_heads, head_dim] or None.
        """
        self._require(seq)
        n = int(n)
        if n < 0:
            raise PoolError("token count must be non-negative")
        if keys is not None:
            keys = np.asarray(keys)
            values = np.asarray(values)
            want = (n, self.num_kv_heads, self.head_dim)
            if keys.shape != want or values.shape != want:
                raise PoolError(f"keys/values must have shape {want}")
        need = self.blocks_needed(seq, n)
        if need > len(self._free):
            raise PoolExhausted(f"need {need} free blocks, {len(self._free)} remain")
        table = self.tables[seq]
        slots, cow = [], []
        if n and table and self.lengths[seq] % self.block_size and self.refs[table[-1]] > 1:
            old = table[-1]
            new = self._allocate()
            if self.keys is not None:
                self.keys[new] = self.keys[old]
                self.values[new] = self.values[old]
            table[-1] = new
            self.refs[old] -= 1
            cow.append((old, new))
        for i in range(n):
            pos = self.lengths[seq]
            logical, offset = divmod(pos, self.block_size)
            if offset == 0:
                table.append(self._allocate())
            blk = table[logical]
            if keys is not None and self.heads:
                self.keys[blk, offset] = keys[i][self.heads]
                self.values[blk, offset] = values[i][self.heads]
            slots.append(blk * self.block_size + offset)
            self.lengths[seq] = pos + 1
        return slots, cow

    def share_prefix(self, src, dst, prefix):
        """New sequence ``dst`` sharing the blocks of ``src``'s first ``prefix``
        tokens ("vladkulikov.com ... PagedKVPool.share_prefix")."""
        self._require(src)
        prefix = int(prefix)
        if prefix < 0 or prefix > self.lengths[src]:
            raise PoolError("prefix exceeds the source length")
        if dst in self.tables:
            raise PoolError(f"duplicate sequence {dst!r}")
        shared = self.tables[src][:math.ceil(prefix / self.block_size)]
        for blk in shared:
            self.refs[blk] += 1
        self.tables[dst] = list(shared)
        self.lengths[dst] = prefix

    def fork(self, parent, child):
        """Share the parent's whole table ("abhik.ai ... KVPool.fork")."""
        self._require(parent)
        self.share_prefix(parent, child, self.lengths[parent])

    def release(self, seq):
        """Drop one reference per block; zero-ref blocks become free
        ("abhik.ai ... KVPool.release")."""
        self._require(seq)
        for blk in self.tables[seq]:
            self.refs[blk] -= 1
            if self.refs[blk] == 0:
                self._give_back(blk)
        del self.tables[seq]
        del self.lengths[seq]

    def truncate(self, seq, length):
        """Keep the first ``length`` tokens of ``seq`` (a rollback of its
        newest tokens).  Not on the pages; it is the pages' release applied
        to the dropped tail ("abhik.ai ... KVPool.release"): every block
        wholly past ``length`` loses this sequence's reference and is freed at
        zero, and the result equals share_prefix(seq, tmp, length) followed by
        release(seq), with tmp then named seq.  A kept partial block stays as
        it is, so a copy-on-write already made is not undone."""
        self._require(seq)
        length = int(length)
        if length < 0 or length > self.lengths[seq]:
            raise PoolError("length must lie within the sequence")
        table = self.tables[seq]
        keep = math.ceil(length / self.block_size)
        for blk in table[keep:]:
            self.refs[blk] -= 1
            if self.refs[blk] == 0:
                self._give_back(blk)
        del table[keep:]
        self.lengths[seq] = length

    # -- addressing ("abhik.ai ... region logical_address") -------------------
    def address(self, seq, token):
        """(block, offset) of a live token: divmod(token, block_size) through
        the table ("abhik.ai examples/pagedattention.py", region logical_address)."""
        self._require(seq)
        if not 0 <= token < self.lengths[seq]:
            raise PoolError("token index must address a live token")
        logical, offset = divmod(token, self.block_size)
        return self.tables[seq][logical], offset

    def slot(self, seq, token):
        """Flat slot block * block_size + offset: the slot mapping the append
        writes through ("docs.rs ferrum-kv 0.4.0 src/attention.rs"'s per-token layout stored block by block)."""
        blk, off = self.address(seq, token)
        return blk * self.block_size + off

    def gather(self, seq, kv_len=None):
        """Live K, V rows in logical order: two arrays [kv_len, stored heads, d]
        ("abhik.ai examples/pagedattention.py", the gather of ``KVPool.attention``)."""
        self._require(seq)
        n = self.lengths[seq] if kv_len is None else int(kv_len)
        k = np.empty((n, len(self.heads), self.head_dim), self.keys.dtype)
        v = np.empty_like(k)
        for t in range(n):
            blk, off = self.address(seq, t)
            k[t] = self.keys[blk, off]
            v[t] = self.values[blk, off]
        return k, v

    def block_table(self, seqs, width=None, pad=0):
        """Tables of ``seqs`` as an int32 matrix padded with ``pad`` (the block
        tables "docs.rs ferrum-kv 0.4.0 src/attention.rs"'s ``paged_attention`` reads, one row per sequence)."""
        width = width or max([len(self.tables[s]) for s in seqs] + [1])
        out = np.full((len(seqs), width), pad, np.int32)
        for i, s in enumerate(seqs):
            t = self.tables[s]
            out[i, :len(t)] = t
        return out

    # -- accounting ("vladkulikov.com ... _refresh_fills, snapshot") -----------
    def fills(self):
        """Live slots per physical block: the largest fill any sharer gives it
        ("vladkulikov.com modern-llms module 9 notebook", ``PagedKVPool._refresh_fills``; "abhik.ai examples/pagedattention.py", the
        ownership snapshot's occupied slots); a block a prefix cache maps is
        full."""
        fill = [0] * self.num_blocks
        for blk in self.external:              # blocks a prefix cache maps are full
            fill[blk] = self.block_size
        for seq, table in self.tables.items():
            length = self.lengths[seq]
            for j, blk in enumerate(table):
                fill[blk] = max(fill[blk], min(self.block_size, length - j * self.block_size))
        return fill

    @property
    def free_blocks(self):
        """Number of free physical blocks ("vladkulikov.com modern-llms module 9 notebook", ``free_blocks``)."""
        return len(self._free)

    def snapshot(self):
        """The second page's state summary (its key names)."""
        fill = self.fills()
        allocated = self.num_blocks - len(self._free)
        payload = sum(f for b, f in enumerate(fill) if self.refs[b])
        logical = sum(self.lengths.values())
        capacity = allocated * self.block_size
        return {
            "sequences": {str(s): {"length": self.lengths[s], "blocks": list(self.tables[s])}
                          for s in sorted(self.tables, key=repr)},
            "allocated_blocks": allocated,
            "free_blocks": len(self._free),
            "physical_capacity_tokens": capacity,
            "physical_payload_tokens": payload,
            "logical_tokens": logical,
            "internal_waste_tokens": capacity - payload,
            "sharing_savings_tokens": logical - payload,
        }

    def ownership(self):
        """The first page's per-event figures (``KVPool.snapshot``)."""
        occupied = {}
        for seq, table in self.tables.items():
            for j, blk in enumerate(table):
                filled = min(self.block_size, self.lengths[seq] - j * self.block_size)
                occupied[blk] = max(occupied.get(blk, 0), filled)
        live = sum(occupied.values())
        return {"tables": {s: list(t) for s, t in self.tables.items()},
                "lengths": dict(self.lengths), "refs": list(self.refs),
                "free": sorted(self._free),
                "logical_live_slots": sum(self.lengths.values()),
                "unique_live_slots": live, "unique_blocks": len(occupied),
                "tail_waste_slots": len(occupied) * self.block_size - live}

    def validate(self):
        """The second page's invariants (``PagedKVPool.validate``)."""
        if len(self._free) != len(self._free_heap):
            raise AssertionError("free heap and free set disagree")
        expect = [0] * self.num_blocks
        for seq, table in self.tables.items():
            length = self.lengths[seq]
            if length < 0:
                raise AssertionError("negative length")
            if len(table) != math.ceil(length / self.block_size):
                raise AssertionError("table length does not match sequence length")
            if len(set(table)) != len(table):
                raise AssertionError("a sequence references a block twice")
            for blk in table:
                if not 0 <= blk < self.num_blocks:
                    raise AssertionError("invalid block id in a table")
                expect[blk] += 1
        for blk, cnt in self.external.items():
            expect[blk] += cnt
        fill = self.fills()
        for blk in range(self.num_blocks):
            if self.refs[blk] != expect[blk]:
                raise AssertionError("refcount does not match the tables")
            if self.refs[blk] == 0:
                if blk not in self._free or fill[blk] != 0:
                    raise AssertionError("unreferenced block not clean and free")
            else:
                if blk in self._free:
                    raise AssertionError("referenced block on the free list")
                if not 1 <= fill[blk] <= self.block_size:
                    raise AssertionError("referenced block has an invalid fill")
        snap = self.snapshot()
        # a block only a prefix cache holds is payload no live sequence counts
        held = set(b for table in self.tables.values() for b in table)
        cache_only = sum(self.block_size for b in self.external if b not in held)
        if snap["logical_tokens"] + cache_only < snap["physical_payload_tokens"]:
            raise AssertionError("physical payload exceeds logical payload")
