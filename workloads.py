"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds no part of the method's arithmetic: it draws numbers and
writes down sequences of pool operations.  It never computes a slot, a table
entry, a score or a softmax; both the oracle and the CUDA path receive the same
arrays from here and do that work independently.

Recipe (same for every workload):
  * host integers (allocation orders, lengths) come from
    ``numpy.random.default_rng(seed)``;
  * tensors come from a seeded CPU ``torch.Generator`` drawing N(0, 1) float32,
    optionally multiplied by a scale, then rounded to bfloat16
    (round-to-nearest-even, ``Tensor.to(torch.bfloat16)``) for bf16 workloads;
    the oracle receives the same rounded values widened exactly to float64;
  * each append operation draws its own tensor from a generator seeded with
    ``seed * 1_000_003 + op_index`` so that any single sequence can be
    regenerated without drawing the rest.

Workloads (sizes of the five configurations the method is measured on):
  tiny       pool 8 x 4 slots, 1 head, head_dim 8, fp32; A gets 6 tokens, B
             shares A's 6 tokens then appends 3 (copy-on-write of the shared
             partial tail, then a fresh block); decode both.
  decode32   32 sequences x 8192 tokens, 32 query / 8 KV heads, head_dim 128,
             block 16, pool of 16384 blocks in a seeded permuted order, bf16.
  ragged256  256 sequences in 32 groups of 8 sharing a 2048-token prefix,
             lengths log-uniform in [1, 4096]; one appended token each, bf16.
  splitk128k 4 sequences x 131072 tokens, 64 query / 8 KV heads, Q scaled 0.5,
             partitions of 4096 tokens, bf16.
  prefill    8 sequences, 4096 cached tokens + a 512-token chunk attended
             causally, 32 / 8 heads, bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

SEED_TINY = 7
SEED_BASE = 20260800


def seed_for(config_index: int) -> int:
    """Seed of configuration ``config_index`` (1-based; the tiny trace uses 7)."""
    return SEED_TINY if config_index == 1 else SEED_BASE + config_index


def permutation(n: int, seed: int) -> np.ndarray:
    """A seeded permutation of ``range(n)`` as int32 (the allocation order)."""
    return np.random.default_rng(seed).permutation(n).astype(np.int32)


def normal(shape, seed: int, dtype: str = "bf16", scale: float = 1.0) -> torch.Tensor:
    """N(0, 1) * scale drawn on the CPU from ``seed``, rounded to ``dtype``.

    Returns a CPU tensor of dtype bfloat16 or float32.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    if dtype == "bf16":
        return x.to(torch.bfloat16)
    if dtype == "f32":
        return x
    raise ValueError(f"unknown dtype {dtype}")


def as_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a bf16/f32 tensor to a float64 numpy array."""
    return t.to(torch.float64).numpy()


@dataclass
class Op:
    """One pool operation: ('create', seq) | ('append', seq, n) |
    ('share', src, dst, prefix) | ('release', seq)."""
    kind: str
    args: tuple
    index: int = 0          # position in the script; seeds the append's tensor


@dataclass
class Workload:
    name: str
    num_blocks: int
    block_size: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str                      # 'bf16' or 'f32' for K, V and Q
    seed: int
    order: np.ndarray               # allocation order (permutation of num_blocks)
    setup: list = field(default_factory=list)   # untimed ops
    step: list = field(default_factory=list)    # ops of one timed step
    decode_seqs: list = field(default_factory=list)
    q_tokens: int = 1
    q_scale: float = 1.0
    partition_tokens: int = 0

    def kv_for(self, op: Op):
        """K and V of an append op: two tensors [n, num_kv_heads, head_dim]."""
        assert op.kind == "append"
        n = op.args[1]
        base = self.seed * 1_000_003 + op.index
        shape = (n, self.num_kv_heads, self.head_dim)
        return (normal(shape, 2 * base, self.dtype),
                normal(shape, 2 * base + 1, self.dtype))

    def queries(self):
        """Q [len(decode_seqs), q_tokens, num_heads, head_dim]."""
        shape = (len(self.decode_seqs), self.q_tokens, self.num_heads, self.head_dim)
        return normal(shape, self.seed * 7919 + 13, self.dtype, self.q_scale)


def _script(ops):
    return [Op(k, tuple(a), i) for i, (k, *a) in enumerate(ops)]


def tiny(seed: int = SEED_TINY) -> Workload:
    """Tiny paged trace, fp32: 8 blocks of 4 slots, 1 head, head_dim 8."""
    ops = [("create", 0), ("append", 0, 6), ("share", 0, 1, 6), ("append", 1, 3)]
    return Workload("tiny", 8, 4, 1, 1, 8, "f32", seed, permutation(8, seed),
                    setup=_script(ops), decode_seqs=[0, 1])


def decode32(seed: int = seed_for(2)) -> Workload:
    """Decode batch 32 at 8K context, GQA 32/8, head_dim 128, block 16.

    Setup caches 8191 tokens per sequence; the step appends token 8192 of every
    sequence and decodes at kv_len 8192.  The 16384-block pool is exactly full.
    """
    B, L = 32, 8192
    ops = [("create", b) for b in range(B)] + [("append", b, L - 1) for b in range(B)]
    setup = _script(ops)
    step = [Op("append", (b, 1), len(ops) + b) for b in range(B)]
    return Workload("decode32", 16384, 16, 32, 8, 128, "bf16", seed,
                    permutation(16384, seed), setup=setup, step=step,
                    decode_seqs=list(range(B)))


def ragged_lengths(n: int, seed: int, lo: int = 1, hi: int = 4096) -> np.ndarray:
    """round(exp(U(0, ln hi))) clamped to [lo, hi]."""
    u = np.random.default_rng(seed).uniform(0.0, math.log(hi), size=n)
    return np.clip(np.rint(np.exp(u)), lo, hi).astype(np.int64)


def ragged256(seed: int = seed_for(3), groups: int = 32, per_group: int = 8,
              prefix: int = 2048, spare_blocks: int = 1024) -> Workload:
    """Ragged decode batch 256 with 2048-token shared prefixes.

    Per group a root sequence writes the prefix; each member shares
    min(L_i, prefix) tokens of it, appends max(0, L_i - prefix) private tokens,
    then the root is released.  The step appends one token per member (a
    copy-on-write when the member's tail block is partial and still shared) and
    decodes at kv_len L_i + 1.
    """
    bs = 16
    B = groups * per_group
    lens = ragged_lengths(B, seed)
    ops, need = [], 0
    for g in range(groups):
        root = 100000 + g
        ops += [("create", root), ("append", root, prefix)]
        need += -(-prefix // bs)
        for m in range(per_group):
            b = g * per_group + m
            L = int(lens[b])
            ops.append(("share", root, b, min(L, prefix)))
            if L > prefix:
                ops.append(("append", b, L - prefix))
                need += -(-(L - prefix) // bs)
            need += 1   # room for a copy-on-write or a boundary block per member
        ops.append(("release", root))
    setup = _script(ops)
    step = [Op("append", (b, 1), len(ops) + b) for b in range(B)]
    nb = need + spare_blocks
    return Workload("ragged256", nb, bs, 32, 8, 128, "bf16", seed,
                    permutation(nb, seed), setup=setup, step=step,
                    decode_seqs=list(range(B)))


def splitk128k(seed: int = seed_for(4)) -> Workload:
    """Long-context split-K decode: 4 x 131072 tokens, GQA 64/8, Q scaled 0.5."""
    B, L = 4, 131072
    ops = [("create", b) for b in range(B)] + [("append", b, L) for b in range(B)]
    return Workload("splitk128k", 32768, 16, 64, 8, 128, "bf16", seed,
                    permutation(32768, seed), setup=_script(ops),
                    decode_seqs=list(range(B)), q_scale=0.5, partition_tokens=4096)


def prefill(seed: int = seed_for(5), batch: int = 8, cached: int = 4096,
            chunk: int = 512, num_heads: int = 32, num_kv_heads: int = 8,
            head_dim: int = 128, dtype: str = "bf16", block_size: int = 16) -> Workload:
    """Chunked prefill: cached tokens, then a chunk appended and attended causally."""
    bs = block_size
    ops = [("create", b) for b in range(batch)]
    ops += [("append", b, cached) for b in range(batch) if cached > 0]
    setup = _script(ops)
    step = [Op("append", (b, chunk), len(ops) + b) for b in range(batch)]
    nb = batch * (-(-(cached + chunk) // bs)) + 64
    return Workload("prefill", nb, bs, num_heads, num_kv_heads, head_dim, dtype, seed,
                    permutation(nb, seed), setup=setup, step=step,
                    decode_seqs=list(range(batch)), q_tokens=chunk)


def custom_decode(name: str, lens, num_heads: int, num_kv_heads: int, head_dim: int,
                  block_size: int, dtype: str, seed: int, spare_blocks: int = 0,
                  q_tokens: int = 1, q_scale: float = 1.0, partition_tokens: int = 0,
                  split_last: int = 0) -> Workload:
    """Independent sequences of the given lengths in a permuted pool.

    ``split_last`` > 0 moves the last ``split_last`` tokens of every sequence
    into the step (appended by the timed step rather than the setup).
    """
    lens = [int(x) for x in lens]
    nb = sum(-(-L // block_size) for L in lens) + spare_blocks
    ops = [("create", b) for b in range(len(lens))]
    ops += [("append", b, L - split_last) for b, L in enumerate(lens) if L - split_last > 0]
    setup = _script(ops)
    step = [Op("append", (b, split_last), len(ops) + b) for b in range(len(lens))] if split_last else []
    return Workload(name, max(nb, 1), block_size, num_heads, num_kv_heads, head_dim,
                    dtype, seed, permutation(max(nb, 1), seed), setup=setup, step=step,
                    decode_seqs=list(range(len(lens))), q_tokens=q_tokens,
                    q_scale=q_scale, partition_tokens=partition_tokens)


ALL = {"tiny": tiny, "decode32": decode32, "ragged256": ragged256,
       "splitk128k": splitk128k, "prefill": prefill}
