"""Replays a workload script on the GPU library and on the oracle.

Both sides receive the same seeded arrays from ``workloads``; neither sees the
other's results.  The oracle side stores data for a chosen subset of KV heads
(float32 holding bf16-exact values) so full-size configurations fit in host
memory; its attention then runs on the matching query heads.
"""
from __future__ import annotations

import numpy as np
import torch

import paged_kv_cache_483_b200 as pa
import workloads
from oracle import KVPool, stored_rows, stored_rows_fp8


def torch_dtype(w):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


class DeviceRun:
    def __init__(self, w, device="cuda", init="zeros", q8=False):
        """q8: True / "int8" for an int8 pool, "fp8" for an FP8 (E4M3) pool
        (packed (block, head) records), fed the same bf16 rows."""
        self.w = w
        alloc = torch.zeros if init == "zeros" else torch.empty
        if q8:
            self.records = alloc((w.num_blocks, w.num_kv_heads, pa.PA_INT8_RECORD_BYTES),
                                 dtype=torch.uint8, device=device)
            self.pool = pa.Pool(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim,
                                "fp8" if q8 == "fp8" else "int8", self.records, None,
                                alloc_order=w.order)
        else:
            dt = torch_dtype(w)
            shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
            self.k_cache = alloc(shape, dtype=dt, device=device)
            self.v_cache = alloc(shape, dtype=dt, device=device)
            self.pool = pa.Pool(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim,
                                w.dtype, self.k_cache, self.v_cache, alloc_order=w.order)
        self.slots = {}
        self.device = device

    def apply(self, ops):
        for op in ops:
            if op.kind == "create":
                self.pool.create(op.args[0])
            elif op.kind == "share":
                self.pool.fork(*op.args)
            elif op.kind == "release":
                self.pool.release(op.args[0])
            elif op.kind == "append":
                k, v = self.w.kv_for(op)
                self.slots[op.index] = self.pool.append_kv(
                    [op.args[0]], [op.args[1]], k.to(self.device), v.to(self.device),
                    return_slots=True)
            else:
                raise ValueError(op.kind)
        return self

    def tables(self, seqs=None):
        seqs = self.w.decode_seqs if seqs is None else seqs
        width = max(len(self.pool.table(s)[0]) for s in seqs)
        t, lens = self.pool.block_tables(seqs, max(width, 1))
        return (torch.from_numpy(t).to(self.device), torch.from_numpy(lens).to(self.device),
                t, lens)

    def decode(self, q=None, partition_tokens=0):
        q = self.w.queries() if q is None else q
        tables, lens, _, _ = self.tables()
        out = self.pool.decode(q[:, 0].contiguous().to(self.device), tables, lens,
                               partition_tokens=partition_tokens)
        torch.cuda.synchronize()
        return out.cpu().numpy()

    def prefill(self, q=None, max_kv_splits=0):
        q = self.w.queries() if q is None else q
        tables, lens, _, _ = self.tables()
        out = self.pool.prefill_chunk(q.contiguous().to(self.device), tables, lens,
                                      max_kv_splits=max_kv_splits)
        torch.cuda.synchronize()
        return out.cpu().numpy()


class OracleRun:
    def __init__(self, w, heads="all", q8=False):
        """q8: True / "int8" / "fp8": store each row as that pool reads it
        back (value of the code x float32 scale, float64)."""
        self.w = w
        self.q8 = q8
        self.heads = list(range(w.num_kv_heads)) if heads == "all" else list(heads)
        self.pool = KVPool(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim,
                           w.order, store_heads=self.heads,
                           dtype=np.float64 if (w.dtype == "f32" or q8) else np.float32)
        self.slots, self.cows = {}, {}

    def apply(self, ops):
        for op in ops:
            if op.kind == "create":
                self.pool.create(op.args[0])
            elif op.kind == "share":
                self.pool.share_prefix(*op.args)
            elif op.kind == "release":
                self.pool.release(op.args[0])
            elif op.kind == "append":
                k, v = self.w.kv_for(op)
                dt = self.pool.keys.dtype
                k64, v64 = k.to(torch.float64).numpy(), v.to(torch.float64).numpy()
                if self.q8:        # the rows an int8 / FP8 pool reads back
                    rows = stored_rows_fp8 if self.q8 == "fp8" else stored_rows
                    k64, v64 = rows(k64)[2], rows(v64)[2]
                s, c = self.pool.append(op.args[0], op.args[1], k64.astype(dt), v64.astype(dt))
                self.slots[op.index], self.cows[op.index] = s, c
        return self

    def attention(self, seq_index, q, heads=None, abs_values=False):
        """Output of query rows q [q_tokens, H, d] (float64) for the decode
        sequence at position seq_index, restricted to query heads whose KV head
        is stored.  Returns {h: out[q_tokens, d]}.  abs_values: the same
        attention over |V|, i.e. sum_j p_j |v_j| / sum_j p_j, the scale that
        every per-term relative rounding error of the kernels is bounded by."""
        w = self.w
        G = w.num_heads // w.num_kv_heads
        seq = w.decode_seqs[seq_index]
        k, v = self.pool.gather(seq)
        if abs_values:
            v = np.abs(v)
        res = {}
        for i, kvh in enumerate(self.heads):
            hs = list(range(kvh * G, (kvh + 1) * G)) if heads is None else \
                [h for h in heads if h // G == kvh]
            if not hs:
                continue
            from oracle import attention_two_pass
            out = attention_two_pass(q[:, hs], k[:, i:i + 1].astype(np.float64),
                                     v[:, i:i + 1].astype(np.float64))
            for j, h in enumerate(hs):
                res[h] = out[:, j]
        return res


def q64(w):
    return w.queries().to(torch.float64).numpy()


def scaled_error(out, ref, scale):
    """max |out - ref| / scale, elementwise (scale = attention over |V|)."""
    return float((np.abs(out - ref) / np.maximum(scale, 1e-30)).max())
