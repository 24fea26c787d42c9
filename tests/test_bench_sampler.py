"""The bench's CPU-baseline sampler (host logic, no GPU): for every pool type
and window it must compute exactly what the oracle computes on the stored
rows, so that its outputs can check the timed GPU step and its byte count is
the metric's."""
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402
from oracle import KVPool, attention_two_pass, attention_window  # noqa: E402
from oracle import stored_rows, stored_rows_fp8  # noqa: E402


def _direct(w, q8, window, sinks):
    rows = {"int8": stored_rows, "fp8": stored_rows_fp8}.get(q8)
    p = KVPool(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.order,
               store_heads="all", dtype=np.float64)
    for op in w.setup + w.step:
        if op.kind == "create":
            p.create(op.args[0])
        elif op.kind == "share":
            p.share_prefix(*op.args)
        elif op.kind == "release":
            p.release(op.args[0])
        else:
            k, v = (t.double().numpy() for t in w.kv_for(op))
            if rows:
                k, v = rows(k)[2], rows(v)[2]
            p.append(op.args[0], op.args[1], k, v)
    q = w.queries().to(torch.float64).numpy()
    out = []
    for i, seq in enumerate(w.decode_seqs):
        k, v = p.gather(seq)
        out.append(attention_window(q[i], k, v, window, sinks) if window
                   else attention_two_pass(q[i], k, v))
    return out, [p.lengths[s] for s in w.decode_seqs]


@pytest.mark.parametrize("q8", [False, "int8", "fp8"])
@pytest.mark.parametrize("window,sinks", [(0, 0), (5, 2), (40, 0)])
def test_sampler_matches_the_oracle(q8, window, sinks):
    w = workloads.custom_decode("smp", [3, 17, 40, 90], 8, 2, 16, 4, "bf16", seed=5,
                                spare_blocks=4, split_last=1)
    s = bench.OracleSampler(w, q8, window, sinks)
    n = len(w.decode_seqs)
    work, spent, done = s.run(1e9, max_units=n, keep=n)
    assert done == n and spent > 0
    want, lens = _direct(w, q8, window, sinks)
    for i in range(n):
        np.testing.assert_allclose(s.outs[i], want[i], rtol=0, atol=1e-12)
    vis = [min(L, window + sinks) if window else L for L in lens]
    per_tok = (2 * w.head_dim + 8) if q8 else 2 * w.head_dim * 2
    assert work == sum(vis) * w.num_kv_heads * per_tok
    assert work == bench.decode_bytes(w, np.array(lens), bool(q8), window, sinks)


def test_metric_names_follow_the_options():
    w = workloads.custom_decode("smp2", [5], 8, 2, 16, 4, "bf16", seed=1, spare_blocks=2)
    assert bench.metric_name(w) == \
        "decode KV HBM GB/s (fraction of B200 peak) and seqs/s at 8K ctx, GQA 32/8"
    assert bench.metric_name(w, "fp8", 1024, 4).startswith("decode fp8-KV HBM GB/s")
    assert bench.metric_name(w, False, 1024, 4).endswith("window 1024 + 4 sinks (visible keys only)")
