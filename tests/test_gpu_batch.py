"""The prepared decode batch (pa_batch_*) on a B200.

A batch step is the serving decode step in one call: plan one token per
sequence on the host manager ("abhik.ai examples/pagedattention.py", KVPool
append and copy-on-write; "vladkulikov.com modern-llms module 9 notebook",
the preflight), upload plan, changed table entries, queries and new K/V,
copy shared partial tails, write and attend ("docs.rs ferrum-kv 0.4.0
src/attention.rs", paged_attention with q_tokens = 1), download the output.

Checks, over several steps with copies-on-write, block boundaries and a
rollback: tables and lengths bit-exact against the oracle pool; outputs
identical to the same step issued as separate calls on a second pool (same
kernels, same partitions) and within 2e-3 of the oracle (the bf16 decode bar).
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_483_b200 as pa
import workloads
from harness import DeviceRun, OracleRun, q64

pytestmark = pytest.mark.gpu

TOL_DECODE = 2e-3


def _workload(kind):
    # lengths that sit mid-block, one short of a boundary and on a boundary;
    # sequence 9 shares 20 tokens of sequence 2 (a partial tail: the first
    # step copies it)
    lens = [1, 15, 40, 16, 47, 300, 511, 2]
    w = workloads.custom_decode("batch", lens, 32, 8, 128, 16, "bf16", seed=71,
                                spare_blocks=64)
    w.setup.append(workloads.Op("share", (2, 9, 20), len(w.setup)))
    w.decode_seqs.append(9)
    return w


def _step_inputs(w, step):
    n = len(w.decode_seqs)
    q = workloads.normal((n, w.num_heads, w.head_dim), 9000 + step)
    k = workloads.normal((n, w.num_kv_heads, w.head_dim), 9100 + step)
    v = workloads.normal((n, w.num_kv_heads, w.head_dim), 9200 + step)
    return q, k, v


@pytest.mark.parametrize("kind", ["bf16", "int8", "fp8"])
def test_batch_steps_match_separate_calls_and_oracle(kind):
    w = _workload(kind)
    q8 = kind if kind != "bf16" else False
    g = DeviceRun(w, q8=q8).apply(w.setup)           # the batch path
    r = DeviceRun(w, q8=q8).apply(w.setup)           # the same step as separate calls
    o = OracleRun(w, q8=q8).apply(w.setup)
    seqs = w.decode_seqs
    mb = 40
    batch = pa.Batch(g.pool, seqs, w.num_heads, mb)
    n = len(seqs)
    h_out = torch.empty((n, w.num_heads, w.head_dim), dtype=torch.float32).pin_memory()
    for step in range(4):
        q, k, v = _step_inputs(w, step)
        hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
        batch.step(hq, hk, hv, h_out)
        batch.sync()
        got = h_out.numpy().copy()
        # the reference path: plan, copy-on-write, fused append + decode
        slots, cow = r.pool.plan_append(seqs, [1] * n)
        if cow:
            src = torch.tensor([c[0] for c in cow], dtype=torch.int32, device="cuda")
            dst = torch.tensor([c[1] for c in cow], dtype=torch.int32, device="cuda")
            r.pool.cow_copy(src, dst)
        # tables as wide as the batch's (the automatic partitions follow the width)
        t, lens = r.pool.block_tables(seqs, mb)
        ref = r.pool.decode_append(q.cuda(), k.cuda(), v.cuda(),
                                   torch.tensor(slots, dtype=torch.int64, device="cuda"),
                                   torch.from_numpy(t).cuda(),
                                   torch.from_numpy(lens).cuda()).cpu().numpy()
        assert np.array_equal(got, ref), step
        # the oracle: same plan, same rows, attention over the gathered cache
        for i, s in enumerate(seqs):
            kk, vv = k[i:i + 1].double().numpy(), v[i:i + 1].double().numpy()
            if q8:
                from oracle import stored_rows, stored_rows_fp8
                rows = stored_rows_fp8 if q8 == "fp8" else stored_rows
                kk, vv = rows(kk)[2], rows(vv)[2]
            o_slots, _ = o.pool.append(s, 1, kk.astype(o.pool.keys.dtype),
                                       vv.astype(o.pool.keys.dtype))
            assert o_slots == [slots[i]]
        assert g.pool.refcounts() == o.pool.refs
        for s in seqs:
            assert g.pool.table(s) == (o.pool.tables[s], o.pool.lengths[s])
        qd = q.to(torch.float64).numpy()
        worst = 0.0
        for i in range(n):
            ref_o = o.attention(i, qd[i:i + 1])
            for h, val in ref_o.items():
                worst = max(worst, float(np.abs(got[i, h] - val[0]).max()))
        assert worst <= TOL_DECODE, (step, worst)
        if step == 1:
            # drafted tokens rejected: every sequence gives its last token back
            batch.rollback()
            keep = [r.pool.table(s)[1] - 1 for s in seqs]
            r.pool.truncate(seqs, keep)
            for s, kl in zip(seqs, keep):
                o.pool.truncate(s, kl)
            assert g.pool.table(seqs[0]) == (o.pool.tables[seqs[0]], o.pool.lengths[seqs[0]])
    assert g.pool.get_error() == 0
    batch.close()


def test_batch_rejects_a_full_table():
    w = workloads.custom_decode("batchfull", [32, 5], 8, 8, 128, 16, "bf16", seed=3,
                                spare_blocks=8)
    g = DeviceRun(w).apply(w.setup)
    batch = pa.Batch(g.pool, [0, 1], 8, 2)           # sequence 0 fills its 2 blocks
    q, k, v = (workloads.normal((2, 8, 128), s) for s in (1, 2, 3))
    out = torch.empty((2, 8, 128), dtype=torch.float32)
    before = g.pool.table(0)
    with pytest.raises(pa.PAError) as e:
        batch.step(q, k[:, :8], v[:, :8], out)
    assert e.value.code == 1
    assert g.pool.table(0) == before                 # nothing was planned
    batch.close()


@pytest.mark.parametrize("kind", ["bf16", "int8"])
def test_batch_window_steps_match_separate_calls_and_oracle(kind):
    """pa_batch_set_window: later steps decode over 5 sink tokens and the last
    40 ("vladkulikov.com modern-llms module 9 notebook", streaming_keep_indices
    with budget = sinks + window); then full attention again."""
    from oracle import attention_window
    w = _workload(kind)
    q8 = kind if kind != "bf16" else False
    g = DeviceRun(w, q8=q8).apply(w.setup)
    r = DeviceRun(w, q8=q8).apply(w.setup)
    o = OracleRun(w, q8=q8).apply(w.setup)
    seqs = w.decode_seqs
    mb, window, sinks = 40, 40, 5
    batch = pa.Batch(g.pool, seqs, w.num_heads, mb)
    batch.set_window(window, sinks)
    n = len(seqs)
    G = w.num_heads // w.num_kv_heads
    h_out = torch.empty((n, w.num_heads, w.head_dim), dtype=torch.float32).pin_memory()
    for step in range(3):
        if step == 2:
            batch.set_window(0)                      # back to full attention
        q, k, v = _step_inputs(w, step)
        batch.step(q.pin_memory(), k.pin_memory(), v.pin_memory(), h_out)
        batch.sync()
        got = h_out.numpy().copy()
        slots, cow = r.pool.plan_append(seqs, [1] * n)
        if cow:
            src = torch.tensor([c[0] for c in cow], dtype=torch.int32, device="cuda")
            dst = torch.tensor([c[1] for c in cow], dtype=torch.int32, device="cuda")
            r.pool.cow_copy(src, dst)
        t, lens = r.pool.block_tables(seqs, mb)
        args = (q.cuda(), k.cuda(), v.cuda(), torch.tensor(slots, dtype=torch.int64, device="cuda"),
                torch.from_numpy(t).cuda(), torch.from_numpy(lens).cuda())
        ref = (r.pool.decode_window_append(*args, window, sinks) if step < 2
               else r.pool.decode_append(*args)).cpu().numpy()
        assert np.array_equal(got, ref), step
        for i, s in enumerate(seqs):
            kk, vv = k[i:i + 1].double().numpy(), v[i:i + 1].double().numpy()
            if q8:
                from oracle import stored_rows
                kk, vv = stored_rows(kk)[2], stored_rows(vv)[2]
            o.pool.append(s, 1, kk.astype(o.pool.keys.dtype), vv.astype(o.pool.keys.dtype))
        qd = q.to(torch.float64).numpy()
        worst = 0.0
        for i, s in enumerate(seqs):
            kc, vc = o.pool.gather(s)
            for j, kvh in enumerate(o.heads):
                hs = list(range(kvh * G, (kvh + 1) * G))
                win = window if step < 2 else 10 ** 9
                ref_o = attention_window(qd[i:i + 1][:, hs], kc[:, j:j + 1].astype(np.float64),
                                         vc[:, j:j + 1].astype(np.float64), win,
                                         sinks if step < 2 else 0)
                worst = max(worst, float(np.abs(got[i, hs] - ref_o[0]).max()))
        assert worst <= TOL_DECODE, (step, worst)
    assert g.pool.get_error() == 0
    batch.close()


def test_batch_upload_paths_agree():
    """The step's uploads take one kernel that reads pinned, mapped host
    buffers, or one copy per buffer for pageable or unaligned ones: both give
    the same tables and bit-identical outputs."""
    w = _workload("bf16")
    runs = [DeviceRun(w).apply(w.setup) for _ in range(2)]
    seqs = w.decode_seqs
    n, mb = len(seqs), 40
    batches = [pa.Batch(r.pool, seqs, w.num_heads, mb) for r in runs]
    outs = [torch.empty((n, w.num_heads, w.head_dim), dtype=torch.float32).pin_memory(),
            torch.empty((n, w.num_heads, w.head_dim), dtype=torch.float32)]
    for step in range(3):
        q, k, v = _step_inputs(w, step)
        # the host buffers stay referenced until the steps are synchronised
        pinned = (q.pin_memory(), k.pin_memory(), v.pin_memory())
        # pageable K/V and a pinned query 8 bytes off a 16-byte boundary
        buf = torch.empty(q.numel() + 4, dtype=q.dtype).pin_memory()
        q_off = buf[4:4 + q.numel()].view(q.shape)
        q_off.copy_(q)
        assert q_off.data_ptr() % 16 == 8
        other = (q_off, k.clone(), v.clone())
        batches[0].step(*pinned, outs[0])
        batches[1].step(*other, outs[1])
        for b in batches:
            b.sync()
        assert np.array_equal(outs[0].numpy(), outs[1].numpy()), step
        for s in seqs:
            assert runs[0].pool.table(s) == runs[1].pool.table(s)
    for r in runs:
        assert r.pool.get_error() == 0
    for b in batches:
        b.close()


def test_batch_pipelined_steps_deliver_every_output():
    """Steps queued back to back with one sync at the end (each download is
    queued by the next step call or by the sync), and a last step completed
    by closing the batch: every output equals the same step run with a sync
    after each call."""
    w = _workload("bf16")
    runs = [DeviceRun(w).apply(w.setup) for _ in range(2)]
    seqs = w.decode_seqs
    n, mb, steps = len(seqs), 40, 5
    shape = (n, w.num_heads, w.head_dim)
    inputs = [tuple(t.pin_memory() for t in _step_inputs(w, s)) for s in range(steps)]
    piped = [torch.full(shape, float("nan")).pin_memory() for _ in range(steps)]
    ref = [torch.empty(shape, dtype=torch.float32).pin_memory() for _ in range(steps)]
    a = pa.Batch(runs[0].pool, seqs, w.num_heads, mb)
    for s in range(steps - 1):
        a.step(*inputs[s], piped[s])
    a.sync()
    a.step(*inputs[steps - 1], piped[steps - 1])
    a.close()                                        # completes the last download
    b = pa.Batch(runs[1].pool, seqs, w.num_heads, mb)
    for s in range(steps):
        b.step(*inputs[s], ref[s])
        b.sync()
    b.close()
    for s in range(steps):
        assert np.array_equal(piped[s].numpy(), ref[s].numpy()), s
    for r in runs:
        assert r.pool.get_error() == 0
