"""Sink + recent-window decode on the GPU (needs a B200) against the oracle's
``attention_window`` ("vladkulikov.com modern-llms module 9 notebook",
streaming and sliding-window caches), bf16 and int8 pools, max-abs <= 2e-3."""
import numpy as np
import pytest
import torch

import paged_kv_cache_483_b200 as pa
import workloads
from harness import DeviceRun, OracleRun, q64
from oracle import attention_window

pytestmark = pytest.mark.gpu

TOL = 2e-3
LENS = [1, 3, 15, 16, 17, 40, 100, 255, 513, 1000, 2049, 0]
WINDOWS = [(1, 0), (3, 0), (16, 0), (17, 4), (100, 16), (64, 1), (1000, 0), (5000, 0), (33, 40)]


def _oracle_window(o, w, q, window, sinks):
    G = w.num_heads // w.num_kv_heads
    res = []
    for i, seq in enumerate(w.decode_seqs):
        k, v = o.pool.gather(seq)
        rows = {}
        for kvh in range(w.num_kv_heads):
            hs = list(range(kvh * G, (kvh + 1) * G))
            out = attention_window(q[i][:, hs], k[:, kvh:kvh + 1].astype(np.float64),
                                   v[:, kvh:kvh + 1].astype(np.float64), window, sinks)
            for j, h in enumerate(hs):
                rows[h] = out[0, j]
        res.append(rows)
    return res


@pytest.mark.parametrize("q8", [False, True, "fp8"])
@pytest.mark.parametrize("part", [0, 64])
def test_window_decode_parity(q8, part):
    w = workloads.custom_decode("win", LENS, 32, 8, 128, 16, "bf16", seed=31 + part,
                                spare_blocks=4)
    g = DeviceRun(w, q8=q8).apply(w.setup)
    o = OracleRun(w, q8=q8).apply(w.setup)
    tables, lens, _, _ = g.tables()
    qd = w.queries()[:, 0].contiguous().cuda()
    q = q64(w)
    for window, sinks in WINDOWS:
        out = g.pool.decode_window(qd, tables, lens, window, sinks,
                                   partition_tokens=part).cpu().numpy()
        ref = _oracle_window(o, w, q, window, sinks)
        worst = max(float(np.abs(out[i, h] - r).max()) for i, rows in enumerate(ref)
                    for h, r in rows.items())
        assert worst <= TOL, (window, sinks, worst)
        assert np.all(out[LENS.index(0)] == 0)
    assert g.pool.get_error() == 0


@pytest.mark.parametrize("q8", [False, True, "fp8"])
def test_window_covering_everything_equals_decode(q8):
    w = workloads.custom_decode("win2", [5, 300, 1111], 32, 8, 128, 16, "bf16", seed=3,
                                spare_blocks=4)
    g = DeviceRun(w, q8=q8).apply(w.setup)
    tables, lens, _, _ = g.tables()
    qd = w.queries()[:, 0].contiguous().cuda()
    full = g.pool.decode(qd, tables, lens).cpu().numpy()
    for window, sinks in ((1111, 0), (2000, 7), (1, 1200)):
        got = g.pool.decode_window(qd, tables, lens, window, sinks).cpu().numpy()
        assert np.array_equal(got, full)                 # same blocks, same order


def test_window_stale_slots_and_errors():
    w = workloads.custom_decode("win3", [7, 70, 400], 32, 8, 128, 16, "bf16", seed=5,
                                spare_blocks=4)
    g = DeviceRun(w, init="empty")
    g.k_cache.fill_(float("nan"))
    g.v_cache.fill_(float("inf"))
    g.apply(w.setup)
    o = OracleRun(w).apply(w.setup)
    tables, lens, _, _ = g.tables()
    qd = w.queries()[:, 0].contiguous().cuda()
    out = g.pool.decode_window(qd, tables, lens, 20, 3).cpu().numpy()
    ref = _oracle_window(o, w, q64(w), 20, 3)
    assert np.isfinite(out).all()
    assert max(float(np.abs(out[i, h] - r).max()) for i, rows in enumerate(ref)
               for h, r in rows.items()) <= TOL
    with pytest.raises(pa.PAError) as e:
        g.pool.decode_window(qd, tables, lens, 0, 3)
    assert e.value.code == 1
    bad = tables.clone()
    bad[2, -1] = w.num_blocks + 1                          # inside the window
    out = g.pool.decode_window(qd, bad, lens, 20, 3)
    assert g.pool.get_error() & pa.PA_DEVERR_BLOCK_ID and torch.all(out[2] == 0)
    assert g.pool.get_error() == 0


@pytest.mark.parametrize("shape", [
    ("f32", 8, 2, 32, 8, False),      # fp32 pool, head_dim 32, block 8
    ("f32", 6, 3, 80, 4, False),      # head_dim 80, block 4
    ("bf16", 128, 8, 128, 16, True),  # int8 pool, group 16
    ("bf16", 128, 8, 128, 16, "fp8"), # FP8 pool, group 16
])
def test_window_on_generic_path(shape):
    # shapes outside the tensor-core kernels: the CUDA-core kernel walks the
    # visible keys only, fp32 arithmetic, every row at 1e-4
    dtype, H, Hkv, d, bs, q8 = shape
    w = workloads.custom_decode("win4", LENS, H, Hkv, d, bs, dtype, seed=4 + H + d,
                                spare_blocks=4)
    g = DeviceRun(w, q8=q8).apply(w.setup)
    assert g.pool.decode_path(H) == 0
    o = OracleRun(w, q8=q8).apply(w.setup)
    tables, lens, _, _ = g.tables()
    qd = w.queries()[:, 0].contiguous().cuda()
    q = q64(w)
    for window, sinks in WINDOWS:
        out = g.pool.decode_window(qd, tables, lens, window, sinks).cpu().numpy()
        ref = _oracle_window(o, w, q, window, sinks)
        worst = max(float(np.abs(out[i, h] - r).max()) for i, rows in enumerate(ref)
                    for h, r in rows.items())
        assert worst <= 1e-4, (window, sinks, worst)
        assert np.all(out[LENS.index(0)] == 0)
    assert g.pool.get_error() == 0


def test_window_append_on_generic_path_equals_two_calls():
    # the new token's append, then the windowed decode (group 16, int8 pool)
    w = workloads.custom_decode("win5", [5, 40, 300], 128, 8, 128, 16, "bf16", seed=5,
                                spare_blocks=4, split_last=1)
    a = DeviceRun(w, q8=True).apply(w.setup)
    b = DeviceRun(w, q8=True).apply(w.setup)
    seqs = [op.args[0] for op in w.step]
    slots, _ = a.pool.plan_append(seqs, [1] * len(seqs))
    slots_b, _ = b.pool.plan_append(seqs, [1] * len(seqs))
    assert slots == slots_b
    ks, vs = zip(*[w.kv_for(op) for op in w.step])
    key, val = torch.cat(ks).cuda(), torch.cat(vs).cuda()
    d_slots = torch.tensor(slots, dtype=torch.int64, device="cuda")
    tables, lens, _, _ = a.tables()
    q = w.queries()[:, 0].contiguous().cuda()
    fused = a.pool.decode_window_append(q, key, val, d_slots, tables, lens, 17, 4)
    b.pool.reshape_and_cache(key, val, d_slots)
    two = b.pool.decode_window(q, tables, lens, 17, 4)
    assert torch.equal(fused, two)
    assert a.pool.get_error() == 0 and b.pool.get_error() == 0


@pytest.mark.parametrize("q8", [False, True, "fp8"])
def test_full_decode32_window_sampled(q8):
    # 32 x 8192 with a 1024-token window and 4 sinks: three sequences, two KV heads
    w = workloads.decode32()
    g = DeviceRun(w, q8=q8).apply(w.setup)
    o = OracleRun(w, heads=[1, 6], q8=q8).apply(w.setup)
    tables, lens, _, _ = g.tables()
    qd = w.queries()[:, 0].contiguous().cuda()
    out = g.pool.decode_window(qd, tables, lens, 1024, 4).cpu().numpy()
    q = q64(w)
    G = w.num_heads // w.num_kv_heads
    worst = 0.0
    for i in (0, 17, 31):
        k, v = o.pool.gather(w.decode_seqs[i])
        for j, kvh in enumerate(o.heads):
            hs = list(range(kvh * G, (kvh + 1) * G))
            ref = attention_window(q[i][:, hs], k[:, j:j + 1].astype(np.float64),
                                   v[:, j:j + 1].astype(np.float64), 1024, 4)
            worst = max(worst, float(np.abs(out[i, hs] - ref[0]).max()))
    assert worst <= TOL, worst
    assert g.pool.get_error() == 0


@pytest.mark.parametrize("q8", [False, True, "fp8"])
@pytest.mark.parametrize("part", [0, 32])
def test_window_append_equals_two_calls(q8, part):
    # the fused step (write the new token, decode over the window) against
    # reshape_and_cache followed by decode_window, and against the oracle
    lens = [1, 2, 16, 17, 40, 300, 1000]
    w = workloads.custom_decode("winf", lens, 32, 8, 128, 16, "bf16", seed=13 + part,
                                spare_blocks=8, split_last=1)
    windows = [(1, 0), (17, 4), (100, 16), (2000, 0)]
    outs = {}
    for fused in (True, False):
        g = DeviceRun(w, q8=q8).apply(w.setup)
        seqs = [op.args[0] for op in w.step]
        slots, cow = g.pool.plan_append(seqs, [1] * len(seqs))
        assert not cow
        ks, vs = zip(*[w.kv_for(op) for op in w.step])
        key, val = torch.cat(ks).cuda(), torch.cat(vs).cuda()
        d_slots = torch.tensor(slots, dtype=torch.int64, device="cuda")
        tables, tl, _, _ = g.tables()
        q = w.queries()[:, 0].contiguous().cuda()
        if not fused:
            g.pool.reshape_and_cache(key, val, d_slots)
        for window, sinks in windows:
            if fused:
                out = g.pool.decode_window_append(q, key, val, d_slots, tables, tl, window,
                                                  sinks, partition_tokens=part)
            else:
                out = g.pool.decode_window(q, tables, tl, window, sinks, partition_tokens=part)
            outs[fused, window, sinks] = out.cpu().numpy()
        assert g.pool.get_error() == 0
    o = OracleRun(w, q8=q8).apply(w.setup + w.step)
    qq = q64(w)
    for window, sinks in windows:
        assert np.array_equal(outs[True, window, sinks], outs[False, window, sinks])
        ref = _oracle_window(o, w, qq, window, sinks)
        worst = max(float(np.abs(outs[True, window, sinks][i, h] - r).max())
                    for i, rows in enumerate(ref) for h, r in rows.items())
        assert worst <= TOL, (window, sinks, worst)


def test_window_append_argument_errors():
    w = workloads.custom_decode("winf2", [5, 40], 32, 8, 128, 16, "bf16", seed=2,
                                spare_blocks=4, split_last=1)
    g = DeviceRun(w).apply(w.setup)
    seqs = [op.args[0] for op in w.step]
    slots, _ = g.pool.plan_append(seqs, [1] * len(seqs))
    ks, vs = zip(*[w.kv_for(op) for op in w.step])
    key, val = torch.cat(ks).cuda(), torch.cat(vs).cuda()
    d_slots = torch.tensor(slots, dtype=torch.int64, device="cuda")
    tables, tl, _, _ = g.tables()
    q = w.queries()[:, 0].contiguous().cuda()
    for window, sinks in ((0, 0), (4, -1)):
        with pytest.raises(pa.PAError) as e:
            g.pool.decode_window_append(q, key, val, d_slots, tables, tl, window, sinks)
        assert e.value.code == 1
    bad = d_slots.clone()
    bad[1] = w.num_blocks * 16                            # one past the pool
    out = g.pool.decode_window_append(q, key, val, bad, tables, tl, 8, 2)
    assert g.pool.get_error() & pa.PA_DEVERR_SLOT
    assert torch.all(torch.isfinite(out))
    assert g.pool.get_error() == 0
