"""Parity of the CUDA path with the float64 oracle (needs a B200).

Bars (written in each test): bit-exact for slot mappings, copy-on-write pairs,
tables, refcounts and KV bytes; attention max-abs error <= 1e-4 for fp32 K/V,
<= 2e-3 for bf16 decode, <= 5e-3 for bf16 prefill, all against the oracle run
on the same (bf16-rounded) inputs.
"""
import dataclasses

import numpy as np
import pytest
import torch

import paged_kv_cache_483_b200 as pa
import workloads
from harness import DeviceRun, OracleRun, q64, scaled_error

pytestmark = pytest.mark.gpu

TOL_F32, TOL_DECODE, TOL_PREFILL = 1e-4, 2e-3, 5e-3
# Relative bars: error / (attention over |V|), elementwise.  Every rounding in
# the kernels is a relative error per term p_j v_j, so the error of an output
# element is bounded by that relative error times sum_j p_j |v_j| / sum_j p_j.
# Decode: fp32 scores of exact bf16 products (~6e-5 of a score) and fp32
# sums, P carried as bf16 hi + lo (2^-16): bar 1e-3.  Prefill: P rounded to
# bf16 for PV (bf16's unit roundoff 2^-8 per weight, 3.9e-3 if every error
# aligned; the row sum l stays fp32): bar 8e-3.
REL_DECODE, REL_PREFILL = 1e-3, 8e-3


def _check_decode(g, o, w, tol, partition_tokens=0):
    out = g.decode(partition_tokens=partition_tokens)
    q = q64(w)
    worst = 0.0
    for i in range(len(w.decode_seqs)):
        rows = o.attention(i, q[i])
        for h, ref in rows.items():
            worst = max(worst, float(np.abs(out[i, h] - ref[0]).max()))
    assert worst <= tol, worst
    return out


def test_tiny_trace_fp32():
    w = workloads.tiny()
    g = DeviceRun(w).apply(w.setup)
    o = OracleRun(w).apply(w.setup)
    assert g.slots == o.slots                                 # bit-exact plan
    assert g.pool.refcounts() == o.pool.refs
    assert len(o.cows[3]) == 1                               # B's shared tail copied
    torch.cuda.synchronize()
    # whole pool, bit-exact (both sides start from zeros; no block is reused)
    assert np.array_equal(g.k_cache.cpu().numpy().astype(np.float64), o.pool.keys)
    assert np.array_equal(g.v_cache.cpu().numpy().astype(np.float64), o.pool.values)
    _check_decode(g, o, w, TOL_F32)
    assert g.pool.get_error() == 0


def _small(lens, H, Hkv, d=128, bs=16, dtype="bf16", seed=1, split_last=0):
    return workloads.custom_decode("small", lens, H, Hkv, d, bs, dtype, seed,
                                   spare_blocks=4, split_last=split_last)


LENS = [1, 15, 16, 17, 33, 100, 255, 256, 513, 1000, 0, 2]


@pytest.mark.parametrize("H,Hkv", [(32, 8), (64, 8), (8, 8), (16, 8), (4, 1), (8, 1)])
@pytest.mark.parametrize("part", [0, 16, 64, 256])
def test_decode_fast_parity(H, Hkv, part):
    w = _small(LENS, H, Hkv, seed=H * 7 + Hkv + part)
    g = DeviceRun(w).apply(w.setup)
    assert g.pool.decode_path(H) == 1
    o = OracleRun(w).apply(w.setup)
    _check_decode(g, o, w, TOL_DECODE, part)
    assert g.pool.get_error() == 0


def test_decode_uninitialised_pool_is_safe():
    # stale slots past a sequence end must not leak into the result
    w = _small([3, 17, 31], 32, 8, seed=5)
    g = DeviceRun(w, init="empty")
    g.k_cache.fill_(float("nan"))
    g.v_cache.fill_(float("inf"))
    g.apply(w.setup)
    o = OracleRun(w).apply(w.setup)
    _check_decode(g, o, w, TOL_DECODE)


def test_decode_is_invariant_under_block_permutation():
    w = _small([700, 1234, 40, 511], 32, 8, seed=11)
    outs = []
    for k in range(3):
        wk = dataclasses.replace(w, order=workloads.permutation(w.num_blocks, 100 + k))
        outs.append(DeviceRun(wk).apply(wk.setup).decode())
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_generic_path_bf16_head_dim_64():
    w = _small([5, 70, 129], 8, 2, d=64, seed=3)
    g = DeviceRun(w).apply(w.setup)
    assert g.pool.decode_path(8) == 0
    _check_decode(g, OracleRun(w).apply(w.setup), w, TOL_DECODE)


@pytest.mark.parametrize("d,bs,H,Hkv,dtype", [
    (512, 16, 4, 2, "f32"),      # the largest head_dim the generic kernel takes
    (80, 4, 6, 3, "bf16"),       # head_dim not a multiple of 32
    (128, 1, 16, 1, "bf16"),     # one-token blocks, group 16
    (128, 32, 32, 2, "bf16"),    # group 16 at head_dim 128 (beyond the fast path)
    (256, 7, 2, 2, "f32"),       # odd block size
])
def test_generic_path_edge_shapes(d, bs, H, Hkv, dtype):
    w = _small([1, 2, 31, 130, 0], H, Hkv, d=d, bs=bs, dtype=dtype, seed=d + bs + H)
    g = DeviceRun(w).apply(w.setup)
    assert g.pool.decode_path(H) == 0
    out = _check_decode(g, OracleRun(w).apply(w.setup), w,
                        TOL_F32 if dtype == "f32" else TOL_DECODE)
    assert np.all(out[4] == 0)                             # the empty sequence
    assert g.pool.get_error() == 0


def test_generic_path_fp32_gqa():
    w = _small([9, 40, 64], 8, 2, d=32, bs=8, dtype="f32", seed=4)
    g = DeviceRun(w).apply(w.setup)
    _check_decode(g, OracleRun(w).apply(w.setup), w, TOL_F32)


def test_append_with_sharing_is_bit_exact():
    # groups sharing prefixes, private tails, a copy-on-write in the step
    w = workloads.ragged256(groups=3, per_group=4, prefix=40, spare_blocks=8)
    g = DeviceRun(w).apply(w.setup + w.step)
    o = OracleRun(w).apply(w.setup + w.step)
    assert g.slots == o.slots
    assert any(o.cows.values())
    assert g.pool.refcounts() == o.pool.refs
    kc = g.k_cache.cpu().float().numpy()
    vc = g.v_cache.cpu().float().numpy()
    for s in o.pool.tables:
        for t in range(o.pool.lengths[s]):
            blk, off = o.pool.address(s, t)
            assert np.array_equal(kc[blk, off], o.pool.keys[blk, off])
            assert np.array_equal(vc[blk, off], o.pool.values[blk, off])
    _check_decode(g, o, w, TOL_DECODE)


def test_reshape_and_cache_and_cow_entry_points():
    w = workloads.custom_decode("rc", [40], 8, 8, 128, 16, "bf16", 9, spare_blocks=4)
    g = DeviceRun(w)
    T = 20
    key = torch.randn(T, 8, 128, device="cuda").to(torch.bfloat16)
    val = torch.randn(T, 8, 128, device="cuda").to(torch.bfloat16)
    slots = torch.tensor([5 * 16 + i for i in range(T - 1)] + [-1], device="cuda")
    g.pool.reshape_and_cache(key, val, slots)
    src = torch.tensor([5], dtype=torch.int32, device="cuda")
    dst = torch.tensor([2], dtype=torch.int32, device="cuda")
    g.pool.cow_copy(src, dst)
    torch.cuda.synchronize()
    flat_k = g.k_cache.view(-1, 8, 128)
    assert torch.equal(flat_k[80:80 + T - 1], key[:T - 1])
    assert torch.equal(g.k_cache[2], g.k_cache[5]) and torch.equal(g.v_cache[2], g.v_cache[5])
    assert torch.equal(g.v_cache.view(-1, 8, 128)[80:80 + T - 1], val[:T - 1])
    assert g.pool.get_error() == 0


def test_device_bounds_errors_zero_rows():
    w = _small([40, 40], 32, 8, seed=21)
    g = DeviceRun(w).apply(w.setup)
    tables, lens, _, _ = g.tables()
    q = w.queries()[:, 0].contiguous().cuda()
    bad = tables.clone()
    bad[1, 1] = w.num_blocks + 5
    out = g.pool.decode(q, bad, lens)
    assert g.pool.get_error() & pa.PA_DEVERR_BLOCK_ID
    assert torch.all(out[1] == 0) and torch.any(out[0] != 0)
    long = lens.clone()
    long[0] = tables.shape[1] * 16 + 1
    out = g.pool.decode(q, tables, long)
    assert g.pool.get_error() & pa.PA_DEVERR_KV_LEN
    assert torch.all(out[0] == 0)
    key = torch.zeros(1, 8, 128, device="cuda", dtype=torch.bfloat16)
    g.pool.reshape_and_cache(key, key, torch.tensor([w.num_blocks * 16], device="cuda"))
    assert g.pool.get_error() & pa.PA_DEVERR_SLOT
    assert g.pool.get_error() == 0                       # cleared by the read


@pytest.mark.parametrize("batch,cached,chunk,H,Hkv", [
    (2, 0, 37, 32, 8), (2, 40, 37, 32, 8), (1, 200, 130, 32, 8), (3, 5, 1, 32, 8),
    (2, 300, 129, 8, 8), (2, 17, 200, 16, 8), (2, 250, 64, 64, 8), (1, 1000, 300, 32, 8)])
@pytest.mark.parametrize("splits", [0, 1])
def test_prefill_parity_small(batch, cached, chunk, H, Hkv, splits):
    # these grids are smaller than one wave: splits=0 cuts every query tile
    # over its keys (up to 4 parts, some of them empty), splits=1 never does
    w = workloads.prefill(seed=batch * 100 + cached + chunk + H, batch=batch, cached=cached,
                          chunk=chunk, num_heads=H, num_kv_heads=Hkv)
    g = DeviceRun(w).apply(w.setup + w.step)
    assert g.pool.prefill_path(H) == 1
    o = OracleRun(w).apply(w.setup + w.step)
    out = g.prefill(max_kv_splits=splits)
    q = q64(w)
    worst = 0.0
    for i in range(batch):
        rows = o.attention(i, q[i])
        for h, ref in rows.items():
            worst = max(worst, float(np.abs(out[i, :, h] - ref).max()))
    assert worst <= TOL_PREFILL, worst
    assert g.pool.get_error() == 0


@pytest.mark.parametrize("dtype,H,Hkv,d,bs", [
    ("f32", 8, 2, 128, 16),      # fp32 pool: the 1e-4 bar
    ("f32", 4, 4, 64, 8),        # fp32, no grouping, head_dim 64
    ("bf16", 32, 2, 128, 16),    # group 16 (beyond the tensor-core kernel's 8)
    ("bf16", 8, 2, 64, 16),      # head_dim 64
    ("bf16", 6, 3, 80, 4),       # head_dim 80, block 4
])
@pytest.mark.parametrize("cached,chunk", [(0, 1), (1, 37), (130, 129)])
def test_prefill_generic_path(dtype, H, Hkv, d, bs, cached, chunk):
    # q_tokens > 1 on the CUDA-core kernel: the causal offset rule
    # j <= kv_len - q_tokens + qt for every query row of the chunk
    w = workloads.prefill(seed=d * 31 + H + cached + chunk, batch=2, cached=cached,
                          chunk=chunk, num_heads=H, num_kv_heads=Hkv, head_dim=d,
                          dtype=dtype, block_size=bs)
    g = DeviceRun(w).apply(w.setup + w.step)
    assert g.pool.prefill_path(H) == 0
    o = OracleRun(w).apply(w.setup + w.step)
    assert g.slots == o.slots
    out = g.prefill()
    q = q64(w)
    worst = 0.0
    for i in range(2):
        rows = o.attention(i, q[i])
        assert sorted(rows) == list(range(H))
        for h, ref in rows.items():
            worst = max(worst, float(np.abs(out[i, :, h] - ref).max()))
    assert worst <= (TOL_F32 if dtype == "f32" else TOL_PREFILL), worst
    assert g.pool.get_error() == 0


# ---------------------------------------------------------------- full sizes
def _full(w, kv_heads, sample_seqs, decode=True, partition_tokens=0, check_slots=True):
    g = DeviceRun(w).apply(w.setup + w.step)
    o = OracleRun(w, heads=kv_heads).apply(w.setup + w.step)
    if check_slots:
        assert g.slots == o.slots
    assert g.pool.refcounts() == o.pool.refs
    _, _, t_gpu, lens = g.tables()
    assert np.array_equal(t_gpu, o.pool.block_table(w.decode_seqs, t_gpu.shape[1]))
    q = q64(w)
    out = g.decode(partition_tokens=partition_tokens) if decode else g.prefill()
    return g, o, out, q


def test_full_decode32_sampled():
    # three sequences, every head of every KV head
    w = workloads.decode32()
    g, o, out, q = _full(w, "all", None)
    worst = rel = 0.0
    for i in (0, 13, 31):
        scale = o.attention(i, q[i], abs_values=True)
        for h, ref in o.attention(i, q[i]).items():
            worst = max(worst, float(np.abs(out[i, h] - ref[0]).max()))
            rel = max(rel, scaled_error(out[i, h], ref[0], scale[h][0]))
    assert worst <= TOL_DECODE, worst
    assert rel <= REL_DECODE, rel
    assert g.pool.get_error() == 0


def test_full_ragged256_sampled():
    w = workloads.ragged256()
    g, o, out, q = _full(w, [3], None)
    assert any(o.cows.values())
    lens = [o.pool.lengths[s] for s in w.decode_seqs]
    pick = sorted(set([int(np.argmin(lens)), int(np.argmax(lens))] + list(range(0, 256, 37))))
    worst = rel = 0.0
    for i in pick:
        scale = o.attention(i, q[i], abs_values=True)
        for h, ref in o.attention(i, q[i]).items():
            worst = max(worst, float(np.abs(out[i, h] - ref[0]).max()))
            rel = max(rel, scaled_error(out[i, h], ref[0], scale[h][0]))
    assert worst <= TOL_DECODE, worst
    assert rel <= REL_DECODE, rel
    assert g.pool.get_error() == 0


def test_full_splitk128k_sampled():
    w = workloads.splitk128k()
    g, o, out, q = _full(w, [2], None, partition_tokens=w.partition_tokens)
    worst = rel = 0.0
    for i in (0, 3):
        scale = o.attention(i, q[i], abs_values=True)
        for h, ref in o.attention(i, q[i]).items():
            worst = max(worst, float(np.abs(out[i, h] - ref[0]).max()))
            rel = max(rel, scaled_error(out[i, h], ref[0], scale[h][0]))
    assert worst <= TOL_DECODE, worst
    assert rel <= REL_DECODE, rel
    assert g.pool.get_error() == 0


def test_full_prefill_sampled():
    # KV heads 1 and 6 of sequences 0, 3 and 7: all 512 query rows of each of
    # their query heads
    w = workloads.prefill()
    g, o, out, q = _full(w, [1, 6], None, decode=False)
    worst = rel = 0.0
    for i in (0, 3, 7):
        ref = o.attention(i, q[i])
        scale = o.attention(i, q[i], abs_values=True)
        assert len(ref) == 8
        for h, r in ref.items():
            worst = max(worst, float(np.abs(out[i, :, h] - r).max()))
            rel = max(rel, scaled_error(out[i, :, h], r, scale[h]))
    assert worst <= TOL_PREFILL, worst
    assert rel <= REL_PREFILL, rel
    assert g.pool.get_error() == 0


@pytest.mark.parametrize("splits", [0, 1])
def test_prefill_device_errors_zero_rows(splits):
    w = workloads.prefill(seed=41, batch=2, cached=100, chunk=70)
    g = DeviceRun(w).apply(w.setup + w.step)
    tables, lens, _, _ = g.tables()
    q = w.queries().contiguous().cuda()
    assert g.pool.prefill_path(32) == 1
    bad = tables.clone()
    bad[1, 2] = w.num_blocks + 3
    out = g.pool.prefill_chunk(q, bad, lens, max_kv_splits=splits)
    assert g.pool.get_error() & pa.PA_DEVERR_BLOCK_ID
    assert torch.all(out[1] == 0) and torch.any(out[0] != 0)
    short = lens.clone()
    short[0] = 50                                        # fewer keys than the chunk
    out = g.pool.prefill_chunk(q, tables, short, max_kv_splits=splits)
    assert g.pool.get_error() & pa.PA_DEVERR_KV_LEN
    assert torch.all(out[0] == 0) and torch.any(out[1] != 0)
    out = g.pool.prefill_chunk(q, tables, lens, max_kv_splits=splits)   # recovers
    assert g.pool.get_error() == 0 and torch.all(torch.isfinite(out))
    assert g.pool.get_error() == 0


@pytest.mark.parametrize("splits", [0, 2, 3, 4])
def test_prefill_tail_split(splits):
    # 10 sequences x 8 KV heads x 4 query tile pairs = 320 CTAs of work: two
    # full waves on 148 SMs and a tail of 24 that is split over its keys; a
    # second call must give the same bits (the merge tickets reset themselves)
    w = workloads.prefill(seed=47, batch=10, cached=500, chunk=256)
    g = DeviceRun(w).apply(w.setup + w.step)
    o = OracleRun(w).apply(w.setup + w.step)
    out = g.prefill(max_kv_splits=splits)
    again = g.prefill(max_kv_splits=splits)
    assert np.array_equal(out, again)
    q = q64(w)
    worst = 0.0
    for i in range(10):
        for h, ref in o.attention(i, q[i]).items():
            worst = max(worst, float(np.abs(out[i, :, h] - ref).max()))
    assert worst <= TOL_PREFILL, worst
    unsplit = g.prefill(max_kv_splits=1)
    assert float(np.abs(out - unsplit).max()) <= TOL_PREFILL
    assert g.pool.get_error() == 0


def test_prefill_split_arg_checked():
    w = workloads.prefill(seed=48, batch=1, cached=20, chunk=30)
    g = DeviceRun(w).apply(w.setup + w.step)
    with pytest.raises(pa.PAError):
        g.prefill(max_kv_splits=-1)


def test_prefill_uninitialised_pool_is_safe():
    # stale slots past the sequence end (NaN / Inf bit patterns) must not leak
    w = workloads.prefill(seed=43, batch=2, cached=37, chunk=60)
    g = DeviceRun(w, init="empty")
    g.k_cache.fill_(float("nan"))
    g.v_cache.fill_(float("inf"))
    g.apply(w.setup + w.step)
    o = OracleRun(w).apply(w.setup + w.step)
    out = g.prefill()
    q = q64(w)
    worst = 0.0
    for i in range(2):
        for h, ref in o.attention(i, q[i]).items():
            worst = max(worst, float(np.abs(out[i, :, h] - ref).max()))
    assert np.isfinite(out).all()
    assert worst <= TOL_PREFILL, worst


def _fused_step(w, fused=True, init="zeros"):
    """Setup through the library, then the step's one-token appends either
    fused into the decode or as reshape_and_cache + decode."""
    g = DeviceRun(w, init=init).apply(w.setup)
    seqs = [op.args[0] for op in w.step]
    slots, cow = g.pool.plan_append(seqs, [1] * len(seqs))
    if cow:
        src = torch.tensor([c[0] for c in cow], dtype=torch.int32, device="cuda")
        dst = torch.tensor([c[1] for c in cow], dtype=torch.int32, device="cuda")
        g.pool.cow_copy(src, dst)
    ks, vs = zip(*[w.kv_for(op) for op in w.step])
    key = torch.cat(ks).cuda()
    val = torch.cat(vs).cuda()
    d_slots = torch.tensor(slots, dtype=torch.int64, device="cuda")
    tables, lens, _, _ = g.tables()
    q = w.queries()[:, 0].contiguous().cuda()
    if fused:
        out = g.pool.decode_append(q, key, val, d_slots, tables, lens)
    else:
        g.pool.reshape_and_cache(key, val, d_slots)
        out = g.pool.decode(q, tables, lens)
    torch.cuda.synchronize()
    return g, out.cpu().numpy(), slots, key, val


@pytest.mark.parametrize("H,Hkv", [(32, 8), (64, 8), (8, 8)])
def test_decode_append_matches_oracle_and_two_calls(H, Hkv):
    # new tokens land mid-block, at block starts (a fresh block) and at ends
    lens = [1, 2, 16, 17, 32, 33, 300, 513, 1024, 1025]
    w = workloads.custom_decode("fused", lens, H, Hkv, 128, 16, "bf16", seed=H + 3,
                                spare_blocks=8, split_last=1)
    g, out, slots, key, val = _fused_step(w, fused=True)
    assert g.pool.decode_path(H) == 1
    _, out2, _, _, _ = _fused_step(w, fused=False)
    assert np.array_equal(out, out2)                       # same arithmetic, same order
    o = OracleRun(w).apply(w.setup + w.step)
    assert slots == o.slots[w.step[0].index] + sum((o.slots[op.index] for op in w.step[1:]), [])
    q = q64(w)
    worst = 0.0
    for i in range(len(lens)):
        for h, ref in o.attention(i, q[i]).items():
            worst = max(worst, float(np.abs(out[i, h] - ref[0]).max()))
    assert worst <= TOL_DECODE, worst
    flat_k = g.k_cache.view(-1, Hkv, 128)
    flat_v = g.v_cache.view(-1, Hkv, 128)
    assert torch.equal(flat_k[torch.tensor(slots)], key) and torch.equal(flat_v[torch.tensor(slots)], val)
    assert g.pool.get_error() == 0


def test_decode_append_with_copy_on_write_and_stale_pool():
    w = workloads.ragged256(groups=2, per_group=4, prefix=40, spare_blocks=8)
    g, out, _, _, _ = _fused_step(w, fused=True, init="empty")
    o = OracleRun(w).apply(w.setup + w.step)
    assert any(o.cows.values())
    q = q64(w)
    worst = 0.0
    for i in range(len(w.decode_seqs)):
        for h, ref in o.attention(i, q[i]).items():
            worst = max(worst, float(np.abs(out[i, h] - ref[0]).max()))
    assert np.isfinite(out).all() and worst <= TOL_DECODE, worst
    assert g.pool.get_error() == 0


def test_decode_append_generic_path_fp32():
    w = workloads.custom_decode("fused32", [5, 16, 40], 8, 2, 32, 8, "f32", seed=8,
                                spare_blocks=4, split_last=1)
    g, out, _, _, _ = _fused_step(w, fused=True)
    assert g.pool.decode_path(8) == 0
    o = OracleRun(w).apply(w.setup + w.step)
    q = q64(w)
    worst = 0.0
    for i in range(3):
        for h, ref in o.attention(i, q[i]).items():
            worst = max(worst, float(np.abs(out[i, h] - ref[0]).max()))
    assert worst <= TOL_F32, worst
