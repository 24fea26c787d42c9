"""int8 KV pools on the GPU (needs a B200): the quantising append against the
oracle's codes and float32 scales, bit for bit; the int8 decode against the
oracle's attention over the rows the pool reads back, within the bf16 decode
bar (2e-3); and the page's own bound against the unquantised decode (relative
error < 3 %, "vladkulikov.com modern-llms module 9 notebook", KV
quantisation experiment)."""
import numpy as np
import pytest
import torch

import paged_kv_cache_483_b200 as pa
import workloads
from harness import DeviceRun, OracleRun, q64
from oracle import stored_rows

pytestmark = pytest.mark.gpu

TOL_DECODE = 2e-3


def _small(lens, H, Hkv, seed=1, split_last=0, spare=4):
    return workloads.custom_decode("q8", lens, H, Hkv, 128, 16, "bf16", seed,
                                   spare_blocks=spare, split_last=split_last)


def _worst(g, o, w, partition_tokens=0):
    out = g.decode(partition_tokens=partition_tokens)
    q = q64(w)
    worst = 0.0
    for i in range(len(w.decode_seqs)):
        for h, ref in o.attention(i, q[i]).items():
            worst = max(worst, float(np.abs(out[i, h] - ref[0]).max()))
    return worst, out


def _expect_rows(g, w, ops):
    """Codes and scales each appended row should have, keyed by slot."""
    want = {}
    for op in ops:
        if op.kind != "append":
            continue
        k, v = w.kv_for(op)
        kc, ks, _ = stored_rows(k.to(torch.float64).numpy())
        vc, vs, _ = stored_rows(v.to(torch.float64).numpy())
        for t, slot in enumerate(g.slots[op.index]):
            want[slot] = (kc[t], ks[t], vc[t], vs[t])
    return want


def _pool_rows(g, slot):
    """(K codes, K scales, V codes, V scales) of a slot, every head, read
    from the packed records: K chunks stored swizzled, V d-major."""
    blk, tok = divmod(slot, 16)
    rec = g.records[blk].cpu().numpy()                      # [Hkv, record]
    Hkv = rec.shape[0]
    kc = np.empty((Hkv, 128), np.int8)
    for ch in range(8):
        pos = tok * 128 + ((ch ^ (tok & 7)) << 4)
        kc[:, ch * 16:(ch + 1) * 16] = rec[:, pos:pos + 16].view(np.int8)
    vc = rec[:, 2048 + np.arange(128) * 16 + tok].view(np.int8)
    ks = rec[:, 4096:4160].copy().view(np.float32)[:, tok]
    vs = rec[:, 4160:4224].copy().view(np.float32)[:, tok]
    return kc, ks, vc, vs


def test_q8_append_codes_and_scales_bit_exact():
    w = _small([1, 15, 16, 17, 100, 300], 32, 8, seed=3)
    g = DeviceRun(w, q8=True).apply(w.setup)
    torch.cuda.synchronize()
    want = _expect_rows(g, w, w.setup)
    assert len(want) == sum([1, 15, 16, 17, 100, 300])
    for slot, (kc, ks, vc, vs) in want.items():
        gkc, gks, gvc, gvs = _pool_rows(g, slot)
        assert np.array_equal(gkc, kc) and np.array_equal(gvc, vc)
        assert np.array_equal(gks, ks) and np.array_equal(gvs, vs)
    assert g.pool.get_error() == 0


def test_q8_append_special_rows():
    # a zero row (scale 1, codes 0), exact half-way ties (round half to even)
    # and a row whose absmax is negative
    w = _small([3], 8, 8, seed=4)
    g = DeviceRun(w, q8=True)
    g.pool.create(0)
    k = torch.zeros(3, 8, 128, dtype=torch.bfloat16)
    k[1, :, 0] = 127.0
    k[1, :, 1:7] = torch.tensor([2.5, -3.5, 0.5, -0.5, 1.5, -1.5])
    k[2] = torch.randn(8, 128).to(torch.bfloat16)
    k[2, :, 5] = -1000.0
    v = -k
    slots = g.pool.append_kv([0], [3], k.cuda(), v.cuda(), return_slots=True)
    torch.cuda.synchronize()
    kc, ks, _ = stored_rows(k.to(torch.float64).numpy())
    for t, slot in enumerate(slots):
        gkc, gks, gvc, gvs = _pool_rows(g, slot)
        assert np.array_equal(gkc, kc[t]) and np.array_equal(gks, ks[t])
        assert np.array_equal(gvc, -kc[t]) and np.array_equal(gvs, ks[t])
    assert np.all(_pool_rows(g, slots[0])[0] == 0) and np.all(_pool_rows(g, slots[0])[1] == 1.0)
    assert _pool_rows(g, slots[1])[0][0, :7].tolist() == [127, 2, -4, 0, 0, 2, -2]
    assert np.all(_pool_rows(g, slots[2])[0][:, 5] == -127)


LENS = [1, 15, 16, 17, 33, 100, 255, 256, 513, 1000, 0, 2]


@pytest.mark.parametrize("H,Hkv", [(32, 8), (64, 8), (8, 8), (16, 8), (8, 1), (24, 8), (48, 8)])
@pytest.mark.parametrize("part", [0, 16, 64, 256])
def test_q8_decode_parity(H, Hkv, part):
    w = _small(LENS, H, Hkv, seed=H * 5 + Hkv + part)
    g = DeviceRun(w, q8=True).apply(w.setup)
    assert g.pool.decode_path(H) == 1
    o = OracleRun(w, q8=True).apply(w.setup)
    worst, out = _worst(g, o, w, part)
    assert worst <= TOL_DECODE, worst
    assert np.all(out[LENS.index(0)] == 0)                 # empty sequence: zero rows
    assert g.pool.get_error() == 0


def test_q8_decode_with_sharing_and_copy_on_write():
    # shared prefixes, a released root, one-token appends that copy shared
    # partial tails (codes and scales must both move)
    w = workloads.ragged256(groups=3, per_group=4, prefix=40, spare_blocks=16)
    g = DeviceRun(w, q8=True).apply(w.setup + w.step)
    o = OracleRun(w, q8=True).apply(w.setup + w.step)
    assert any(o.cows.values())
    worst, _ = _worst(g, o, w)
    assert worst <= TOL_DECODE, worst
    assert g.pool.refcounts() == o.pool.refs
    assert g.pool.get_error() == 0


def test_q8_stale_slots_do_not_leak():
    # never-written slots hold arbitrary codes and NaN / Inf scales
    w = _small([3, 17, 31, 64], 32, 8, seed=6)
    g = DeviceRun(w, q8=True, init="empty")
    g.records.random_(0, 256)
    sc = g.records[:, :, 4096:].view(torch.float32)         # every scale slot
    sc[:, :, :16].fill_(float("nan"))
    sc[:, :, 16:].fill_(float("inf"))
    g.apply(w.setup)
    o = OracleRun(w, q8=True).apply(w.setup)
    worst, out = _worst(g, o, w)
    assert np.isfinite(out).all() and worst <= TOL_DECODE, worst


def test_q8_within_page_bound_of_bf16_decode():
    w = _small([64, 300, 1000, 2048], 32, 8, seed=7)
    out_q8 = DeviceRun(w, q8=True).apply(w.setup).decode()
    out_bf = DeviceRun(w).apply(w.setup).decode()
    for i in range(4):
        rel = np.linalg.norm(out_q8[i] - out_bf[i]) / np.linalg.norm(out_bf[i])
        assert rel < 0.03, rel


def test_q8_two_calls_equal_decode_append():
    lens = [1, 16, 17, 300]
    w = workloads.custom_decode("q8f", lens, 32, 8, 128, 16, "bf16", seed=9,
                                spare_blocks=8, split_last=1)
    outs = []
    for fused in (True, False):
        g = DeviceRun(w, q8=True).apply(w.setup)
        seqs = [op.args[0] for op in w.step]
        slots, cow = g.pool.plan_append(seqs, [1] * len(seqs))
        assert not cow
        ks, vs = zip(*[w.kv_for(op) for op in w.step])
        key, val = torch.cat(ks).cuda(), torch.cat(vs).cuda()
        d_slots = torch.tensor(slots, dtype=torch.int64, device="cuda")
        tables, tl, _, _ = g.tables()
        q = w.queries()[:, 0].contiguous().cuda()
        if fused:
            out = g.pool.decode_append(q, key, val, d_slots, tables, tl)
        else:
            g.pool.reshape_and_cache(key, val, d_slots)
            out = g.pool.decode(q, tables, tl)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy())
    assert np.array_equal(outs[0], outs[1])
    o = OracleRun(w, q8=True).apply(w.setup + w.step)
    q = q64(w)
    worst = 0.0
    for i in range(len(lens)):
        for h, ref in o.attention(i, q[i]).items():
            worst = max(worst, float(np.abs(outs[0][i, h] - ref[0]).max()))
    assert worst <= TOL_DECODE, worst


def test_q8_device_errors_zero_rows():
    w = _small([40, 70], 32, 8, seed=10)
    g = DeviceRun(w, q8=True).apply(w.setup)
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
    assert g.pool.get_error() == 0


def test_q8_pool_shape_limits():
    # group 16 and chunked prefill take the CUDA-core path (tests/test_gpu_q8_generic.py);
    # the pool itself needs block 16 and head_dim 128
    w = _small([20], 128, 8, seed=11)
    g = DeviceRun(w, q8=True).apply(w.setup)
    assert g.pool.decode_path(128) == 0
    with pytest.raises(pa.PAError):                       # int8 pools need block 16, d 128
        pa.Pool(4, 8, 1, 128, "int8",
                torch.zeros(4, 1, pa.PA_INT8_RECORD_BYTES, dtype=torch.uint8, device="cuda"), None)


def test_full_decode32_int8_sampled():
    # the bench configuration (32 x 8192, GQA 32/8) over an int8 pool; the
    # oracle stores two KV heads and checks three sequences against them
    w = workloads.decode32()
    g = DeviceRun(w, q8=True).apply(w.setup)
    o = OracleRun(w, heads=[0, 5], q8=True).apply(w.setup)
    out = g.decode()
    q = q64(w)
    worst = 0.0
    for i in (0, 13, 31):
        for h, ref in o.attention(i, q[i]).items():
            worst = max(worst, float(np.abs(out[i, h] - ref[0]).max()))
    assert worst <= TOL_DECODE, worst
    assert g.pool.get_error() == 0
