"""FP8 (E4M3) KV pools on the GPU (needs a B200): the quantising append
against the oracle's E4M3 codes and float32 scales, bit for bit; the decode
against the oracle's attention over the rows the pool reads back, within
the bf16 decode bar (2e-3).  The per-row absmax recipe is the one of
"vladkulikov.com modern-llms module 9 notebook" (KV quantisation
experiment) on the E4M3 grid of the OCP 8-bit floating point
specification."""
import numpy as np
import pytest
import torch

import paged_kv_cache_483_b200 as pa
import workloads
from harness import DeviceRun, OracleRun, q64
from oracle import e4m3_values, stored_rows_fp8
from test_gpu_q8 import _pool_rows, _worst

pytestmark = pytest.mark.gpu

TOL_DECODE = 2e-3


def _small(lens, H, Hkv, seed=1, split_last=0, spare=4):
    return workloads.custom_decode("f8", lens, H, Hkv, 128, 16, "bf16", seed,
                                   spare_blocks=spare, split_last=split_last)


def _codes(g, slot):
    kc, ks, vc, vs = _pool_rows(g, slot)
    return kc.view(np.uint8), ks, vc.view(np.uint8), vs


def test_fp8_append_codes_and_scales_bit_exact():
    w = _small([1, 15, 16, 17, 100, 300], 32, 8, seed=3)
    g = DeviceRun(w, q8="fp8").apply(w.setup)
    torch.cuda.synchronize()
    n = 0
    for op in w.setup:
        if op.kind != "append":
            continue
        k, v = w.kv_for(op)
        kc, ks, _ = stored_rows_fp8(k.to(torch.float64).numpy())
        vc, vs, _ = stored_rows_fp8(v.to(torch.float64).numpy())
        for t, slot in enumerate(g.slots[op.index]):
            gkc, gks, gvc, gvs = _codes(g, slot)
            assert np.array_equal(gkc, kc[t]) and np.array_equal(gvc, vc[t])
            assert np.array_equal(gks, ks[t]) and np.array_equal(gvs, vs[t])
            n += 1
    assert n == sum([1, 15, 16, 17, 100, 300])
    assert g.pool.get_error() == 0


def test_fp8_append_special_rows():
    # a zero row (scale 1, codes 0) and a row whose absmax is 448 (scale 1)
    # holding exact E4M3 ties and subnormals
    w = _small([2], 8, 8, seed=4)
    g = DeviceRun(w, q8="fp8")
    g.pool.create(0)
    k = torch.zeros(2, 8, 128, dtype=torch.bfloat16)
    vals = [448.0, 1.0625, 432.0, 400.0, 2.0 ** -10, 3 * 2.0 ** -10, -1.0625, -(2.0 ** -11),
            -448.0, 1.1875, -0.0]
    k[1, :, :len(vals)] = torch.tensor(vals)
    v = k.clone()
    slots = g.pool.append_kv([0], [2], k.cuda(), v.cuda(), return_slots=True)
    torch.cuda.synchronize()
    z = _codes(g, slots[0])
    assert np.all(z[0] == 0) and np.all(z[1] == 1.0) and np.all(z[2] == 0)
    row = _codes(g, slots[1])
    assert np.all(row[1] == 1.0)
    assert row[0][0, :len(vals)].tolist() == [0x7E, 0x38, 0x7E, 0x7C, 0x00, 0x02, 0xB8, 0x00,
                                              0xFE, 0x3A, 0x00]
    assert np.array_equal(row[2], row[0])


LENS = [1, 15, 16, 17, 33, 100, 255, 256, 513, 1000, 0, 2]


@pytest.mark.parametrize("H,Hkv", [(32, 8), (64, 8), (8, 8), (16, 8), (8, 1), (24, 8), (48, 8)])
@pytest.mark.parametrize("part", [0, 16, 256])
def test_fp8_decode_parity(H, Hkv, part):
    w = _small(LENS, H, Hkv, seed=H * 7 + Hkv + part)
    g = DeviceRun(w, q8="fp8").apply(w.setup)
    assert g.pool.decode_path(H) == 1
    o = OracleRun(w, q8="fp8").apply(w.setup)
    worst, out = _worst(g, o, w, part)
    assert worst <= TOL_DECODE, worst
    assert np.all(out[LENS.index(0)] == 0)
    assert g.pool.get_error() == 0


def test_fp8_stale_slots_hold_nan_codes():
    # never-written slots hold the E4M3 NaN code (0x7F) and NaN / Inf scales;
    # dead tokens must add exactly nothing
    w = _small([3, 17, 31, 64], 32, 8, seed=6)
    g = DeviceRun(w, q8="fp8", init="empty")
    g.records.fill_(0x7F)
    sc = g.records[:, :, 4096:].view(torch.float32)
    sc[:, :, :16].fill_(float("nan"))
    sc[:, :, 16:].fill_(float("inf"))
    g.apply(w.setup)
    o = OracleRun(w, q8="fp8").apply(w.setup)
    worst, out = _worst(g, o, w)
    assert np.isfinite(out).all() and worst <= TOL_DECODE, worst
    assert np.isnan(e4m3_values()[0x7F])


def test_fp8_decode_with_sharing_and_copy_on_write():
    w = workloads.ragged256(groups=3, per_group=4, prefix=40, spare_blocks=16)
    g = DeviceRun(w, q8="fp8").apply(w.setup + w.step)
    o = OracleRun(w, q8="fp8").apply(w.setup + w.step)
    assert any(o.cows.values())
    worst, _ = _worst(g, o, w)
    assert worst <= TOL_DECODE, worst
    assert g.pool.refcounts() == o.pool.refs
    assert g.pool.get_error() == 0


def test_fp8_within_grid_bound_of_bf16_decode():
    # every stored element is within 2^-4 of its value (relative), so the
    # decode stays within that of the unquantised one
    w = _small([64, 300, 1000, 2048], 32, 8, seed=7)
    out_f8 = DeviceRun(w, q8="fp8").apply(w.setup).decode()
    out_bf = DeviceRun(w).apply(w.setup).decode()
    for i in range(4):
        rel = np.linalg.norm(out_f8[i] - out_bf[i]) / np.linalg.norm(out_bf[i])
        assert rel < 2.0 ** -4, rel


def test_fp8_two_calls_equal_decode_append():
    lens = [1, 16, 17, 300]
    w = workloads.custom_decode("f8f", lens, 32, 8, 128, 16, "bf16", seed=9,
                                spare_blocks=8, split_last=1)
    outs = []
    for fused in (True, False):
        g = DeviceRun(w, q8="fp8").apply(w.setup)
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
    o = OracleRun(w, q8="fp8").apply(w.setup + w.step)
    qq = q64(w)
    worst = 0.0
    for i in range(len(lens)):
        for h, ref in o.attention(i, qq[i]).items():
            worst = max(worst, float(np.abs(outs[0][i, h] - ref[0]).max()))
    assert worst <= TOL_DECODE, worst


def test_fp8_device_errors_and_shape_limits():
    w = _small([40, 70], 32, 8, seed=10)
    g = DeviceRun(w, q8="fp8").apply(w.setup)
    tables, lens, _, _ = g.tables()
    q = w.queries()[:, 0].contiguous().cuda()
    bad = tables.clone()
    bad[1, 1] = w.num_blocks + 5
    out = g.pool.decode(q, bad, lens)
    assert g.pool.get_error() & pa.PA_DEVERR_BLOCK_ID
    assert torch.all(out[1] == 0) and torch.any(out[0] != 0)
    assert g.pool.get_error() == 0
    assert g.pool.decode_path(128) == 0   # group 16 > 8: CUDA-core path (test_gpu_q8_generic.py)
    with pytest.raises(pa.PAError):                          # block 16, head_dim 128 only
        pa.Pool(4, 8, 1, 128, "fp8",
                torch.zeros(4, 1, pa.PA_INT8_RECORD_BYTES, dtype=torch.uint8, device="cuda"), None)


def test_full_decode32_fp8_sampled():
    w = workloads.decode32()
    g = DeviceRun(w, q8="fp8").apply(w.setup)
    o = OracleRun(w, heads=[2, 7], q8="fp8").apply(w.setup)
    out = g.decode()
    q = q64(w)
    worst = 0.0
    for i in (0, 11, 31):
        for h, ref in o.attention(i, q[i]).items():
            worst = max(worst, float(np.abs(out[i, h] - ref[0]).max()))
    assert worst <= TOL_DECODE, worst
    assert g.pool.get_error() == 0
