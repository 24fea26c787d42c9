"""int8 and FP8 (E4M3) pools on the CUDA-core path (needs a B200).

Chunked prefill ("docs.rs ferrum-kv 0.4.0 src/attention.rs", paged_attention
with q_tokens > 1: query qt sees j <= kv_len - q_tokens + qt) and decode with
more than 8 query heads per KV head, over the rows such a pool stores ("vladkulikov.com
modern-llms module 9 notebook", KV quantisation experiment; the E4M3 grid for
FP8).  The kernel reads each code and its float32 scale, multiplies them in
fp32 and accumulates in fp32, so the oracle over the stored rows (float64) is
met at the fp32 bar, 1e-4, on every output row.
"""
import numpy as np
import pytest

import workloads
from harness import DeviceRun, OracleRun, q64

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.mark.parametrize("q8", [True, "fp8"])
@pytest.mark.parametrize("H,Hkv", [(32, 8), (32, 2)])
@pytest.mark.parametrize("cached,chunk", [(0, 1), (1, 37), (130, 129)])
def test_q8_prefill_every_row(q8, H, Hkv, cached, chunk):
    w = workloads.prefill(seed=7 * cached + chunk + H // Hkv, batch=2, cached=cached,
                          chunk=chunk, num_heads=H, num_kv_heads=Hkv, head_dim=128,
                          dtype="bf16", block_size=16)
    g = DeviceRun(w, q8=q8).apply(w.setup + w.step)
    assert g.pool.prefill_path(H) == 0
    o = OracleRun(w, q8=q8).apply(w.setup + w.step)
    assert g.slots == o.slots
    out = g.prefill()
    q = q64(w)
    worst = 0.0
    for i in range(2):
        rows = o.attention(i, q[i])
        assert sorted(rows) == list(range(H))
        for h, ref in rows.items():
            worst = max(worst, float(np.abs(out[i, :, h] - ref).max()))
    assert worst <= TOL, worst
    assert g.pool.get_error() == 0


@pytest.mark.parametrize("q8", [True, "fp8"])
def test_q8_decode_group_16(q8):
    # 128 query heads over 8 KV heads: above the tensor-core kernels' 8
    lens = [1, 15, 16, 17, 100, 513, 0]
    w = workloads.custom_decode("q8g16", lens, 128, 8, 128, 16, "bf16", 23, spare_blocks=4)
    g = DeviceRun(w, q8=q8).apply(w.setup)
    assert g.pool.decode_path(128) == 0
    o = OracleRun(w, q8=q8).apply(w.setup)
    out = g.decode()
    q = q64(w)
    worst = 0.0
    for i, L in enumerate(lens):
        rows = o.attention(i, q[i])
        for h, ref in rows.items():
            if L == 0:
                assert np.all(out[i, h] == 0)         # an empty cache gives zeros
            worst = max(worst, float(np.abs(out[i, h] - ref[0]).max()))
    assert worst <= TOL, worst
    assert g.pool.get_error() == 0
