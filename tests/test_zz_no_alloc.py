"""pa_decode_static_scratch: decode for callers that cannot allocate.

A serving process that gives all device memory to its KV pool and weights at
start-up, or a plugin whose host framework owns the device allocator, cannot
hand pa_decode a workspace for its split-K partitions.  The static-scratch
entry point takes that scratch from a fixed device array inside the library
instead.  These checks call it through the C ABI and compare it with
pa_decode given a caller workspace, on two calls in a row (the array keeps the
first call's contents): both run the same kernels with the same partitions, so
the results must be identical bit for bit, at a given partition size and at
the automatic one.  A warm call must not change the device's free memory, and
a request larger than the array is refused with PA_ERR_SCRATCH_LIMIT.

The file is named so that pytest collects it last.
"""
import ctypes as C
import math

import pytest
import torch

import paged_kv_cache_483_b200 as pa
import workloads
from harness import DeviceRun

pytestmark = pytest.mark.gpu

PA_ERR_SCRATCH_LIMIT = 10


def _call(L, g, q, tables, lens, part, out):
    return L.pa_decode_static_scratch(
        g.pool.handle, C.c_void_p(q.data_ptr()), q.shape[0], q.shape[1],
        C.c_void_p(tables.data_ptr()), tables.shape[1], C.c_void_p(lens.data_ptr()),
        C.c_float(1.0 / math.sqrt(128)), part, C.c_void_p(out.data_ptr()),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("part", [256, 0])     # 0: the library picks the partitions
def test_static_scratch_matches_workspace_decode_twice(part):
    w = workloads.custom_decode("noalloc", [700, 1234, 40, 4097, 1, 0, 333], 64, 8, 128, 16,
                                "bf16", seed=99, spare_blocks=4)
    g = DeviceRun(w).apply(w.setup)
    tables, lens, _, _ = g.tables()
    q = w.queries()[:, 0].contiguous().cuda()
    # several partitions per sequence in both cases, so the scratch is used
    assert g.pool.decode_workspace_bytes(q.shape[0], q.shape[1], tables.shape[1], part) > 0
    ref = g.pool.decode(q, tables, lens, partition_tokens=part)
    torch.cuda.synchronize()
    L = pa.lib()
    outs = [torch.full_like(ref, float("nan")) for _ in range(2)]
    free_after = []
    for out in outs:
        assert _call(L, g, q, tables, lens, part, out) == 0
        torch.cuda.synchronize()
        free_after.append(torch.cuda.mem_get_info()[0])
        assert torch.equal(out, ref)               # same kernels, same partitions
    # the first call may load the library's module on this device; the
    # second allocates nothing
    assert free_after[1] == free_after[0]
    assert g.pool.get_error() == 0


def test_static_scratch_refuses_oversized_requests():
    w = workloads.custom_decode("noalloc_big", [64] * 8, 64, 8, 128, 16, "bf16", seed=5,
                                spare_blocks=4)
    g = DeviceRun(w).apply(w.setup)
    q = w.queries()[:, 0].contiguous().cuda()
    wide = torch.zeros((8, 4096), dtype=torch.int32, device="cuda")
    lens = torch.full((8,), 64, dtype=torch.int32, device="cuda")
    need = g.pool.decode_workspace_bytes(8, 64, 4096, 16)
    assert need > (16 << 20)
    out = torch.zeros((8, 64, 128), dtype=torch.float32, device="cuda")
    assert _call(pa.lib(), g, q, wide, lens, 16, out) == PA_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0          # nothing was launched
    assert g.pool.get_error() == 0
