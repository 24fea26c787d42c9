"""The C ABI loads without a GPU, exports every declared symbol, and its host
block manager makes exactly the oracle's decisions (tables, slot mappings,
copy-on-write pairs, refcounts, snapshot figures, error codes)."""
import os
import re

import numpy as np
import torch
import pytest

import paged_kv_cache_483_b200 as pa
import workloads
from oracle import KVPool, PoolError, PoolExhausted

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = pa.lib()
    names = _declared_symbols()
    assert len(names) >= 20
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(pa.EXPORTS)


def test_status_strings():
    L = pa.lib()
    for code in range(10):
        assert L.pa_status_string(code)


def test_host_only_pool_rejects_device_calls():
    p = pa.Pool(4, 4, 1, 8, "f32")
    with pytest.raises(pa.PAError) as e:
        pa._check(pa.lib().pa_append_kv(p.handle, None, None, 0, None, None, None, None),
                  "append")
    assert e.value.code == 8


def test_create_rejects_bad_arguments():
    L = pa.lib()
    import ctypes as C
    h = C.c_void_p()
    assert L.pa_pool_create(0, 4, 1, 8, 0, None, None, None, C.byref(h)) == 1
    bad = np.array([0, 0, 1, 2], np.int32)
    assert L.pa_pool_create(4, 4, 1, 8, 0, None, None, bad.ctypes.data_as(pa._PI32),
                            C.byref(h)) == 1


def test_quantised_and_layered_creation_checks():
    # argument checks that return before any device call
    L = pa.lib()
    import ctypes as C
    h = C.c_void_p()
    fake = C.c_void_p(16)                       # never dereferenced: rejected first
    for fn in (L.pa_pool_create_int8, L.pa_pool_create_fp8):
        assert fn(4, 8, 1, 128, fake, None, C.byref(h)) == 7      # block_size != 16
        assert fn(4, 16, 1, 64, fake, None, C.byref(h)) == 7      # head_dim != 128
        assert fn(4, 16, 1, 128, None, None, C.byref(h)) == 1     # no records
        assert h.value is None
    # quantised dtypes only through their own entry points or the layered one
    for dt in (pa.PA_INT8, pa.PA_FP8, 9):
        assert L.pa_pool_create(4, 16, 1, 128, dt, None, None, None, C.byref(h)) == 1
    assert L.pa_pool_create_layers(4, 16, 1, 128, 9, 2, fake, fake, None, C.byref(h)) == 1
    assert L.pa_pool_create_layers(4, 16, 1, 128, pa.PA_FP8, 0, fake, None, None,
                                   C.byref(h)) == 1                # no layers
    assert L.pa_pool_create_layers(4, 16, 1, 128, pa.PA_FP8, 2, fake, fake, None,
                                   C.byref(h)) == 1                # records take no v_cache
    assert L.pa_pool_create_layers(4, 8, 1, 128, pa.PA_FP8, 2, fake, None, None,
                                   C.byref(h)) == 7


def test_window_calls_reject_bad_arguments_on_host_pools():
    # a host-only pool answers NO_DEVICE before looking at device pointers
    p = pa.Pool(4, 16, 1, 128, "bf16")
    L = pa.lib()
    assert L.pa_decode_window(p.handle, None, 1, 1, None, 1, None, 1.0, 4, 0, 0, None, 0, None,
                              None) == 8
    assert L.pa_decode_window_append(p.handle, None, None, None, None, 1, 1, None, 1, None, 1.0,
                                     4, 0, 0, None, 0, None, None) == 8
    assert L.pa_decode_window_workspace_bytes(p.handle, 1, 1, 4, 0, 0, 0) == 0   # window < 1


def test_static_scratch_decode_answers_no_device_on_host_pools():
    # answered before the scratch array's address is looked up, so no CUDA
    # call runs (on a host without a GPU it would fail with PA_ERR_CUDA)
    p = pa.Pool(4, 16, 1, 128, "bf16")
    L = pa.lib()
    assert L.pa_decode_static_scratch(p.handle, None, 1, 1, None, 1, None, 1.0, 0, None,
                                      None) == 8
    assert L.pa_decode_static_scratch(None, None, 1, 1, None, 1, None, 1.0, 0, None,
                                      None) == 1


def _mirror(oracle, pool, op):
    kind, args = op[0], op[1:]
    if kind == "create":
        oracle.create(args[0]); pool.create(args[0])
        return None
    if kind == "share":
        oracle.share_prefix(*args); pool.fork(*args)
        return None
    if kind == "release":
        oracle.release(args[0]); pool.release(args[0])
        return None
    if kind == "append":
        s_o, c_o = oracle.append(args[0], args[1])
        s_g, c_g = pool.plan_append([args[0]], [args[1]])
        assert s_g == s_o and c_g == [tuple(c) for c in c_o]
        return None
    raise ValueError(kind)


def _same_state(oracle, pool):
    assert pool.refcounts() == oracle.refs
    for s in oracle.tables:
        t, length = pool.table(s)
        assert t == oracle.tables[s] and length == oracle.lengths[s]
    snap, st = oracle.snapshot(), pool.stats()
    for k in ("allocated_blocks", "free_blocks", "physical_capacity_tokens",
              "physical_payload_tokens", "logical_tokens", "internal_waste_tokens",
              "sharing_savings_tokens"):
        assert st[k] == snap[k], k
    assert pool.validate()


def test_manager_reproduces_printed_sharing_trace(golden_dir):
    import json
    g = json.load(open(os.path.join(golden_dir, "p2_paged_trace.json")))
    pool = pa.Pool(8, 4, 1, 1, "f32")
    names = {"A": 0, "B": 1}
    for op in g["_ops"]:
        if op[0] == "create":
            pool.create(names[op[1]])
        elif op[0] == "append":
            pool.plan_append([names[op[1]]], [op[2]])
        elif op[0] == "share":
            pool.fork(names[op[1]], names[op[2]], op[3])
        elif op[0] == "release":
            pool.release(names[op[1]])
        else:
            want = g["trace"][op[1]]
            st = pool.stats()
            for k, v in want.items():
                if k == "sequences":
                    for sname, sv in v.items():
                        assert pool.table(names[sname]) == (sv["blocks"], sv["length"])
                else:
                    assert st[k] == v, (op[1], k)


def test_manager_reproduces_p1_trace(golden_dir):
    import json
    g = json.load(open(os.path.join(golden_dir, "p1_ownership_trace.json")))
    pool = pa.Pool(8, 4, 1, 1, "f32", alloc_order=g["order"])
    ev = {e["event"]: e for e in g["events"]}

    def check(name):
        e = ev[name]
        assert pool.refcounts() == e["refs"]
        for s, t in e["tables"].items():
            assert pool.table({"A": 0, "B": 1}[s])[0] == t
    pool.create(0)
    for _ in range(7):
        pool.plan_append([0], [1])
    check("prompt-7")
    pool.fork(0, 1); check("fork")
    _, cow = pool.plan_append([1], [1]); check("B-copy-on-write-8")
    assert cow == [(2, 7)]
    pool.plan_append([0], [1]); check("A-private-8")
    pool.plan_append([1], [1]); check("B-boundary-9")
    pool.release(0); check("release-A")
    pool.release(1); check("release-B")


def test_error_codes_and_preflight():
    pool = pa.Pool(2, 4, 1, 1, "f32")
    with pytest.raises(pa.PAError) as e:
        pool.plan_append([5], [1])
    assert e.value.code == 2
    pool.create(1)
    with pytest.raises(pa.PAError) as e:
        pool.create(1)
    assert e.value.code == 3
    pool.plan_append([1], [6])
    before = (pool.stats(), pool.refcounts(), pool.table(1))
    with pytest.raises(pa.PAError) as e:
        pool.plan_append([1], [3])
    assert e.value.code == 4
    assert (pool.stats(), pool.refcounts(), pool.table(1)) == before
    with pytest.raises(pa.PAError) as e:
        pool.fork(1, 2, 7)
    assert e.value.code == 1
    with pytest.raises(pa.PAError) as e:
        pool.plan_append([1, 1], [0, 0])          # duplicate ids in one batch
    assert e.value.code == 1
    with pytest.raises(pa.PAError):
        pool.release(9)


def test_batch_preflight_is_all_or_nothing():
    # two sequences share a partial tail: the batch needs one copy (the second
    # member then owns the tail alone) -- exactly what sequential appends need
    o = KVPool(4, 4, store_heads=None)
    pool = pa.Pool(4, 4, 1, 1, "f32")
    for op in [("create", 0), ("append", 0, 3), ("share", 0, 1, 3), ("share", 0, 2, 3)]:
        _mirror(o, pool, op)
    slots, cow = pool.plan_append([1, 2], [1, 1])
    s1, c1 = o.append(1, 1)
    s2, c2 = o.append(2, 1)
    assert slots == s1 + s2 and cow == [tuple(c) for c in c1 + c2]
    _same_state(o, pool)
    # now too small: 3 more sequences x 2 blocks each cannot fit
    before = (pool.stats(), pool.refcounts())
    with pytest.raises(pa.PAError) as e:
        pool.plan_append([0, 1, 2], [5, 5, 5])
    assert e.value.code == 4
    assert (pool.stats(), pool.refcounts()) == before


def test_random_traces_match_oracle_bit_exactly():
    rng = np.random.default_rng(2024)
    for trial in range(25):
        nb, bs = int(rng.integers(8, 60)), int(rng.integers(1, 9))
        order = rng.permutation(nb)
        o = KVPool(nb, bs, allocation_order=order, store_heads=None)
        pool = pa.Pool(nb, bs, 1, 1, "f32", alloc_order=order)
        live, nxt = [], 0
        for _ in range(120):
            r = rng.random()
            try:
                if r < 0.15 or not live:
                    _mirror(o, pool, ("create", nxt)); live.append(nxt); nxt += 1
                elif r < 0.6:
                    s = live[rng.integers(len(live))]
                    n = int(rng.integers(0, 3 * bs + 2))
                    try:
                        o_res = o.append(s, n)
                    except PoolExhausted:
                        with pytest.raises(pa.PAError) as e:
                            pool.plan_append([s], [n])
                        assert e.value.code == 4
                        continue
                    s_g, c_g = pool.plan_append([s], [n])
                    assert s_g == o_res[0] and c_g == [tuple(c) for c in o_res[1]]
                elif r < 0.8:
                    src = live[rng.integers(len(live))]
                    p = int(rng.integers(0, o.lengths[src] + 1))
                    _mirror(o, pool, ("share", src, nxt, p)); live.append(nxt); nxt += 1
                elif r < 0.9:
                    s = live.pop(rng.integers(len(live)))
                    _mirror(o, pool, ("release", s))
                else:
                    # a rollback of one or two sequences' newest tokens
                    ss = list(rng.choice(live, size=min(len(live), 2), replace=False))
                    keep = [int(rng.integers(0, o.lengths[s] + 1)) for s in ss]
                    for s, k in zip(ss, keep):
                        o.truncate(int(s), k)
                    pool.truncate(ss, keep)
            except PoolError:
                raise
            _same_state(o, pool)


def test_truncate_checks_before_changing_anything():
    pool = pa.Pool(8, 4, 1, 1, "f32")
    pool.create(0); pool.create(1)
    pool.plan_append([0, 1], [9, 5])
    before = (pool.stats(), pool.refcounts(), pool.table(0), pool.table(1))
    for seqs, lens, code in (([0, 7], [1, 1], 2),      # unknown sequence
                             ([0, 1], [1, 6], 1),      # beyond the length
                             ([0, 1], [-1, 0], 1),     # negative
                             ([1, 1], [2, 1], 1)):     # named twice
        with pytest.raises(pa.PAError) as e:
            pool.truncate(seqs, lens)
        assert e.value.code == code
        assert (pool.stats(), pool.refcounts(), pool.table(0), pool.table(1)) == before
    pool.truncate([0, 1], [4, 0])
    assert pool.table(0) == ([0, 1][:1], 4) and pool.table(1) == ([], 0)
    assert pool.stats()["free_blocks"] == 7 and pool.validate()


@pytest.mark.parametrize("name", ["tiny", "ragged256", "prefill"])
def test_workload_scripts_match_oracle(name):
    w = workloads.ALL[name]()
    o = KVPool(w.num_blocks, w.block_size, allocation_order=w.order, store_heads=None)
    pool = pa.Pool(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.dtype,
                   alloc_order=w.order)
    for op in w.setup + w.step:
        _mirror(o, pool, (op.kind, *op.args))
    _same_state(o, pool)
    tables, lens = pool.block_tables(w.decode_seqs, max(len(o.tables[s]) for s in w.decode_seqs))
    assert np.array_equal(tables, o.block_table(w.decode_seqs, tables.shape[1]))
    assert lens.tolist() == [o.lengths[s] for s in w.decode_seqs]


def test_binding_checks_sizes_before_any_device_pointer():
    # the C ABI cannot see device array sizes: the binding rejects a short
    # table / kv_lens / row buffer, a wrong head_dim or output shape first
    p = pa.Pool(8, 16, 2, 128, "bf16")
    bf = torch.bfloat16
    q = torch.zeros(3, 8, 128, dtype=bf)
    t = torch.zeros(3, 4, dtype=torch.int32)
    lens = torch.zeros(3, dtype=torch.int32)
    cases = [
        (lambda: p.decode(torch.zeros(3, 8, 64, dtype=bf), t, lens), "head_dim"),
        (lambda: p.decode(torch.zeros(3, 7, 128, dtype=bf), t, lens), "multiple"),
        (lambda: p.decode(q, t[:2], lens), "block_tables"),
        (lambda: p.decode(q, t, lens[:2]), "kv_lens"),
        (lambda: p.decode(q, t, lens, out=torch.zeros(3, 8, 64)), "out must have shape"),
        (lambda: p.decode(q[0], t, lens), "dimensions"),
        (lambda: p.prefill_chunk(torch.zeros(3, 5, 8, 128, dtype=bf), t[:1], lens), "block_tables"),
        (lambda: p.decode_append(q, torch.zeros(3, 2, 128, dtype=bf), torch.zeros(2, 2, 128, dtype=bf),
                                 torch.zeros(3, dtype=torch.int64), t, lens), "value must have shape"),
        (lambda: p.decode_append(q, torch.zeros(3, 2, 128, dtype=bf), torch.zeros(3, 2, 128, dtype=bf),
                                 torch.zeros(2, dtype=torch.int64), t, lens), "slot_mapping"),
        (lambda: p.decode_window_append(q, torch.zeros(3, 1, 128, dtype=bf),
                                        torch.zeros(3, 1, 128, dtype=bf),
                                        torch.zeros(3, dtype=torch.int64), t, lens, 4), "key must"),
        (lambda: p.reshape_and_cache(torch.zeros(4, 2, 128, dtype=bf), torch.zeros(4, 2, 128, dtype=bf),
                                     torch.zeros(5, dtype=torch.int64)), "key must"),
        (lambda: p.cow_copy(torch.zeros(2, dtype=torch.int32), torch.zeros(3, dtype=torch.int32)),
         "pair up"),
    ]
    for call, msg in cases:
        with pytest.raises(ValueError, match=msg):
            call()
    # sizes that fit get as far as the device-pointer check
    with pytest.raises(ValueError, match="CUDA tensor"):
        p.decode(q, t, lens)


def test_manager_preflight_counts_the_copy_of_a_shared_partial_tail():
    # the same case as the oracle pin: one free block covers the new block
    # but not the copy of the shared partial tail, so the plan must fail
    # whole and change nothing
    pool = pa.Pool(3, 4, 1, 1, "f32")
    pool.create(0)
    pool.plan_append([0], [6])
    pool.fork(0, 1, 6)
    before = (pool.refcounts(), pool.table(0), pool.table(1), pool.stats())
    with pytest.raises(pa.PAError) as e:
        pool.plan_append([1], [3])
    assert e.value.code == 4                             # PA_ERR_POOL_EXHAUSTED
    assert (pool.refcounts(), pool.table(0), pool.table(1), pool.stats()) == before
    slots, cow = pool.plan_append([1], [2])              # the copy alone fits
    assert len(cow) == 1 and pool.validate()


def test_manager_payload_takes_the_largest_fill_among_sharers():
    pool = pa.Pool(4, 4, 1, 1, "f32")
    pool.create(0)
    pool.plan_append([0], [6])
    pool.fork(0, 1, 5)                                   # child sees the tail with 1 slot
    st = pool.stats()
    assert st["physical_payload_tokens"] == 6 and st["logical_tokens"] == 11
    assert st["internal_waste_tokens"] == 2 and st["sharing_savings_tokens"] == 5


def test_batch_calls_on_host_pools_and_bad_arguments():
    import ctypes as C
    L = pa.lib()
    p = pa.Pool(8, 4, 1, 8, "f32")
    p.create(0)
    seqs = np.array([0], np.int32)
    h = C.c_void_p()
    assert L.pa_batch_create(p.handle, seqs.ctypes.data_as(pa._PI32), 1, 1, 4, 0,
                             C.byref(h)) == 8                       # host-only pool
    assert h.value is None
    assert L.pa_batch_create(p.handle, seqs.ctypes.data_as(pa._PI32), 1, 1, 4, 0, None) == 1
    assert L.pa_batch_create(None, seqs.ctypes.data_as(pa._PI32), 1, 1, 4, 0, C.byref(h)) == 1
    for fn in (L.pa_batch_rollback, L.pa_batch_sync):
        assert fn(None) == 1
    assert L.pa_batch_free(None) == 0
    assert L.pa_batch_step(None, None, None, None, 1.0, None, None) == 1
    assert L.pa_batch_set_window(None, 16, 0) == 1
