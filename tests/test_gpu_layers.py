"""Multi-layer pools on the GPU (needs a B200): one host manager and one
block table per sequence serve every layer ("docs.rs ferrum-kv 0.4.0
src/attention.rs", paged_attention's layer argument).  Each layer gets its
own K/V data; the oracle keeps one pool per layer under the same script, so
the tables agree and each layer's decode is checked against its own oracle.
A copy-on-write must copy the block in every layer."""
import numpy as np
import pytest
import torch

import paged_kv_cache_483_b200 as pa
import workloads
from harness import q64
from oracle import KVPool, attention_two_pass, stored_rows, stored_rows_fp8

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _layer_rows(k, layer):
    # distinct, bf16-exact data per layer
    return (k.float() * (1.0 + 0.25 * layer) + 0.125 * layer).to(torch.bfloat16)


def _run(w, L, q8):
    NB, bs, Hkv, d = w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim
    if q8:
        kc = torch.zeros((L, NB, Hkv, pa.PA_INT8_RECORD_BYTES), dtype=torch.uint8, device="cuda")
        pool = pa.Pool.layered(NB, bs, Hkv, d, "fp8" if q8 == "fp8" else "int8", L, kc, None,
                               alloc_order=w.order)
    else:
        kc = torch.zeros((L, NB, bs, Hkv, d), dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        pool = pa.Pool.layered(NB, bs, Hkv, d, "bf16", L, kc, vc, alloc_order=w.order)
    refs = [KVPool(NB, bs, Hkv, d, w.order) for _ in range(L)]
    n_cow = 0
    for op in w.setup + w.step:
        if op.kind == "create":
            pool.create(op.args[0])
            for r in refs:
                r.create(op.args[0])
        elif op.kind == "share":
            pool.fork(*op.args)
            for r in refs:
                r.share_prefix(*op.args)
        elif op.kind == "release":
            pool.release(op.args[0])
            for r in refs:
                r.release(op.args[0])
        else:
            seq, n = op.args
            k, v = w.kv_for(op)
            slots, cow = pool.plan_append([seq], [n])          # one plan for all layers
            if cow:
                n_cow += len(cow)
                src = torch.tensor([c[0] for c in cow], dtype=torch.int32, device="cuda")
                dst = torch.tensor([c[1] for c in cow], dtype=torch.int32, device="cuda")
                pool.layer(L - 1).cow_copy(src, dst)           # copies in every layer
            d_slots = torch.tensor(slots, dtype=torch.int64, device="cuda")
            for layer in range(L):
                kl, vl = _layer_rows(k, layer), _layer_rows(v, layer)
                pool.layer(layer).reshape_and_cache(kl.cuda(), vl.cuda(), d_slots)
                k64, v64 = kl.double().numpy(), vl.double().numpy()
                if q8:
                    rows = stored_rows_fp8 if q8 == "fp8" else stored_rows
                    k64, v64 = rows(k64)[2], rows(v64)[2]
                got, _ = refs[layer].append(seq, n, k64, v64)
                assert got == slots
    assert pool.refcounts() == refs[0].refs
    width = max(len(pool.table(s)[0]) for s in w.decode_seqs)
    tables, lens = pool.block_tables(w.decode_seqs, width)
    t, ln = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    q = w.queries()[:, 0].contiguous().cuda()
    qq = q64(w)
    G = w.num_heads // Hkv
    for layer in range(L):
        out = pool.layer(layer).decode(q, t, ln).cpu().numpy()
        worst = 0.0
        for i, s in enumerate(w.decode_seqs):
            kk, vv = refs[layer].gather(s)
            o = attention_two_pass(qq[i], kk, vv)
            worst = max(worst, float(np.abs(out[i] - o[0]).max()))
        assert worst <= TOL, (layer, worst)
    assert pool.get_error() == 0
    return pool, n_cow


@pytest.mark.parametrize("q8", [False, True, "fp8"])
def test_layers_share_tables_and_copy_on_write(q8):
    w = workloads.ragged256(groups=2, per_group=3, prefix=40, spare_blocks=16)
    pool, n_cow = _run(w, 3, q8)
    assert n_cow > 0                       # the step copied shared partial tails
    with pytest.raises(pa.PAError):
        pool.layer(3)
    assert pa.lib().pa_free(pool.layer(1).handle) == 1     # a layer handle is not freed alone
    pool.close()
