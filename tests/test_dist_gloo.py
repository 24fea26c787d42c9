"""Multi-process plumbing of bench.py on CPU (gloo, world size 2).

The hot path shards by sequence with no exchange, so N GPUs run N replicas;
what the ranks share is only the barrier around the timed region and the
max-over-ranks reduction of the step time.  These tests run that logic as two
gloo ranks on the CPU, plus the per-rank workload seeding.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    d = bench.Dist(world)
    d.init("gloo")
    try:
        d.barrier()
        local_ms = 1.0 + rank * 2.5              # rank 1 is the slow one
        worst = d.max(local_ms)
        # every rank decodes its own replica batch: seeds differ per rank
        import workloads
        seed = workloads.seed_for(2) + 1000 * rank
        w = workloads.decode32(seed=seed)
        first_key = w.kv_for(w.setup[32])[0][0, 0, :4].float().tolist()
        q.put((rank, worst, d.world, seed, first_key))
    finally:
        d.close()


def test_two_rank_max_and_replica_seeds():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [3.5, 3.5]            # max over ranks on both
    assert all(r[2] == 2 for r in res)
    assert res[0][3] != res[1][3]                       # independent replicas
    assert res[0][4] != res[1][4]


def test_single_process_dist_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    d = bench.Dist(1)
    d.init("gloo")
    assert d.world == 1 and d.max(4.2) == 4.2
    d.barrier()
    d.close()


def test_reference_arm_runs_on_rank_zero_only():
    # under torchrun every rank starts bench.py --impl reference; ranks other
    # than 0 must exit 0 at once, with no output and no collective
    import subprocess
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1",
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--config", "tiny", "--steps", "3", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
