#!/usr/bin/env python
"""Benchmark of the paged-attention hot path on B200.

Default workload (the headline metric): decode batch 32 at 8K context, GQA
32/8, head_dim 128, block 16, bf16 K/V/Q, a 16384-block pool in a seeded
permuted order.  One step = append of every sequence's new token (K/V written
at the slots the host manager planned for position 8191) and paged decode
attention at kv_len 8192, fused in one kernel (pa_decode_append).  The device
step replays one plan (a repeated step must rewrite the same slots); the host
plan is timed on its own (``host_plan_us``, median of warm calls) and inside
every ``e2e`` step, which plans, copies, runs and rolls the step back.

Metric: effective KV bytes read by decode per second (sum_b kv_len_b * Hkv *
head_dim * 2 (K and V) * 2 bytes), whole job over all ranks; ``seqs_per_s``
is the same time expressed as sequences decoded per second.

Other workloads (``--config``): ragged256 (copy-on-write + append + decode),
splitk128k (split-K decode + log-sum-exp combine), prefill (512-token chunk
append + causal chunked prefill; metric TFLOP/s of causal pairs).  The
default run also measures each of them, and decode32 over int8 and FP8
pools, under ``configs`` (each with its own roofline, e2e and clocks).

Timing: each workload's step (its launches, same arguments every step) is
captured once in a CUDA graph and replayed K times back to back between two
CUDA events, as a serving loop replays its decode step; the kernel time of a
step with launches before attention (copy-on-write, an unfused append) comes
from a second pass of K replays of a graph of the attention launches alone.
``e2e`` calls the public API eagerly, with host copies, every step.

Multi-GPU: one process per GPU (torchrun); every rank decodes its own replica
batch (different seeds), no collective on the data path ("scaling": "weak");
the time is the max over ranks.  ``--impl reference`` times the float64 CPU
oracle on this host's cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

MIB = 1 << 20
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
# datasheet figures, for the second fraction the measurement plan asks for
NOMINAL_HBM_GBS, NOMINAL_BF16_TFLOPS = 8000.0, 2250.0


# ------------------------------------------------------------------ helpers --
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained", p["bf16_tflops"]), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "paged_kv_cache_483_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_file, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel (else None)."""
    path = os.path.join(ROOT, "profiles", f"traffic_{workload}.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    if d.get("source_hash") != source_hash(kernel_file):
        return None
    return d.get("dram_bytes_per_launch")


SAMPLER = None                # the bench run's clock sampler (main)

CLOCK_REASONS = {
    0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


def _clock_sampler_main(uuid, index, period, conn):
    """Child process: after 'begin', samples (time, SM MHz, reason bits)
    every `period` seconds until 'end', then sends the samples back."""
    try:
        import pynvml
        pynvml.nvmlInit()
        try:
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
        except Exception:
            h = pynvml.nvmlDeviceGetHandleByIndex(index)
        conn.send(("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)))
    except Exception as e:            # no NVML: report it, sample nothing
        conn.send(("error", repr(e)))
        return
    while True:
        msg = conn.recv()
        if msg == "quit":
            return
        buf = []
        first = True
        while not conn.poll():
            try:
                buf.append((time.time(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                            pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except Exception:
                pass
            if first:
                conn.send("sampling")      # the window opens after the first sample
                first = False
            time.sleep(period)
        conn.recv()                    # 'end'
        conn.send(buf)


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML by a separate
    process (no contention with the launch loop for the interpreter lock).
    ``with sampler.window() as w:`` brackets a timed region; ``w.summary()``
    then covers only the samples taken between its two time stamps."""

    def __init__(self, cuda_index, period=0.0002):
        import multiprocessing as mp
        import torch
        self.max_mhz, self.error = None, None
        uuid = str(torch.cuda.get_device_properties(cuda_index).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        ctx = mp.get_context("spawn")
        self.conn, child = ctx.Pipe()
        self.proc = ctx.Process(target=_clock_sampler_main, args=(uuid, cuda_index, period, child),
                                daemon=True)
        self.proc.start()
        try:
            kind, val = self.conn.recv() if self.conn.poll(120) else ("error", "no answer")
        except (EOFError, OSError) as e:
            kind, val = "error", repr(e)
        if kind == "max":
            self.max_mhz = val
        else:
            self.error = val

    def window(self):
        return _ClockWindow(self)

    def close(self):
        if self.proc.is_alive():
            try:
                self.conn.send("quit")
            except Exception:
                pass
            self.proc.join(timeout=5)


class _ClockWindow:
    def __init__(self, sampler):
        self.s, self.samples, self.t0, self.t1 = sampler, [], None, None

    def __enter__(self):
        if self.s.error is None:
            self.s.conn.send("begin")
            self.s.conn.recv()         # 'sampling': the sampler is running
        self.t0 = time.time()
        return self

    def __exit__(self, *a):
        self.t1 = time.time()
        if self.s.error is None:
            time.sleep(0.001)
            self.s.conn.send("end")
            self.samples = self.s.conn.recv()

    def summary(self):
        inside = [(t, mhz, r) for t, mhz, r in self.samples if self.t0 <= t <= self.t1]
        reasons = sorted({name for _, _, r in inside for bit, name in CLOCK_REASONS.items()
                          if r & bit})
        out = {"sm_mhz": float(statistics.median(m for _, m, _ in inside)) if inside else None,
               "sm_max_mhz": self.s.max_mhz, "reasons": reasons, "samples": len(inside)}
        if self.s.error:
            out["error"] = self.s.error
        return out


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------- distributed --
class Dist:
    def __init__(self, want):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.want = want
        self.pg = None

    def init(self, backend):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x, device=None):
        if not self.pg:
            return x
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# --------------------------------------------------------- our CUDA path ----
class Setup:
    """A workload brought up on the GPU through the C ABI (untimed).

    ``memo`` (optional dict) keeps each append op's host K/V so that another
    pool type over the same workload reuses them instead of drawing again."""

    def __init__(self, w, device, q8=False, memo=None):
        import torch
        import paged_kv_cache_483_b200 as pa
        self.w, self.device, self.q8 = w, device, q8
        if q8:    # "int8" / "fp8" pool: packed (block, head) records, bf16 rows quantised on append
            self.k_cache = torch.empty((w.num_blocks, w.num_kv_heads, pa.PA_INT8_RECORD_BYTES),
                                       dtype=torch.uint8, device=device)
            self.v_cache = None
            self.pool = pa.Pool(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, q8,
                                self.k_cache, None, alloc_order=w.order)
        else:
            dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
            shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
            self.k_cache = torch.empty(shape, dtype=dt, device=device)
            self.v_cache = torch.empty(shape, dtype=dt, device=device)
            self.pool = pa.Pool(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.dtype,
                                self.k_cache, self.v_cache, alloc_order=w.order)

        def kv(op):
            if memo is None:
                return w.kv_for(op)
            if op.index not in memo:
                memo[op.index] = w.kv_for(op)
            return memo[op.index]

        for op in w.setup:
            if op.kind == "create":
                self.pool.create(op.args[0])
            elif op.kind == "share":
                self.pool.fork(*op.args)
            elif op.kind == "release":
                self.pool.release(op.args[0])
            else:
                k, v = kv(op)
                self.pool.append_kv([op.args[0]], [op.args[1]], k.to(device), v.to(device))
        torch.cuda.synchronize()
        # the step's appends: planned once by the host manager (the plan's own
        # cost is measured separately, on warm calls)
        self.step_k = self.step_v = None
        self.slots = None
        self.cow_src = self.cow_dst = None
        if w.step:
            seqs = [op.args[0] for op in w.step]
            n_new = [op.args[1] for op in w.step]
            slots, cow = self.pool.plan_append(seqs, n_new)
            ks, vs = zip(*[kv(op) for op in w.step])
            self.step_k = torch.cat(ks).to(device)
            self.step_v = torch.cat(vs).to(device)
            self.slots = torch.tensor(slots, dtype=torch.int64, device=device)
            if cow:
                self.cow_src = torch.tensor([c[0] for c in cow], dtype=torch.int32, device=device)
                self.cow_dst = torch.tensor([c[1] for c in cow], dtype=torch.int32, device=device)
        t, lens = self.pool.block_tables(w.decode_seqs, max(len(self.pool.table(s)[0])
                                                            for s in w.decode_seqs))
        self.tables_h, self.lens_h = t, lens
        self.tables = torch.from_numpy(t).to(device)
        self.lens = torch.from_numpy(lens).to(device)
        q = w.queries()
        self.q = (q[:, 0] if w.q_tokens == 1 else q).contiguous().to(device)
        self.out = torch.empty(self.q.shape, dtype=torch.float32, device=device)
        self.n_cow = 0 if self.cow_src is None else int(self.cow_src.numel())


def decode_bytes(w, lens, q8=False, window=0, sinks=0):
    """K/V bytes a decode step must read: every token, or with a window the
    min(kv_len, sinks + window) visible ones."""
    lens = lens.astype(np.int64)
    if window > 0:
        lens = np.minimum(lens, window + sinks)
    if q8:    # int8 / fp8 records: K and V codes plus two float32 scales per (token, head)
        return int(np.sum(lens)) * w.num_kv_heads * (2 * w.head_dim + 8)
    eb = 2 if w.dtype == "bf16" else 4
    return int(np.sum(lens)) * w.num_kv_heads * w.head_dim * 2 * eb


def prefill_flops(w, lens):
    # 4 * d * H * (q * cached + q (q + 1) / 2) per sequence: causal pairs only
    q = w.q_tokens
    return int(sum(4 * w.head_dim * w.num_heads * (q * (int(L) - q) + q * (q + 1) // 2)
                   for L in lens))


def default_seed(config):
    return (workloads.SEED_TINY if config == "tiny" else
            workloads.seed_for({"decode32": 2, "ragged256": 3, "splitk128k": 4,
                                "prefill": 5}[config]))


def run_workload(args, dist, config, kv="bf16", win=0, sinks=0, *, steps, min_ms=0.0,
                 cpu=False, memo=None):
    """Bring one workload up, time its step on the device and end to end.

    steps: timed steps; with min_ms > 0 the count grows until the timed region
    lasts about min_ms."""
    import torch
    device = torch.device("cuda", dist.local)
    builder = workloads.ALL[config]
    base_seed = args.seed if args.seed is not None else default_seed(config)
    w = builder(seed=base_seed + 1000 * dist.rank)
    q8 = kv if kv in ("int8", "fp8") else False
    if (q8 or win) and w.q_tokens > 1:
        raise SystemExit("--kv int8/fp8 and --window apply to the decode workloads")
    S = Setup(w, device, q8=q8, memo=memo)
    pool = S.pool
    is_prefill = w.q_tokens > 1
    part = w.partition_tokens
    stream = torch.cuda.current_stream(device)

    import paged_kv_cache_483_b200 as pa
    ws_bytes = 0 if is_prefill else (
        int(pa.lib().pa_decode_window_workspace_bytes(pool.handle, S.q.shape[0], S.q.shape[1],
                                                      S.tables.shape[1], win, sinks, part))
        if win else pool.decode_workspace_bytes(S.q.shape[0], S.q.shape[1],
                                                S.tables.shape[1], part))
    split = ws_bytes > 0                    # a second launch: order prepass or combine
    order_only = ws_bytes == 4 * S.q.shape[0]
    # decode steps fuse the new token's append into the decode kernel (bf16;
    # on an int8 pool the append is its own quantising launch)
    fused = (not is_prefill) and S.slots is not None and not q8
    per_step = ((1 if S.n_cow else 0) + (1 if (S.slots is not None and not fused) else 0)
                + (2 if split else 1))

    has_pre = bool(S.n_cow) or (S.slots is not None and not fused)

    def pre(st):
        """The step's launches before attention: copy-on-write, unfused append."""
        if S.n_cow:
            pool.cow_copy(S.cow_src, S.cow_dst, st)
        if S.slots is not None and not fused:
            pool.reshape_and_cache(S.step_k, S.step_v, S.slots, st)

    def attn(st):
        """The attention launch(es): prefill, or decode (with the new tokens'
        append fused in, and its order prepass / combine when it has them)."""
        if is_prefill:
            pool.prefill_chunk(S.q, S.tables, S.lens, out=S.out, stream=st)
        elif fused and win:
            pool.decode_window_append(S.q, S.step_k, S.step_v, S.slots, S.tables, S.lens, win,
                                      sinks, out=S.out, partition_tokens=part, stream=st)
        elif fused:
            pool.decode_append(S.q, S.step_k, S.step_v, S.slots, S.tables, S.lens, out=S.out,
                               partition_tokens=part, stream=st)
        elif win:
            pool.decode_window(S.q, S.tables, S.lens, win, sinks, out=S.out,
                               partition_tokens=part, stream=st)
        else:
            pool.decode(S.q, S.tables, S.lens, out=S.out, partition_tokens=part, stream=st)

    def step(st):
        pre(st)
        attn(st)

    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    for _ in range(max(1, args.warmup)):
        step(stream)
    w1.record(stream)
    torch.cuda.synchronize()
    assert pool.get_error() == 0, "device error during warm-up"
    K = steps
    if min_ms > 0:
        est = w0.elapsed_time(w1) / max(1, args.warmup)
        K = max(K, int(math.ceil(min_ms / max(est, 1e-3))))
        K = dist.max(K, device) if dist.world > 1 else K
        K = int(K)

    # ------------------------------------------------------ timed region --
    # A serving loop replays its decode step as a CUDA graph: the step's
    # launches are captured once (same arguments every step) and the graph is
    # replayed K times back to back, with no event between steps.  With no
    # launch before attention, the attention kernel's average launch duration
    # is the region's time / K; otherwise a second pass replays a graph of the
    # attention launch(es) alone, K times.
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        step(torch.cuda.current_stream(device))
    g_attn = None
    if has_pre:
        g_attn = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_attn):
            attn(torch.cuda.current_stream(device))
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    with SAMPLER.window() as clk:
        t_start.record(stream)
        for _ in range(K):
            g_step.replay()
        t_end.record(stream)
        torch.cuda.synchronize()
        gpu_launches = per_step * K
        ms_step = t_start.elapsed_time(t_end) / K
        if g_attn is None:
            kern_ms = ms_step
            kern_timing = "timed region / steps (graph replays, one step each, back to back)"
        else:
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(K):
                g_attn.replay()
            a1.record(stream)
            torch.cuda.synchronize()
            kern_ms = a0.elapsed_time(a1) / K
            kern_timing = (f"a second pass: {K} replays of a graph of the attention launch(es) "
                           "alone, back to back")
    del g_step, g_attn
    dist.barrier()
    ms_step_max = dist.max(ms_step, device)
    assert pool.get_error() == 0, "device error in the timed region"

    # the chunk's own append (K1 at the planned slots), timed on its own with
    # L2 flushed between launches (its 32 MiB of traffic would fit in L2)
    append = None
    if is_prefill and S.slots is not None:
        append = time_append(S, stream, torch.cuda.current_device())

    # --------------------------------------------------------------- e2e --
    e2e = run_e2e(args, S, dist, device, is_prefill, part, win, sinks)

    hbm, bf16, bf16_sus, peak_kind = peaks()
    lens = S.lens_h
    if is_prefill:
        flops = prefill_flops(w, lens)
        value = dist.world * flops / (ms_step_max * 1e-3) / 1e12
        metric = metric_name(w, q8, win, sinks)
        unit = "TFLOP/s"
        achieved = flops / (kern_ms * 1e-3) / 1e12
        # The burst peak is the GEMM timed alone; the sustained one the GEMM in
        # a seconds-long loop under the power cap.  A timed region that ran
        # under sw_power_cap is in the sustained regime.
        capped = "sw_power_cap" in (clk.summary().get("reasons") or [])
        pk = bf16_sus if capped else bf16
        roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk,
                "unit": "TFLOP/s", "frac": round(achieved / pk, 4),
                "traffic": profiled_traffic("prefill_tc.cu", w.name),
                "frac_of_nominal": round(achieved / NOMINAL_BF16_TFLOPS, 4),
                "frac_of_burst": round(achieved / bf16, 4),
                "frac_of_sustained": round(achieved / bf16_sus, 4),
                "kernel": "prefill_tc_kernel", "kernel_ms": round(kern_ms, 5),
                "kernel_timing": kern_timing,
                "algorithmic_flops_per_launch": flops,
                "peak_source": (f"{peak_kind} bf16_tflops_sustained (the timed region ran "
                                "under sw_power_cap)" if capped
                                else f"{peak_kind} bf16_tflops (burst)")}
        extra = {"tflops": round(value, 2), "append": append}
    else:
        kvb = decode_bytes(w, lens, q8, win, sinks)
        value = dist.world * kvb / (ms_step_max * 1e-3) / 1e9
        metric = metric_name(w, q8, win, sinks)
        unit = "GB/s"
        achieved = kvb / (kern_ms * 1e-3) / 1e9
        # int8 / FP8 pools: the tcgen05 kernel up to 4 heads per group, the
        # warp-level one above
        q8tc = bool(q8) and w.num_heads // w.num_kv_heads <= 4
        kname = (("decode_q8tc_kernel" if q8tc else "decode_q8_kernel") if q8 else
                 "decode_mma_kernel"
                 if pool.decode_path(w.num_heads) else "attention_generic_kernel")
        kfile = ("decode_q8tc.cu" if q8tc else "decode_q8.cu") if q8 else "decode_mma.cu"
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4),
                "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                "traffic": profiled_traffic(kfile,
                                            w.name + (f"_{q8}" if q8 else "")
                                            + (f"_window{win}_sinks{sinks}" if win else "")),
                "kernel": (f"decode_order_kernel + {kname}" if order_only else
                           f"{kname} + decode_combine_kernel" if split else kname),
                "kernel_ms": round(kern_ms, 5), "kernel_timing": kern_timing,
                "algorithmic_bytes_per_launch": kvb, "peak_source": f"{peak_kind} hbm_gbs"}
        extra = {"seqs_per_s": round(dist.world * len(w.decode_seqs) / (ms_step_max * 1e-3), 1),
                 "frac_of_peak": round(value / hbm, 4)}
        if q8:
            extra["kv_bytes_vs_bf16"] = round(kvb / decode_bytes(w, lens, False, win, sinks), 4)
        if win:
            extra["window"] = {"window": win, "sinks": sinks,
                               "visible_fraction": round(kvb / decode_bytes(w, lens, q8), 4)}
    res = {
        "metric": metric, "value": round(value, 2), "unit": unit, "n_gpus": dist.world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_step_max, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("int8 KV codes (int8 MMA on the codes, fp32 softmax), bf16 Q" if q8 == "int8"
                  else "fp8 e4m3 KV codes (e4m3 MMA on the codes, fp32 softmax), bf16 Q" if q8
                  else "bf16"),
        "data": "synthetic (seeded N(0,1), bf16-rounded)",
        "config": config_of(w, kv, win, sinks, dist),
        **extra,
        "host_plan_us": host_plan_us(S) if S.slots is not None else None,
        "gpu_launches": gpu_launches,
        "roofline": roof,
        "e2e": e2e,
        "clocks": clk.summary(),
    }
    if cpu and dist.rank == 0 and dist.world == 1:
        res["cpu_baseline"] = cpu_baseline(w, args, S.out.float().cpu().numpy(), q8, win, sinks)
    pool.close()
    del S
    torch.cuda.empty_cache()
    return res


def time_append(S, stream, cuda_index, n_app=300, rounds=10):
    """reshape_and_cache of the step's rows at their planned slots with L2
    flushed (a 256 MiB read) before every launch.  Two CUDA graphs, the flush
    alone and the flush followed by the append, are replayed back to back in
    alternating rounds; the append's time is the difference of their means (no
    event between the flush and the append: an event record between two
    launches adds microseconds, as much as this kernel takes)."""
    import torch
    pool = S.pool
    dev = S.device
    # the flush reads a buffer larger than L2, leaving it full of clean lines
    # (a write flush would leave dirty lines for the timed kernel to evict)
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    sink = torch.empty(1, dtype=torch.float32, device=dev)
    for _ in range(3):
        torch.sum(flush, dim=0, keepdim=True, out=sink)
        pool.reshape_and_cache(S.step_k, S.step_v, S.slots, stream)
    torch.cuda.synchronize()
    g_f, g_fa = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_f):
        torch.sum(flush, dim=0, keepdim=True, out=sink)
    with torch.cuda.graph(g_fa):
        torch.sum(flush, dim=0, keepdim=True, out=sink)
        pool.reshape_and_cache(S.step_k, S.step_v, S.slots, torch.cuda.current_stream(dev))
    torch.cuda.synchronize()
    per = max(1, n_app // rounds)
    t_f, t_fa = [], []
    with SAMPLER.window() as clk:
        for _ in range(rounds):
            for g, acc in ((g_f, t_f), (g_fa, t_fa)):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(per):
                    g.replay()
                b.record(stream)
                torch.cuda.synchronize()
                acc.append(a.elapsed_time(b) / per)
    assert pool.get_error() == 0
    del g_f, g_fa
    app_ms = statistics.mean(t_fa) - statistics.mean(t_f)
    moved = 2 * 2 * S.step_k.numel() * S.step_k.element_size()   # K and V, read + write
    hbm, _, _, peak_kind = peaks()
    gbs = moved / (app_ms * 1e-3) / 1e9
    return {"kernel": "reshape_and_cache_kernel<uint4>", "launches": per * rounds,
            "kernel_ms": round(app_ms, 5), "bytes_per_launch": moved,
            "kernel_timing": ("mean of (flush + append) graph replays minus mean of flush-alone "
                              f"replays, {rounds} alternating rounds of {per}"),
            "flush_ms": round(statistics.mean(t_f), 5),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4),
                         "traffic": profiled_traffic("kv_write.cu", "prefill_append"),
                         "peak_source": f"{peak_kind} hbm_gbs"},
            "l2": "flushed before every launch (a 256 MiB read)",
            "clocks": clk.summary()}


def host_plan_us(S, n=200):
    """Median wall time of one warm pa_plan_append of the step's appends (host
    manager, through ctypes), each followed by an untimed rollback
    (pa_seq_truncate) so that every call plans the same step."""
    pool = S.pool
    seqs = [op.args[0] for op in S.w.step]
    n_new = [op.args[1] for op in S.w.step]
    base = [pool.table(s)[1] for s in seqs]           # lengths after the step's plan
    start = [b - k for b, k in zip(base, n_new)]
    pool.truncate(seqs, start)
    t = []
    for _ in range(n):
        t0 = time.perf_counter()
        pool.plan_append(seqs, n_new)
        t.append(time.perf_counter() - t0)
        pool.truncate(seqs, start)
    pool.plan_append(seqs, n_new)                     # the state the step assumes
    return round(statistics.median(t) * 1e6, 2)


def config_of(w, kv, win, sinks, dist):
    G = w.num_heads // w.num_kv_heads
    return {"workload": w.name, "batch_per_gpu": len(w.decode_seqs),
            "global_batch": len(w.decode_seqs) * dist.world,
            "num_heads": w.num_heads, "num_kv_heads": w.num_kv_heads, "group": G,
            "head_dim": w.head_dim, "block_size": w.block_size, "num_blocks": w.num_blocks,
            "q_tokens": w.q_tokens, "partition_tokens": w.partition_tokens,
            "parallelism": f"replicas x{dist.world} (no collective)",
            "kv": kv, "window": win, "sinks": sinks,
            "l2": ("tiny: fits in L2 (correctness scale)" if w.name == "tiny" else
                   "KV per step ~0.5 GB > L2 (shared prefixes may hit in L2)"
                   if w.name == "ragged256" else
                   "visible KV per step just above the 126 MB L2, no flush: in this loop ncu "
                   "reads about 4 % of the walked bytes from L2, not DRAM"
                   if win and w.name == "decode32" and win + sinks <= 1100 else
                   "inputs larger than L2 (KV per step > 126 MB)")}


class _PinnedRing:
    """Pinned host buffers reused round-robin; a buffer is rewritten only after
    the copy that last read it has run."""

    def __init__(self, make, depth=8):
        import torch
        self.bufs = [make() for _ in range(depth)]
        self.evs = [torch.cuda.Event() for _ in range(depth)]
        self.used = [False] * depth
        self.i = 0

    def take(self):
        i = self.i
        self.i = (i + 1) % len(self.bufs)
        if self.used[i]:
            self.evs[i].synchronize()
        self.used[i] = True
        return self.bufs[i], self.evs[i]


def run_e2e(args, S, dist, device, is_prefill, part, win, sinks):
    """Same metric through the public API with host buffers (see run_e2e_steps
    and run_e2e_batch): decode steps that append one token per sequence go
    through the prepared batch, the rest through the separate calls."""
    w = S.w
    one_token = (not is_prefill) and bool(w.step) and all(op.args[1] == 1 for op in w.step) \
        and [op.args[0] for op in w.step] == list(w.decode_seqs)
    if one_token:
        return run_e2e_batch(args, S, dist, device, part, win, sinks)
    return run_e2e_steps(args, S, dist, device, is_prefill, part, win, sinks)


def run_e2e_batch(args, S, dist, device, part, win=0, sinks=0):
    """The serving decode loop through pa_batch_step: each step is one C call
    that plans the step's appends on the host manager (step a1), uploads the
    plan, the changed table entries, the queries and the new K/V from pinned
    host memory, runs copy-on-write copies and the fused append + decode, and
    downloads the output; pa_batch_rollback then gives every sequence's token
    back (host-only) so that every step is the same step.  The timed region
    holds K steps and the final wait for the last output.  The transfers of
    consecutive steps overlap their neighbours' kernels (two buffer sets; an
    upload of up to 1 MiB is one kernel that reads the pinned inputs in place,
    larger ones and those of quantised pools are copies; each download is
    queued behind the next step's uploads).  A copy-on-write of a shared partial tail happens in the first
    step only (the tail is private afterwards), as in serving."""
    import torch
    import paged_kv_cache_483_b200 as pa
    pool, w = S.pool, S.w
    stream = torch.cuda.current_stream(device)
    seqs = list(w.decode_seqs)
    n = len(seqs)
    h_q = S.q.cpu().pin_memory()
    h_k, h_v = S.step_k.cpu().pin_memory(), S.step_v.cpu().pin_memory()
    h_out = torch.empty(S.out.shape, dtype=torch.float32).pin_memory()
    lens_now = [pool.table(s)[1] for s in seqs]
    pool.truncate(seqs, [L - 1 for L in lens_now])        # undo the set-up's plan
    batch = pa.Batch(pool, seqs, S.q.shape[1], S.tables.shape[1], part)
    if win:
        batch.set_window(win, sinks)
    K = max(1, args.e2e_steps)   # its own count: a serving loop's steady state, not the timed K

    def step():
        batch.step(h_q, h_k, h_v, h_out, stream=stream)
        batch.rollback()

    for _ in range(3):
        step()
    batch.sync()
    torch.cuda.synchronize()
    dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    a.record(stream)
    for _ in range(K):
        step()
    host_ms = (time.perf_counter() - t0) * 1e3 / K        # queueing the steps
    batch.sync()
    b.record(stream)
    torch.cuda.synchronize()
    wall_ms = (time.perf_counter() - t0) * 1e3 / K
    ms = dist.max(max(a.elapsed_time(b) / K, wall_ms), device)
    batch.close()
    pool.plan_append(seqs, [1] * n)                       # back to the state the step assumes
    v = dist.world * decode_bytes(w, S.lens_h, S.q8, win, sinks) / (ms * 1e-3) / 1e9
    bi = (h_q.numel() * h_q.element_size() + 2 * h_k.numel() * h_k.element_size()
          + n * (8 + 4))                                  # + the plan: slots and lengths
    return {"value": round(v, 2), "unit": "GB/s", "h2d_bytes_per_step": int(bi),
            "d2h_bytes_per_step": int(h_out.numel() * 4), "ms_per_step": round(ms, 5),
            "steps": K, "host_plan_in_step": True,
            "api": "pa_batch_step + pa_batch_rollback"
                   + (" (after pa_batch_set_window)" if win else ""),
            "host_ms_per_step": round(host_ms, 5)}


def run_e2e_steps(args, S, dist, device, is_prefill, part, win, sinks):
    """Same metric through the separate calls with host buffers.  Every step
    plans its appends on the host manager (pa_plan_append), copies its inputs
    (queries, new K/V, slot mapping, copy-on-write pairs, kv_lens) from pinned
    host memory, runs the step's kernels and reads the output back; then the
    step's tokens are rolled back (pa_seq_truncate) so that every step is the
    same step.  Plans, copies and the rollback are inside the timed region.
    Two buffer sets and two copy streams let a step's uploads and the previous
    step's download run while the kernels of their neighbours do.  A
    copy-on-write of a shared partial tail happens in the first planned step
    only (the tail is private afterwards), as in serving."""
    import torch
    pool = S.pool
    stream = torch.cuda.current_stream(device)
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    w = S.w
    h_q = S.q.cpu().pin_memory()
    h_lens = S.lens.cpu().pin_memory()
    bi = h_q.numel() * h_q.element_size() + h_lens.numel() * 4
    seqs = [op.args[0] for op in w.step]
    n_new = [op.args[1] for op in w.step]
    plan = bool(w.step)
    if plan:
        h_k, h_v = S.step_k.cpu().pin_memory(), S.step_v.cpu().pin_memory()
        T = int(S.slots.numel())
        d_cow = torch.empty(2 * len(seqs), dtype=torch.int32, device=device)
        ring = _PinnedRing(lambda: (torch.empty(T, dtype=torch.int64).pin_memory(),
                                    torch.empty(2 * len(seqs), dtype=torch.int32).pin_memory()))
        bi += 2 * h_k.numel() * h_k.element_size() + T * 8
        lens_now = [pool.table(s)[1] for s in seqs]
        start = [L - k for L, k in zip(lens_now, n_new)]
        pool.truncate(seqs, start)                       # undo the set-up's plan
    sets = []
    for i in range(2):
        b = {"q": torch.empty_like(S.q), "lens": torch.empty_like(S.lens),
             "out": S.out if i == 0 else torch.empty_like(S.out),
             "h_out": torch.empty(S.out.shape, dtype=torch.float32).pin_memory(),
             "up": torch.cuda.Event(), "done": torch.cuda.Event(), "down": torch.cuda.Event(),
             "used": False}
        if plan:
            b.update(k=torch.empty_like(S.step_k), v=torch.empty_like(S.step_v),
                     slots=torch.empty_like(S.slots))
        sets.append(b)
    bo = S.out.numel() * 4
    K = max(1, args.e2e_steps)   # its own count: a serving loop's steady state, not the timed K
    fused = (not is_prefill) and plan and not S.q8
    cow_bytes = [0]
    count = [0]

    def step():
        b = sets[count[0] % 2]
        count[0] += 1
        if plan:
            slots, cow = pool.plan_append(seqs, n_new)            # step a1, on the host
            (hs, hc), ev = ring.take()
            hs.numpy()[:] = slots
        with torch.cuda.stream(up):
            if b["used"]:
                up.wait_event(b["done"])          # this set's last kernels have read it
            b["q"].copy_(h_q, non_blocking=True)
            b["lens"].copy_(h_lens, non_blocking=True)
            if plan:
                b["slots"].copy_(hs, non_blocking=True)
                b["k"].copy_(h_k, non_blocking=True)
                b["v"].copy_(h_v, non_blocking=True)
            b["up"].record(up)
        stream.wait_event(b["up"])
        if b["used"]:
            stream.wait_event(b["down"])          # and its last output has been read back
        if plan:
            if cow:
                n = len(cow)
                hc.numpy()[:n] = [c[0] for c in cow]
                hc.numpy()[n:2 * n] = [c[1] for c in cow]
                d_cow[:2 * n].copy_(hc[:2 * n], non_blocking=True)
                pool.cow_copy(d_cow[:n], d_cow[n:2 * n], stream)
                cow_bytes[0] += 8 * n
            ev.record(stream)                     # after both copies of the pinned plan
            if not fused:
                pool.reshape_and_cache(b["k"], b["v"], b["slots"], stream)
        if is_prefill:
            pool.prefill_chunk(b["q"], S.tables, b["lens"], out=b["out"], stream=stream)
        elif fused and win:
            pool.decode_window_append(b["q"], b["k"], b["v"], b["slots"], S.tables, b["lens"],
                                      win, sinks, out=b["out"], partition_tokens=part,
                                      stream=stream)
        elif fused:
            pool.decode_append(b["q"], b["k"], b["v"], b["slots"], S.tables, b["lens"],
                               out=b["out"], partition_tokens=part, stream=stream)
        elif win:
            pool.decode_window(b["q"], S.tables, b["lens"], win, sinks, out=b["out"],
                               partition_tokens=part, stream=stream)
        else:
            pool.decode(b["q"], S.tables, b["lens"], out=b["out"], partition_tokens=part,
                        stream=stream)
        b["done"].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(b["done"])
            b["h_out"].copy_(b["out"], non_blocking=True)
            b["down"].record(down)
        b["used"] = True
        if plan:
            pool.truncate(seqs, start)                            # roll the step back

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    dist.barrier()
    cow_bytes[0] = 0
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    up.wait_stream(stream)                        # the first uploads start after a
    for _ in range(K):
        step()
    stream.wait_stream(down)                      # b after the last download
    b.record(stream)
    torch.cuda.synchronize()
    ms = dist.max(a.elapsed_time(b) / K, device)
    if plan:
        pool.plan_append(seqs, n_new)                 # back to the state the step assumes
    if is_prefill:
        v = dist.world * prefill_flops(w, S.lens_h) / (ms * 1e-3) / 1e12
        unit = "TFLOP/s"
    else:
        v = dist.world * decode_bytes(w, S.lens_h, S.q8, win, sinks) / (ms * 1e-3) / 1e9
        unit = "GB/s"
    return {"value": round(v, 2), "unit": unit, "h2d_bytes_per_step": int(bi + cow_bytes[0] / K),
            "d2h_bytes_per_step": int(bo), "ms_per_step": round(ms, 5), "steps": K,
            "host_plan_in_step": plan}


# --------------------------------------------------------------- oracle ----
class OracleSampler:
    """The float64 oracle (paged gather, then two-pass softmax) run on
    (sequence, KV head) groups of a workload.  The oracle pool is built once
    (untimed, data stored as float32 holding the bf16 values exactly); only the
    gather and attention calls are timed.  ``q8`` ("int8" / "fp8"): the
    oracle pool holds, in float64, the value that pool type stores for each
    appended row (quantised once, untimed); ``window`` / ``sinks``: the
    windowed decode over the visible keys only."""

    def __init__(self, w, q8=False, window=0, sinks=0):
        import torch
        from oracle import KVPool
        self.w = w
        self.q8, self.window, self.sinks = q8, window, sinks
        self.G = w.num_heads // w.num_kv_heads
        self.q = w.queries().to(torch.float64).numpy()
        from oracle import stored_rows, stored_rows_fp8
        rows = stored_rows_fp8 if q8 == "fp8" else stored_rows
        p = KVPool(w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim, w.order,
                   store_heads="all", dtype=np.float64 if q8 else np.float32)
        for op in w.setup + w.step:
            if op.kind == "create":
                p.create(op.args[0])
            elif op.kind == "share":
                p.share_prefix(*op.args)
            elif op.kind == "release":
                p.release(op.args[0])
            else:
                k, v = w.kv_for(op)
                if q8:
                    kr, vr = rows(k.double().numpy())[2], rows(v.double().numpy())[2]
                else:
                    kr, vr = k.float().numpy(), v.float().numpy()
                p.append(op.args[0], op.args[1], kr, vr)
        self.pool = p
        self.next = 0

    def run(self, budget_s, max_units=None, keep=0):
        """Decode (or prefill) whole sequences -- every head -- until the
        budget is spent; returns (bytes or flops, seconds, sequences).  The
        outputs of the first ``keep`` sequences are kept in ``self.outs``."""
        from oracle import attention_window, paged_attention
        w, p = self.w, self.pool
        tok_bytes = 2 * w.head_dim + 8 if self.q8 else \
            w.head_dim * 2 * (2 if w.dtype == "bf16" else 4)
        work, spent, done = 0, 0.0, 0
        self.outs = {}
        while spent < budget_s and (max_units is None or done < max_units):
            si = self.next % len(w.decode_seqs)
            self.next += 1
            seq = w.decode_seqs[si]
            t0 = time.perf_counter()
            if self.window:
                k, v = p.gather(seq)
                o = attention_window(self.q[si], k, v, self.window, self.sinks)
            else:
                o = paged_attention(p, seq, self.q[si])    # gather + two-pass softmax
            spent += time.perf_counter() - t0
            if len(self.outs) < keep:
                self.outs[si] = o
            L = p.lengths[seq]
            if w.q_tokens > 1:
                qn = w.q_tokens
                work += 4 * w.head_dim * w.num_heads * (qn * (L - qn) + qn * (qn + 1) // 2)
            else:
                vis = min(L, self.window + self.sinks) if self.window else L
                work += vis * w.num_kv_heads * tok_bytes
            done += 1
        return work, spent, done


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return {i.get("internal_api", "?"): i.get("num_threads") for i in threadpool_info()}
    except Exception:
        return None


def oracle_desc(q8, window, sinks):
    return ("oracle paged gather + float64 two-pass softmax"
            + (f" over the window {window} + {sinks} sinks" if window else "")
            + (f", pool holding the rows an {q8} pool stores (quantised once, untimed)"
               if q8 else ""))


def cpu_baseline(w, args, gpu_out=None, q8=False, window=0, sinks=0):
    sampler = OracleSampler(w, q8, window, sinks)
    work, spent, done = sampler.run(args.cpu_budget, keep=2 if gpu_out is not None else 0)
    distinct = min(done, len(w.decode_seqs))
    desc = (f"{done} sequence decodes (all heads) over {distinct} distinct sequences of "
            f"{w.name}: " + oracle_desc(q8, window, sinks))
    if w.q_tokens > 1:
        val, unit = work / spent / 1e12, "TFLOP/s"
    else:
        val, unit = work / spent / 1e9, "GB/s"
    res = {"value": round(val, 6), "unit": unit, "cores": oracle_threads(), "kind": "oracle",
           "sample": desc, "seconds": round(spent, 2), "host_cpus": os.cpu_count(),
           "blas_threads": blas_threads()}
    if gpu_out is not None and sampler.outs:
        # the timed step's output against the oracle's, on the sequences it ran
        err = 0.0
        for si, o in sampler.outs.items():
            got = gpu_out[si] if w.q_tokens > 1 else gpu_out[si][None]
            err = max(err, float(np.abs(got - o).max()))
        res["max_abs_err_vs_gpu"] = err
        res["compared_sequences"] = sorted(int(i) for i in sampler.outs)
    return res


def metric_name(w, q8=False, window=0, sinks=0):
    """The metric both arms report for a workload and pool type."""
    if w.q_tokens > 1:
        return "chunked prefill attention TFLOP/s (causal pairs), 8 x 512 over 4608, GQA 32/8"
    m = (f"decode {q8}-KV HBM GB/s (codes + scales read) and seqs/s at 8K ctx, GQA 32/8" if q8
         else "decode KV HBM GB/s (fraction of B200 peak) and seqs/s at 8K ctx, GQA 32/8")
    if window:
        m += f", window {window} + {sinks} sinks (visible keys only)"
    return m


def run_reference(args, dist):
    """The float64 oracle as the reference arm, on this host's cores."""
    if dist.rank != 0:
        return None
    builder = workloads.ALL[args.config]
    w = builder() if args.seed is None else builder(seed=args.seed)
    q8 = args.kv if args.kv in ("int8", "fp8") else False
    if (q8 or args.window) and w.q_tokens > 1:
        raise SystemExit("--kv int8/fp8 and --window apply to the decode workloads")
    sampler = OracleSampler(w, q8, args.window, args.sinks)
    # each step: one bounded sample (whole groups) so the run stays ~2-3 minutes
    per_step = max(0.005, 120.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        sampler.run(per_step, max_units=1)
    work, spent, groups, steps = 0, 0.0, 0, 0
    for _ in range(args.steps):
        wk, sp, n = sampler.run(per_step)
        work, spent, groups, steps = work + wk, spent + sp, groups + n, steps + 1
        if spent > 150:
            break
    desc = (f"{groups} sequences (all heads) of {w.name} over {steps} steps: "
            + oracle_desc(q8, args.window, args.sinks))
    metric = metric_name(w, q8, args.window, args.sinks)
    if w.q_tokens > 1:
        val, unit = work / spent / 1e12, "TFLOP/s"
    else:
        val, unit = work / spent / 1e9, "GB/s"
    ms = spent / max(1, steps) * 1e3
    return {"impl": "reference", "metric": metric, "value": round(val, 6), "unit": unit,
            "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1), bf16-rounded)",
            "config": {**config_of(w, args.kv, args.window, args.sinks, dist), "sample": desc},
            "cpu_baseline": {"value": round(val, 6), "unit": unit, "cores": oracle_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(val, 6), "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=["tiny", "decode32", "ragged256", "splitk128k", "prefill"],
                    default="decode32")
    ap.add_argument("--e2e-steps", type=int, default=200,
                    help="steps of each end-to-end measurement (independent of --steps)")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kv", choices=["bf16", "int8", "fp8"], default="bf16",
                    help="KV pool type for the decode workloads (int8 / fp8: per-row absmax "
                         "integer / E4M3 codes)")
    ap.add_argument("--window", type=int, default=0,
                    help="decode over the last WINDOW keys (plus --sinks first keys); 0 = all")
    ap.add_argument("--sinks", type=int, default=0)
    ap.add_argument("--seed", type=int, default=None,
                    help="workload seed (default: the configuration's own)")
    ap.add_argument("--configs", choices=["auto", "all", "none"], default="auto",
                    help="also measure every other workload under 'configs' (auto: on the "
                         "default decode32 run at one GPU)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    dist = Dist(args.gpus)
    if args.impl == "reference":
        res = run_reference(args, dist)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    dist.init("nccl")
    global SAMPLER
    try:
        import torch
        torch.cuda.set_device(dist.local)
        SAMPLER = ClockSampler(dist.local)
        memo = {}
        # the headline: exactly --steps timed steps; the clock sampler runs fast
        # enough to see a few milliseconds
        res = run_workload(args, dist, args.config, args.kv, args.window, args.sinks,
                           steps=args.steps,
                           cpu=not args.no_cpu_baseline, memo=memo)
        default_run = (args.config == "decode32" and args.kv == "bf16" and not args.window)
        extras = args.configs == "all" or (args.configs == "auto" and default_run
                                           and dist.world == 1)
        if extras:
            res["configs"] = run_extras(args, dist, memo)
        if dist.rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if SAMPLER is not None:
            SAMPLER.close()
        dist.close()


# (name, workload, pool type, window, sinks)
EXTRAS = [("ragged256", "ragged256", "bf16", 0, 0), ("splitk128k", "splitk128k", "bf16", 0, 0),
          ("prefill", "prefill", "bf16", 0, 0), ("decode32_int8", "decode32", "int8", 0, 0),
          ("decode32_fp8", "decode32", "fp8", 0, 0),
          ("decode32_window1024_sinks4", "decode32", "bf16", 1024, 4)]


def run_extras(args, dist, memo):
    """Every other workload, each timed for at least ~100 ms (so the clock
    sampler sees it), with its own roofline, e2e and clocks.  No CPU baseline
    here (the headline line carries it)."""
    out = {}
    keep = ("metric", "value", "unit", "steps", "ms_per_step", "dtype", "config", "seqs_per_s",
            "tflops", "kv_bytes_vs_bf16", "host_plan_us", "gpu_launches", "roofline", "e2e",
            "clocks", "frac_of_peak")
    for name, config, kv, win, sinks in EXTRAS:
        r = run_workload(args, dist, config, kv, win, sinks, steps=args.steps, min_ms=100.0,
                         memo=memo if config == "decode32" else None)
        out[name] = {k: r[k] for k in keep if k in r}
        if r.get("append"):
            out["prefill_append"] = {"workload": "prefill chunk append: 8 x 512 tokens, 8 KV "
                                                 "heads, head_dim 128, bf16 (reshape_and_cache)",
                                     **r["append"]}
    memo.clear()
    return out


if __name__ == "__main__":
    main()
