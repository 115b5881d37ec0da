"""Benchmark of the paged KV-cache decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one decode step of one layer over the whole batch: the block manager
appends one slot per sequence (copy-on-write pairs where a block is shared), the
metadata goes to the device, pa_copy_blocks, pa_reshape_and_cache and
pa_decode_attention run.  Inputs are synthetic (seeded, see ``workloads``) and
resident in HBM before the timed region; the K/V pool is far larger than L2, so no
flush is needed between steps.

Under torchrun each rank runs its own replica (its own pool, sequences and seed):
the path has no exchange step, so there is no collective on the data path; the
ranks meet only at the barriers around the timed region and in the max-reduction
of the elapsed time.  Rank 0 prints one JSON line.

``--impl reference`` times the CPU oracle (rank 0 only) on bounded samples of the
same workload and prints the same metric.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

METRIC = "paged decode attention: achieved HBM GB/s vs peak; sequences/sec per layer"
PEAKS_FILE = os.path.join(HERE, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    # smaller instances of a workload for profiling captures (reported in "config")
    ap.add_argument("--seqs", type=int, default=None, help="override the batch size")
    ap.add_argument("--pool-blocks", type=int, default=None, help="override the pool size")
    # the pages' block-size trade-off: same lengths and slot capacity, other block size
    ap.add_argument("--block-size", type=int, default=None,
                    help="override the block size (pool keeps the same number of slots)")
    ap.add_argument("--measure", default="decode", choices=["decode", "swap"],
                    help="swap: time swapping half the batch to a pinned host pool and back")
    ap.add_argument("--partition-size", type=int, default=None,
                    help="override the partition size of the decode split")
    ap.add_argument("--cache-fp8", action="store_true",
                    help="store K/V as fp8 e4m3 with per-tensor scales (q/out keep the dtype)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# algorithmic bytes (what one step must move at least once)
# ---------------------------------------------------------------------------

def decode_bytes(cfg, lens, unique_tokens=None, kv_elem_bytes=None) -> int:
    """K/V of every cached token once + q + out + block-table entries + lengths.
    ``unique_tokens`` (shared-prefix workloads) counts each physical slot once;
    ``kv_elem_bytes`` is the cache element size when it differs from q's (fp8)."""
    E = cfg.elem_bytes
    EKV = E if kv_elem_bytes is None else kv_elem_bytes
    tokens = int(np.sum(lens)) if unique_tokens is None else int(unique_tokens)
    kv = tokens * cfg.num_kv_heads * cfg.head_dim * 2 * EKV
    qo = 2 * cfg.num_seqs * cfg.num_heads * cfg.head_dim * E
    tab = int(np.sum((np.asarray(lens) + cfg.block_size - 1) // cfg.block_size)) * 4
    return kv + qo + tab + 4 * cfg.num_seqs


def cache_op_bytes(cfg, num_tokens, num_pairs, kv_elem_bytes=None) -> int:
    E = cfg.elem_bytes
    EKV = E if kv_elem_bytes is None else kv_elem_bytes
    row_in = cfg.num_kv_heads * cfg.head_dim * E
    row = cfg.num_kv_heads * cfg.head_dim * EKV
    reshape = 2 * num_tokens * (row_in + row) + 8 * num_tokens  # K and V: read + write
    copy = 2 * 2 * num_pairs * cfg.block_size * row              # K and V blocks: read + write
    return reshape + copy


def unique_context_tokens(dec, cfg, seq_ids) -> int:
    """Distinct physical slots the decode reads: a shared block counts once, at the
    longest fill among the sequences that map it."""
    fill = {}
    for s in seq_ids:
        blocks = dec.alloc.seq_blocks(int(s))
        L = dec.alloc.seq_len(int(s))
        for j, b in enumerate(blocks):
            n = min(cfg.block_size, L - j * cfg.block_size)
            fill[b] = max(fill.get(b, 0), n)
    return sum(fill.values())


# ---------------------------------------------------------------------------
# replicas: one process per GPU, no collective on the data path
# ---------------------------------------------------------------------------

def replica_env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_seed(base_seed: int, rank: int) -> int:
    """Each rank decodes its own replica of the workload (weak scaling)."""
    return base_seed + rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The slowest rank's elapsed time: every rank must call this, in the same order."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    """The sum over ranks (every rank must call this, in the same order)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_throughput(job_bytes_per_step: float, steps: int, elapsed_max_ms: float) -> float:
    """Whole-job GB/s: the bytes all ranks move per step (their replicas differ: each
    draws its own lengths) over the slowest rank's time."""
    return float(job_bytes_per_step) * steps / (elapsed_max_ms * 1e-3) / 1e9


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        import threading
        self.lines, self.first = [], threading.Event()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return self

        def reader():
            for line in self.proc.stdout:
                if line.strip():
                    self.lines.append((time.perf_counter(), line.strip()))
                    self.first.set()
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        self.first.wait(timeout=10)       # sampling is running before the timed region
        self.t0 = time.perf_counter()
        return self

    def __exit__(self, *a):
        self.t1 = time.perf_counter()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)
            self.lines = [l for t, l in self.lines if self.t0 <= t <= self.t1]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------

def host_cpu() -> dict:
    """The host's logical CPU count and model name (for the CPU baseline)."""
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"logical_cpus": os.cpu_count(), "model": model}


class OracleTimer:
    """The CPU oracle's decode attention on whole sequences (all heads)."""

    def __init__(self, cfg, inp):
        from oracle.step import build_context
        self.cfg, self.inp = cfg, inp
        bm, self.k, self.v, _ = build_context(inp, copy_pool=False)
        ids = list(range(cfg.num_seqs))
        width = max(len(bm.tables[s]) for s in ids) + 1
        rows, lens = bm.block_tables(ids, width)
        self.tables, self.lens = np.array(rows, np.int32), np.array(lens, np.int64)
        try:
            from threadpoolctl import threadpool_info
            self.threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        except Exception:
            self.threads = 1

    def run(self, seqs):
        """Seconds spent and algorithmic bytes covered for the listed sequences."""
        from oracle.attention import paged_decode_attention
        cfg = self.cfg
        t0 = time.perf_counter()
        paged_decode_attention(self.inp.q, self.k, self.v, self.tables, self.lens, cfg.scale,
                               cfg.block_size, cfg.num_kv_heads, cfg.dtype, seqs=seqs)
        dt = time.perf_counter() - t0
        return dt, decode_bytes(cfg.with_(num_seqs=len(seqs)), self.lens[list(seqs)])

    def budgeted(self, budget_s: float):
        """Whole sequences in index order, cycling over the batch, until the budget is
        spent: (GB/s, seq/s, text)."""
        t_all, b_all, n, tokens = 0.0, 0, 0, 0
        S = self.cfg.num_seqs
        while t_all <= budget_s:
            s = n % S
            dt, b = self.run([s])
            t_all, b_all, n, tokens = t_all + dt, b_all + b, n + 1, tokens + int(self.lens[s])
        passes = n / S
        desc = (f"oracle decode attention (float64, all {self.cfg.num_heads} heads) over "
                f"{n} sequences ({passes:.2f} passes over the {S}-sequence batch, "
                f"{tokens} tokens), {t_all:.1f} s")
        return b_all / t_all / 1e9, n / t_all, desc


def run_reference(args, cfg):
    """The oracle as the reference arm: rank 0 only; each step is the oracle on a
    bounded sample of the workload (two sequences, all heads)."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    from workloads import make_inputs
    timer = OracleTimer(cfg, make_inputs(cfg, args.seed))
    # bounded: about 2 minutes of oracle work at the default step count
    per_step = 1 if args.steps * 1 > 500 else 2
    steps = min(args.steps, 200)
    t_all, b_all = 0.0, 0
    warm = min(args.warmup, 3)
    for i in range(warm + steps):
        seqs = [(i * per_step + j) % cfg.num_seqs for j in range(per_step)]
        dt, b = timer.run(seqs)
        if i >= warm:
            t_all, b_all = t_all + dt, b_all + b
    value = b_all / t_all / 1e9
    sample = (f"per step: oracle decode attention (float64, all {cfg.num_heads} heads) of "
              f"{per_step} of the {cfg.num_seqs} sequences, cycling through the batch; "
              f"{steps} timed steps (at most 200 of the requested {args.steps})")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warm,
        "ms_per_step": round(1e3 * t_all / steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "seqs_per_s": round(per_step * steps / t_all, 4),
        "config": {"workload": cfg.name, "description": cfg.description},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": timer.threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, cfg):
    import torch
    import torch.distributed as dist

    world, rank, local = replica_env()

    import paged_kv_cache_342_b200 as pa
    from paged_kv_cache_342_b200.runtime import PagedDecoder
    from workloads import TORCH_DTYPES, make_inputs, step_tokens, storage_to_torch

    # CPU baseline first (before any GPU work), rank 0 at N=1 only
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        timer = OracleTimer(cfg, make_inputs(cfg, args.seed))
        gbs, sps, desc = timer.budgeted(12.0)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": timer.threads, "kind": "oracle",
               "sample": desc, "seqs_per_s": round(sps, 3), "host": host_cpu()}
        try:  # the same oracle on one core
            from threadpoolctl import threadpool_limits
            with threadpool_limits(1):
                gbs1, sps1, desc1 = timer.budgeted(4.0)
            cpu["single_core"] = {"value": round(gbs1, 4), "unit": "GB/s", "cores": 1,
                                  "sample": desc1, "seqs_per_s": round(sps1, 3)}
        except ImportError:
            pass
        del timer

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    seed = replica_seed(args.seed, rank)
    inp = make_inputs(cfg, seed)
    S, Hq, Hkv, D, bs = cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    max_len = int((inp.context_lens + 1).max()) + 1
    max_blocks = (max_len + bs - 1) // bs
    kd = storage_to_torch(inp.k_pool, cfg.dtype).to(dev)
    vd = storage_to_torch(inp.v_pool, cfg.dtype).to(dev)
    kv_scales, ekv = None, None
    if args.cache_fp8:
        # quantize the pool on the device with the library's fp8 write (all slots)
        kv_scales, ekv = (8.0 * cfg.std / 448.0,) * 2, 1
        NB = cfg.num_blocks
        slots_all = torch.arange(NB * bs, dtype=torch.int64, device=dev)
        k8 = torch.empty(kd.shape, dtype=torch.uint8, device=dev)
        v8 = torch.empty_like(k8)
        for src, dst in ((kd, k8), (vd, v8)):
            rows = src.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D).contiguous()
            pa.pa_reshape_and_cache_fp8(rows, rows, dst, dst, slots_all, *kv_scales)
            del rows
        kd, vd = k8, v8
        torch.cuda.synchronize(dev)
    pool_bytes = 2 * kd.numel() * kd.element_size()
    del inp.k_pool, inp.v_pool
    dec = PagedDecoder(kd, vd, Hq, cfg.scale, max_blocks, inp.free_order, cfg.partition_size,
                       kv_scales=kv_scales, query_dtype=TORCH_DTYPES[cfg.dtype])
    if inp.prefix is None:
        for s in range(S):
            dec.admit(s, int(inp.context_lens[s]))
    else:
        p = inp.prefix
        dec.apply_copies(dec.admit_shared_prefix(p.groups, p.samples, p.prefix_len,
                                                 p.private_lens))
    # every step decodes the same lengths: sequences roll back one token per step
    dec.bind(range(S), rolling=True)

    # a ring of distinct per-step token sets: pinned host copies and device copies
    ring = 8
    toks_h, toks_d = [], []
    for i in range(ring):
        q, nk, nv = (inp.q, inp.new_k, inp.new_v) if i == 0 else step_tokens(cfg, seed, i)
        h = [storage_to_torch(a, cfg.dtype).pin_memory() for a in (q, nk, nv)]
        toks_h.append(h)
        toks_d.append([t.to(dev) for t in h])
    out = torch.empty((S, Hq, D), dtype=TORCH_DTYPES[cfg.dtype], device=dev)
    stream = torch.cuda.current_stream(dev)

    def one_step(tokens, ev=None):
        q, nk, nv = tokens
        return dec.step(q, nk, nv, out, events=ev)

    warm_cow = 0
    for i in range(args.warmup):
        warm_cow += one_step(toks_d[i % ring])["num_cow"]
    torch.cuda.synchronize(dev)
    if pa.pa_device_error_read() != 0:
        raise RuntimeError("device error word set during warm-up")

    # the workload is stationary from here on: bytes per step computed once
    meta0 = one_step(toks_d[0])
    torch.cuda.synchronize(dev)
    lens = np.array([dec.alloc.seq_len(s) for s in range(S)], np.int64)
    uniq = unique_context_tokens(dec, cfg, range(S)) if inp.prefix is not None else None
    dec_bytes = decode_bytes(cfg, lens, uniq, ekv)
    step_bytes = dec_bytes + cache_op_bytes(cfg, S, 0, ekv)
    logical_dec_bytes = decode_bytes(cfg, lens, None, ekv)
    launches_per_step = dec.kernel_launches(meta0)

    # per-call events on a sample of the steps (the decode call's own duration)
    n_ev = min(args.steps, 200)
    ev_every = max(1, args.steps // n_ev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n_ev)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cows = 0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        t_start.record(stream)
        e = 0
        for k in range(args.steps):
            ev = None
            if k % ev_every == 0 and e < n_ev:
                ev, e = evs[e], e + 1
            cows += one_step(toks_d[k % ring], ev)["num_cow"]
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    dec_ms = [a.elapsed_time(b) for a, b in evs[:e]]
    err = pa.pa_device_error_read()
    if err:
        raise RuntimeError(f"device error word {err} after the timed region")
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    job_step_bytes = sum_over_ranks(step_bytes, world, dev)
    value = job_throughput(job_step_bytes, args.steps, elapsed_ms)
    seqs_per_s = S * world * args.steps / (elapsed_ms * 1e-3)

    # ---- a pool that fits in L2: the decode call also timed cold ---------------------
    cold_ms = None
    if pool_bytes <= L2_BYTES and rank == 0:
        # between calls, write a buffer of twice the L2 size so that nothing of the
        # pool stays cached (the warm figures above are the steady state)
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
        cevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(50)]
        for ev in cevs:
            flush.fill_(1)
            one_step(toks_d[0], ev)
        torch.cuda.synchronize(dev)
        cold_ms = [a.elapsed_time(b) for a, b in cevs]
        del flush

    # ---- end to end through the public API with host buffers ----------------------
    e2e = None
    if not args.no_e2e:
        # the public host-buffer step: inputs from pinned memory, result back to it,
        # copies overlapped with the neighbouring steps' kernels
        outs_h = [torch.empty((S, Hq, D), dtype=TORCH_DTYPES[cfg.dtype], pin_memory=True)
                  for _ in range(2)]
        done = [None, None]

        def e2e_step(k):
            if done[k % 2] is not None:
                done[k % 2].synchronize()          # the caller consumed that result
            done[k % 2] = dec.step_host(*toks_h[k % ring], outs_h[k % 2])

        for k in range(3):
            e2e_step(k)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for k in range(args.steps):
            e2e_step(k)
        dec.drain_host_io()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        E = job_throughput(job_step_bytes, args.steps, e_ms)
        h2d = sum(t.numel() * t.element_size() for t in toks_h[0]) + dec.staging_bytes
        d2h = S * Hq * D * cfg.elem_bytes
        e2e = {"value": round(E, 2), "unit": "GB/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": round(e_ms / args.steps, 4),
               "seqs_per_s": round(S * world * args.steps / (e_ms * 1e-3), 1)}

    # ---- roofline of the decode call --------------------------------------------
    peak, peak_kind = hbm_peak()
    dec_avg_ms = statistics.mean(dec_ms)
    achieved = dec_bytes / (dec_avg_ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
            "kernel": ("pa_decode_attention_fp8" if args.cache_fp8 else "pa_decode_attention")
                      + " (partition kernel + log-sum-exp merge)",
            "bytes_per_launch": int(dec_bytes), "avg_launch_us": round(dec_avg_ms * 1e3, 2),
            "launches_timed": len(dec_ms),
            "median_launch_us": round(statistics.median(dec_ms) * 1e3, 2),
            "frac_of_nominal_8000": round(achieved / 8000.0, 4),
            "traffic": None if args.cache_fp8 else recorded_traffic(cfg)}  # records: 16-bit caches
    if cold_ms:
        roof["cold_median_launch_us"] = round(statistics.median(cold_ms) * 1e3, 2)
        roof["cold_note"] = "pool smaller than L2: calls after a 2x-L2 buffer write"
    if uniq is not None:
        roof["logical_bytes_per_launch"] = int(logical_dec_bytes)
        roof["logical_achieved"] = round(logical_dec_bytes / (dec_avg_ms * 1e-3) / 1e9, 1)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(elapsed_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "seqs_per_s": round(seqs_per_s, 1),
            "config": {"workload": cfg.name, "description": cfg.description,
                       "num_seqs": S, "num_heads": Hq, "num_kv_heads": Hkv, "head_dim": D,
                       "block_size": bs, "num_blocks": cfg.num_blocks,
                       "partition_size": dec.partition_size,
                       "partition_rule": ("pa_decode_partition_size" if cfg.partition_size == 0
                                          else "fixed"),
                       "mean_seq_len": round(float(lens.mean()), 1),
                       "max_seq_len": int(lens.max()),
                       "l2": ("inputs larger than L2 (K/V pool %.2f GB per rank), no flush"
                              % (pool_bytes / 1e9)) if pool_bytes > L2_BYTES else
                             ("K/V pool of %.1f KB fits in L2: a parity-size workload, "
                              "no flush" % (pool_bytes / 1e3)),
                       "steps": "each step appends one token per sequence and rolls the "
                                "previous one back, so every step decodes these lengths",
                       "parallelism": f"replicas x{world}",
                       "workspace_bytes": int(dec.workspace_bytes),
                       "prefix_group_chunks": int(meta0.get("num_chunks", 0)),
                       "pool": pool_summary(dec.alloc.stats()),
                       "cow_pairs_in_warmup": warm_cow, "cow_pairs_in_timed_steps": cows,
                       "kv_cache": ("fp8 e4m3, per-tensor scales %g" % kv_scales[0])
                                   if args.cache_fp8 else cfg.dtype},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


L2_BYTES = 126 * 1000 * 1000  # B200 L2


def pool_summary(st: dict) -> dict:
    """Block-manager view of the batch: blocks in use, slots, and the tail waste
    (unused slots of each sequence's last block) as a share of allocated slots."""
    return {"used_blocks": st["used_blocks"], "shared_blocks": st["shared_blocks"],
            "allocated_slots": st["allocated_slots"], "logical_tokens": st["logical_tokens"],
            "tail_waste_pct": round(100.0 * st["tail_waste_slots"] / max(1, st["allocated_slots"]), 3)}


def recorded_traffic(cfg):
    """DRAM bytes per decode call from the committed ncu capture of this workload,
    if it was taken on the current kernel sources (else None)."""
    path = os.path.join(HERE, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(cfg.name)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("kernel_sources_sha256") != kernel_sources_sha():
        return None
    return rec.get("traffic_bytes_per_launch")


def kernel_sources_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(HERE, "paged_kv_cache_342_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        # the kernels a decode call runs (the step runtime's host code is not one)
        if (name.startswith("decode") and not name.startswith("decoder")) or \
                name in ("common.cuh", "tensor_map.cu"):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def run_swap(args, cfg):
    """Preemption by swapping: half the batch moves to a page-locked host pool and
    back each step (pa_seqs_move + pa_swap_blocks); reports the copy throughput over
    the host link, device-timed with CUDA events."""
    import torch

    import paged_kv_cache_342_b200 as pa
    from workloads import make_inputs, storage_to_torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = make_inputs(cfg, args.seed)
    S, bs = cfg.num_seqs, cfg.block_size
    kd = storage_to_torch(inp.k_pool, cfg.dtype).to(dev)
    vd = storage_to_torch(inp.v_pool, cfg.dtype).to(dev)
    dev_pool = pa.BlockAllocator(cfg.num_blocks, bs, inp.free_order)
    for s_ in range(S):
        dev_pool.add(s_, int(inp.context_lens[s_]))
    victims = list(range(S // 2, S))
    need = sum(len(dev_pool.seq_blocks(v)) for v in victims)
    host_pool = pa.BlockAllocator(need, bs)
    kh = torch.empty((need,) + tuple(kd.shape[1:]), dtype=kd.dtype).pin_memory()
    vh = torch.empty_like(kh).pin_memory()
    block_bytes = kd[0].numel() * kd.element_size()
    stream = torch.cuda.current_stream(dev)
    mapping = torch.empty((need, 2), dtype=torch.int32, device=dev)

    def swap(src_pool, dst_pool, dk, dv, sk, sv, ev=None):
        pairs = src_pool.move_to(dst_pool, victims)
        mapping[:len(pairs)].copy_(torch.from_numpy(pairs))
        if ev is not None:
            ev[0].record(stream)
        pa.pa_swap_blocks(dk, dv, sk, sv, mapping[:len(pairs)], pairs)
        if ev is not None:
            ev[1].record(stream)
        return len(pairs)

    for _ in range(args.warmup):
        swap(dev_pool, host_pool, kh, vh, kd, vd)
        swap(host_pool, dev_pool, kd, vd, kh, vh)
    torch.cuda.synchronize(dev)
    steps = min(args.steps, 50)
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(2)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    moved = 0
    t0.record(stream)
    for k in range(steps):
        moved += swap(dev_pool, host_pool, kh, vh, kd, vd, evs[k][0])
        moved += swap(host_pool, dev_pool, kd, vd, kh, vh, evs[k][1])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if pa.pa_device_error_read():
        raise RuntimeError("device error word set")
    out_ms = statistics.mean(e[0][0].elapsed_time(e[0][1]) for e in evs)
    in_ms = statistics.mean(e[1][0].elapsed_time(e[1][1]) for e in evs)
    per_dir = need * block_bytes * 2          # K and V blocks one way
    line = {"metric": "swap to host and back: pa_swap_blocks GB/s over the host link",
            "value": round(2 * per_dir / ((out_ms + in_ms) * 1e-3) / 1e9, 2), "unit": "GB/s",
            "n_gpus": 1, "steps": steps, "warmup": args.warmup, "higher_is_better": True,
            "dtype": cfg.dtype, "data": "synthetic",
            "swap_out_GBs": round(per_dir / (out_ms * 1e-3) / 1e9, 2),
            "swap_in_GBs": round(per_dir / (in_ms * 1e-3) / 1e9, 2),
            "ms_per_round_trip_including_block_manager": round(t0.elapsed_time(t1) / steps, 3),
            "config": {"workload": cfg.name, "swapped_sequences": len(victims),
                       "blocks_each_way": need, "bytes_each_way": per_dir}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    from workloads import CONFIGS, HEADLINE
    cfg = CONFIGS[args.workload or HEADLINE]
    if args.seqs is not None:
        if cfg.lens[0] in ("fixed", "prefix"):
            raise SystemExit("--seqs applies to workloads with drawn lengths")
        cfg = cfg.with_(num_seqs=args.seqs, name=f"{cfg.name}_s{args.seqs}")
    if args.pool_blocks is not None:
        cfg = cfg.with_(num_blocks=args.pool_blocks, name=f"{cfg.name}_nb{args.pool_blocks}")
    if args.partition_size is not None and args.partition_size != cfg.partition_size:
        cfg = cfg.with_(partition_size=args.partition_size, name=f"{cfg.name}_ps{args.partition_size}")
    if args.block_size is not None and args.block_size != cfg.block_size:
        slots = cfg.num_blocks * cfg.block_size
        cfg = cfg.with_(block_size=args.block_size, num_blocks=slots // args.block_size,
                        name=f"{cfg.name}_bs{args.block_size}")
    if args.impl == "reference":
        run_reference(args, cfg)
    elif args.measure == "swap":
        run_swap(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
