"""Benchmark of the paged KV-cache decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one decode step of one layer over the whole batch: the block manager
appends one slot per sequence (copy-on-write pairs where a block is shared), the
metadata goes to the device, pa_copy_blocks, pa_reshape_and_cache and
pa_decode_attention run.  Inputs are synthetic (seeded, see ``workloads``) and
resident in HBM before the timed region; the K/V pool is far larger than L2, so no
flush is needed between steps.

Order of a run: set-up; untimed steps for --settle-ms (clocks up); W warm-up steps;
the timed region of exactly K steps (clocks sampled through NVML during it); the
decode call's own loop of --roofline-ms with CUDA events on a sample of its calls
(the roofline); K host-fed steps (e2e); at N=1 the other workloads
(``per_workload``: the 13B-shaped, long-context GQA, shared-prefix and tiny ones,
and fp8 caches), each with loops sized by time; then the CPU oracle on the host.

Under torchrun each rank runs its own replica (its own pool, sequences and seed):
the path has no exchange step, so there is no collective on the data path; the
ranks meet only at the barriers around the timed regions and in the max-reduction
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
    ap.add_argument("--settle-ms", type=float, default=500.0,
                    help="untimed steps before the warm-up, so that clocks settle")
    ap.add_argument("--roofline-ms", type=float, default=1000.0,
                    help="length of the loop in which the decode call is event-timed")
    ap.add_argument("--per-workload-ms", type=float, default=400.0,
                    help="length of each timed loop of the other workloads")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="measure only the selected workload")
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
    """SM clocks and clock-event reasons sampled during a timed region.

    NVML is polled from a thread about once a millisecond, so that even a region of
    a few milliseconds gets samples; without NVML, ``nvidia-smi -lms 50`` is the
    fallback.  Only samples taken between ``__enter__`` and ``__exit__`` count."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    _nvml = None

    def __init__(self, index: int, period_s: float = 0.001):
        self.index, self.period = index, period_s
        self.samples, self.max_mhz, self.source = [], None, None

    @classmethod
    def _handle(cls, index: int):
        try:
            import pynvml
            if cls._nvml is None:
                pynvml.nvmlInit()
                cls._nvml = pynvml
            handle = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(index).uuid)
                handle = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                handle = pynvml.nvmlDeviceGetHandleByIndex(index)
            return pynvml, handle
        except Exception:
            return None, None

    def __enter__(self):
        import threading
        self.stop = threading.Event()
        nv, h = self._handle(self.index)
        if nv is not None:
            self.source = "nvml"
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                                  getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))

            def poll():
                while not self.stop.is_set():
                    try:
                        mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        bits = int(get_reasons(h)) if get_reasons else 0
                        self.samples.append((time.perf_counter(), mhz, bits))
                    except Exception:
                        pass
                    self.stop.wait(self.period)
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
        else:
            self._start_smi()
        deadline = time.perf_counter() + 10
        while not self.samples and time.perf_counter() < deadline and self.source:
            time.sleep(0.001)          # sampling is running before the timed region
        self.t0 = time.perf_counter()
        return self

    def _start_smi(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.source = "nvidia-smi"

        def reader():
            for line in self.proc.stdout:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 7:
                    continue
                try:
                    mhz, self.max_mhz = float(parts[0]), float(parts[1])
                except ValueError:
                    continue
                bits = 0
                for (n, b), v in zip(self.REASONS, parts[3:7]):
                    if v.lower() == "active":
                        bits |= b
                self.samples.append((time.perf_counter(), mhz, bits))
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()

    def __exit__(self, *a):
        self.t1 = time.perf_counter()
        self.stop.set()
        proc = getattr(self, "proc", None)
        if proc is not None:
            proc.terminate()
            try:
                proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                proc.kill()
        if getattr(self, "thread", None) is not None:
            self.thread.join(timeout=5)

    def summary(self):
        inside = [(m, b) for t, m, b in self.samples if self.t0 <= t <= self.t1]
        sm = [m for m, _ in inside]
        reasons = sorted({n for _, b in inside for n, bit in self.REASONS if b & bit})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sm), "source": self.source}


REJECTED_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clocks_rejected(summary: dict) -> bool:
    """A region that saw a hardware or thermal slowdown, or SM clocks far below the
    maximum with no reason given (a leftover clock lock), is measured again."""
    if any(r in summary.get("reasons", ()) for r in REJECTED_REASONS):
        return True
    mhz, mx = summary.get("sm_mhz"), summary.get("sm_max_mhz")
    return bool(mhz and mx and mhz < 0.7 * mx and not summary.get("reasons"))


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


def workload_config(cfg, lens, world: int, cache_fp8: bool) -> dict:
    """The workload as both arms state it in their JSON line (static facts only)."""
    kv_elem = 1 if cache_fp8 else cfg.elem_bytes
    pool_bytes = 2 * cfg.num_blocks * cfg.num_kv_heads * cfg.block_size * cfg.head_dim * kv_elem
    return {
        "workload": cfg.name, "description": cfg.description,
        "num_seqs": cfg.num_seqs, "num_heads": cfg.num_heads,
        "num_kv_heads": cfg.num_kv_heads, "head_dim": cfg.head_dim,
        "block_size": cfg.block_size, "num_blocks": cfg.num_blocks,
        "partition_size": cfg.partition_size or "library choice (pa_decode_partition_size)",
        "mean_seq_len": round(float(np.mean(lens)), 1), "max_seq_len": int(np.max(lens)),
        "l2": ("inputs larger than L2 (K/V pool %.2f GB per rank), no flush"
               % (pool_bytes / 1e9)) if pool_bytes > L2_BYTES else
              ("K/V pool of %.1f KB fits in L2: a parity-size workload, no flush"
               % (pool_bytes / 1e3)),
        "steps": "each step appends one token per sequence and rolls the previous one "
                 "back, so every step decodes these lengths",
        "parallelism": f"replicas x{world}",
        "kv_cache": "fp8 e4m3, per-tensor scales" if cache_fp8 else cfg.dtype,
    }


def run_reference(args, cfg):
    """The oracle as the reference arm: rank 0 only; each step is the oracle on a
    bounded sample of the workload (whole sequences, all heads), the requested number
    of warm-up and timed steps."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    from workloads import draw_lengths, make_inputs
    world = int(os.environ.get("WORLD_SIZE", "1"))
    timer = OracleTimer(cfg, make_inputs(cfg, args.seed))
    # bounded: two sequences per step up to 500 steps, one beyond (the oracle takes
    # about 10-25 ms per 7B-shaped sequence)
    per_step = 2 if args.steps <= 500 else 1
    t_all, b_all = 0.0, 0
    for i in range(args.warmup + args.steps):
        seqs = [(i * per_step + j) % cfg.num_seqs for j in range(per_step)]
        dt, b = timer.run(seqs)
        if i >= args.warmup:
            t_all, b_all = t_all + dt, b_all + b
    value = b_all / t_all / 1e9
    sample = (f"per step: oracle decode attention (float64, all {cfg.num_heads} heads) of "
              f"{per_step} of the {cfg.num_seqs} sequences, cycling through the batch; "
              f"{args.steps} timed steps after {args.warmup} warm-up steps")
    lens, _ = draw_lengths(cfg, args.seed)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * t_all / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "seqs_per_s": round(per_step * args.steps / t_all, 4),
        "config": workload_config(cfg, lens, world, args.cache_fp8),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": timer.threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def _event_pair():
    import torch
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


class WorkloadRun:
    """One workload resident on the device, stepped through the library's step runtime.

    ``host_pool``: the K/V pool is the seeded host draw of ``workloads.make_inputs``
    (the CPU baseline then reads the same values); otherwise it is drawn on the
    device with the same distribution (``workloads.device_normal_fill``)."""

    RING = 8

    def __init__(self, cfg, seed: int, dev, cache_fp8: bool = False, host_pool: bool = True):
        import torch

        import paged_kv_cache_342_b200 as pa
        from paged_kv_cache_342_b200.runtime import PagedDecoder
        from workloads import (TORCH_DTYPES, device_normal_fill, make_inputs, step_tokens,
                               storage_to_torch)
        self.cfg, self.dev, self.pa, self.cache_fp8 = cfg, dev, pa, cache_fp8
        inp = make_inputs(cfg, seed, pool=host_pool)
        self.inp = inp
        S, Hq, Hkv, D, bs = (cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_dim,
                             cfg.block_size)
        max_len = int((inp.context_lens + 1).max()) + 1
        max_blocks = (max_len + bs - 1) // bs
        if host_pool:
            kd = storage_to_torch(inp.k_pool, cfg.dtype).to(dev)
            vd = storage_to_torch(inp.v_pool, cfg.dtype).to(dev)
        else:
            shape = (cfg.num_blocks, Hkv, bs, D)
            kd = device_normal_fill(shape, cfg.dtype, cfg.std, seed, 2, dev)
            vd = device_normal_fill(shape, cfg.dtype, cfg.std, seed, 3, dev)
        self.kv_scales, self.ekv = None, None
        if cache_fp8:
            # quantize the pool on the device with the library's fp8 write (all slots)
            self.kv_scales, self.ekv = (8.0 * cfg.std / 448.0,) * 2, 1
            NB = cfg.num_blocks
            slots_all = torch.arange(NB * bs, dtype=torch.int64, device=dev)
            k8 = torch.empty(kd.shape, dtype=torch.uint8, device=dev)
            v8 = torch.empty_like(k8)
            for src, dst in ((kd, k8), (vd, v8)):
                rows = src.permute(0, 2, 1, 3).reshape(NB * bs, Hkv, D).contiguous()
                pa.pa_reshape_and_cache_fp8(rows, rows, dst, dst, slots_all, *self.kv_scales)
                del rows
            kd, vd = k8, v8
            torch.cuda.synchronize(dev)
        self.pool_bytes = 2 * kd.numel() * kd.element_size()
        self.kd, self.vd = kd, vd
        dec = PagedDecoder(kd, vd, Hq, cfg.scale, max_blocks, inp.free_order,
                           cfg.partition_size, kv_scales=self.kv_scales,
                           query_dtype=TORCH_DTYPES[cfg.dtype])
        if inp.prefix is None:
            for s in range(S):
                dec.admit(s, int(inp.context_lens[s]))
        else:
            p = inp.prefix
            dec.apply_copies(dec.admit_shared_prefix(p.groups, p.samples, p.prefix_len,
                                                     p.private_lens))
        # every step decodes the same lengths: sequences roll back one token per step
        dec.bind(range(S), rolling=True)
        self.dec = dec
        # a ring of distinct per-step token sets: pinned host copies and device copies
        self.toks_h, self.toks_d = [], []
        for i in range(self.RING):
            q, nk, nv = (inp.q, inp.new_k, inp.new_v) if i == 0 else step_tokens(cfg, seed, i)
            h = [storage_to_torch(a, cfg.dtype).pin_memory() for a in (q, nk, nv)]
            self.toks_h.append(h)
            self.toks_d.append([t.to(dev) for t in h])
        self.out = torch.empty((S, Hq, D), dtype=TORCH_DTYPES[cfg.dtype], device=dev)
        self.stream = torch.cuda.current_stream(dev)
        self.k = 0
        # the workload is stationary: bytes per step computed once
        self.meta0 = self.step()
        torch.cuda.synchronize(dev)
        self.lens = np.array([dec.alloc.seq_len(s) for s in range(S)], np.int64)
        self.uniq = (unique_context_tokens(dec, cfg, range(S)) if inp.prefix is not None
                     else None)
        self.dec_bytes = decode_bytes(cfg, self.lens, self.uniq, self.ekv)
        self.step_bytes = self.dec_bytes + cache_op_bytes(cfg, S, 0, self.ekv)
        self.logical_dec_bytes = decode_bytes(cfg, self.lens, None, self.ekv)
        self.launches_per_step = dec.kernel_launches(self.meta0)
        if host_pool:
            pass                      # the host pool stays for the CPU baseline
        self.check_errors("set-up")

    def step(self, ev=None):
        q, nk, nv = self.toks_d[self.k % self.RING]
        self.k += 1
        return self.dec.step(q, nk, nv, self.out, events=ev)

    def check_errors(self, where: str):
        err = self.pa.pa_device_error_read()
        if err:
            raise RuntimeError(f"device error word {err} ({where})")

    def run_for(self, seconds: float) -> int:
        """Untimed steps for about ``seconds`` of device time (clocks settle)."""
        import torch
        n, t0 = 0, time.perf_counter()
        while True:
            for _ in range(10):
                self.step()
            n += 10
            torch.cuda.synchronize(self.dev)
            if time.perf_counter() - t0 >= seconds:
                return n

    def steps_for(self, seconds: float, lo: int = 20, hi: int = 20000) -> int:
        """How many steps take about ``seconds`` (from 10 event-timed steps)."""
        import torch
        a, b = _event_pair()
        a.record(self.stream)
        for _ in range(10):
            self.step()
        b.record(self.stream)
        torch.cuda.synchronize(self.dev)
        per = a.elapsed_time(b) / 10 * 1e-3
        return int(min(hi, max(lo, round(seconds / max(per, 1e-7)))))

    def timed(self, steps: int, world: int = 1, dist=None, clock_index: int = 0):
        """Exactly ``steps`` steps between two events, bracketed by barrier +
        synchronize; returns (elapsed ms, clocks summary, copy pairs)."""
        import torch
        t0, t1 = _event_pair()
        cows = 0
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(self.dev)
        with ClockSampler(clock_index) as clk:
            t0.record(self.stream)
            for _ in range(steps):
                cows += self.step()["num_cow"]
            t1.record(self.stream)
            torch.cuda.synchronize(self.dev)
        if world > 1:
            dist.barrier()
        self.check_errors("timed region")
        return t0.elapsed_time(t1), clk.summary(), cows

    def roofline_loop(self, seconds: float, clock_index: int = 0, samples: int = 200):
        """Steps for about ``seconds``, the decode call event-timed on ``samples`` of
        them (every k-th step); returns (call ms list, clocks summary)."""
        import torch
        n = self.steps_for(seconds, lo=samples)
        every = max(1, n // samples)
        evs = [_event_pair() for _ in range(n // every + 1)]
        torch.cuda.synchronize(self.dev)
        e = 0
        with ClockSampler(clock_index) as clk:
            for i in range(n):
                ev = None
                if i % every == 0:
                    ev, e = evs[e], e + 1
                self.step(ev)
            torch.cuda.synchronize(self.dev)
        self.check_errors("roofline loop")
        return [a.elapsed_time(b) for a, b in evs[:e]], clk.summary()

    def cold_calls(self, n: int = 50):
        """Decode calls after a 2x-L2 buffer write each (pools that fit in L2)."""
        import torch
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=self.dev)
        evs = [_event_pair() for _ in range(n)]
        for ev in evs:
            flush.fill_(1)
            self.step(ev)
        torch.cuda.synchronize(self.dev)
        del flush
        return [a.elapsed_time(b) for a, b in evs]

    def e2e(self, steps: int, world: int = 1, dist=None, max_over=None):
        """The public host-buffer step: inputs from pinned memory, the result back to
        it, copies overlapped with the neighbouring steps' kernels."""
        import torch
        from workloads import TORCH_DTYPES
        cfg = self.cfg
        S, Hq, D = cfg.num_seqs, cfg.num_heads, cfg.head_dim
        outs_h = [torch.empty((S, Hq, D), dtype=TORCH_DTYPES[cfg.dtype], pin_memory=True)
                  for _ in range(2)]
        done = [None, None]

        def e2e_step(k):
            if done[k % 2] is not None:
                done[k % 2].synchronize()          # the caller consumed that result
            done[k % 2] = self.dec.step_host(*self.toks_h[k % self.RING], outs_h[k % 2])

        for k in range(3):
            e2e_step(k)
        torch.cuda.synchronize(self.dev)
        if world > 1:
            dist.barrier()
        e0, e1 = _event_pair()
        e0.record(self.stream)
        for k in range(steps):
            e2e_step(k)
        self.dec.drain_host_io()
        e1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        self.check_errors("e2e")
        e_ms = e0.elapsed_time(e1)
        if max_over is not None:
            e_ms = max_over(e_ms)
        h2d = sum(t.numel() * t.element_size() for t in self.toks_h[0]) + self.dec.staging_bytes
        d2h = S * Hq * D * cfg.elem_bytes
        return e_ms, int(h2d), int(d2h)

    def roofline(self, dec_ms, clk, peak, peak_kind):
        cfg = self.cfg
        avg = statistics.mean(dec_ms)
        achieved = self.dec_bytes / (avg * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                "kernel": ("pa_decode_attention_fp8" if self.cache_fp8 else
                           "pa_decode_attention") + " (partition kernels + log-sum-exp merge)",
                "bytes_per_launch": int(self.dec_bytes), "avg_launch_us": round(avg * 1e3, 2),
                "launches_timed": len(dec_ms),
                "median_launch_us": round(statistics.median(dec_ms) * 1e3, 2),
                "frac_of_nominal_8000": round(achieved / 8000.0, 4),
                "traffic": recorded_traffic(cfg, self.cache_fp8),
                "clocks": clk}
        if clk.get("sm_mhz"):
            # the call in SM clock cycles at the median clock (comparable across clocks)
            roof["avg_launch_kcycles_at_median_clock"] = round(avg * clk["sm_mhz"], 1)
        if self.uniq is not None:
            roof["bytes_note"] = "unique bytes: each shared physical slot counted once"
            roof["logical_bytes_per_launch"] = int(self.logical_dec_bytes)
            roof["logical_achieved"] = round(self.logical_dec_bytes / (avg * 1e-3) / 1e9, 1)
        return roof

    def close(self):
        import torch
        self.dec = None
        self.kd = self.vd = self.out = None
        self.toks_d = self.toks_h = None
        torch.cuda.synchronize(self.dev)
        torch.cuda.empty_cache()


# the other workloads, measured in the same invocation at N=1 (name, fp8 cache, partition)
PER_WORKLOAD = [
    ("13b_fp16", False, None),
    ("gqa_long_bf16", False, None),
    ("gqa_long_bf16", False, 0),
    ("prefix_cow_bf16", False, None),
    ("tiny_fp32", False, None),
    ("7b_bf16", True, None),
    ("13b_fp16", True, None),
    ("gqa_long_bf16", True, None),
]


def per_workload_key(name, fp8, ps) -> str:
    return name + ("+fp8_cache" if fp8 else "") + ("" if ps is None else "@library_partition")


def measure_other(cfg, seed, dev, fp8, peak, peak_kind, seconds: float) -> dict:
    """One entry of ``per_workload``: settle, a timed loop sized by time, the decode
    call's roofline loop, and the host-buffer loop."""
    run = WorkloadRun(cfg, seed, dev, cache_fp8=fp8, host_pool=False)
    try:
        run.run_for(0.3)
        n = run.steps_for(seconds)
        ms, clk, _ = run.timed(n, clock_index=dev.index or 0)
        dec_ms, rclk = run.roofline_loop(seconds, clock_index=dev.index or 0)
        roof = run.roofline(dec_ms, rclk, peak, peak_kind)
        if run.pool_bytes <= L2_BYTES:
            roof["cold_median_launch_us"] = round(statistics.median(run.cold_calls()) * 1e3, 2)
            roof["cold_note"] = "pool smaller than L2: calls after a 2x-L2 buffer write"
        e_ms, h2d, d2h = run.e2e(n)
        S = cfg.num_seqs
        return {
            "value": round(run.step_bytes * n / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "steps": n, "ms_per_step": round(ms / n, 4),
            "seqs_per_s": round(S * n / (ms * 1e-3), 1),
            "partition_size": run.dec.partition_size,
            "kv_cache": ("fp8 e4m3, per-tensor scales %g" % run.kv_scales[0]) if fp8
                        else cfg.dtype,
            "mean_seq_len": round(float(run.lens.mean()), 1), "max_seq_len": int(run.lens.max()),
            "pool": "K/V drawn on the device (same distribution, seeded)",
            "roofline": roof,
            "e2e": {"value": round(run.step_bytes * n / (e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e_ms / n, 4)},
            "gpu_launches": run.launches_per_step * n,
            "clocks": clk,
        }
    finally:
        run.close()


def run_ours(args, cfg):
    import torch
    import torch.distributed as dist

    world, rank, local = replica_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    max_over = lambda v: max_over_ranks(v, world, dev)
    peak, peak_kind = hbm_peak()

    seed = replica_seed(args.seed, rank)
    run = WorkloadRun(cfg, seed, dev, cache_fp8=args.cache_fp8, host_pool=True)
    S = cfg.num_seqs
    # clocks up and the pipeline steady before the warm-up steps
    t_settle = time.perf_counter()
    settle_steps = run.run_for(args.settle_ms * 1e-3)
    settle_ms = (time.perf_counter() - t_settle) * 1e3
    warm_cow = 0
    for _ in range(args.warmup):
        warm_cow += run.step()["num_cow"]
    torch.cuda.synchronize(dev)
    run.check_errors("warm-up")

    # ---- the timed region: exactly --steps steps --------------------------------
    elapsed_ms, clk, cows = run.timed(args.steps, world, dist, local)
    retried = False
    if clocks_rejected(clk):       # measured again once, as the timing rules ask
        retried = True
        elapsed_ms, clk, cows = run.timed(args.steps, world, dist, local)
    elapsed_ms = max_over(elapsed_ms)
    job_step_bytes = sum_over_ranks(run.step_bytes, world, dev)
    value = job_throughput(job_step_bytes, args.steps, elapsed_ms)
    seqs_per_s = S * world * args.steps / (elapsed_ms * 1e-3)

    # ---- the decode call's own duration: its own loop of >= --roofline-ms ---------
    dec_ms, rclk = run.roofline_loop(args.roofline_ms * 1e-3, local)
    roof = run.roofline(dec_ms, rclk, peak, peak_kind)
    if run.pool_bytes <= L2_BYTES and rank == 0:
        roof["cold_median_launch_us"] = round(statistics.median(run.cold_calls()) * 1e3, 2)
        roof["cold_note"] = "pool smaller than L2: calls after a 2x-L2 buffer write"

    # ---- end to end through the public API with host buffers ----------------------
    e2e = None
    if not args.no_e2e:
        e_ms, h2d, d2h = run.e2e(args.steps, world, dist, max_over)
        E = job_throughput(job_step_bytes, args.steps, e_ms)
        e2e = {"value": round(E, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms / args.steps, 4),
               "seqs_per_s": round(S * world * args.steps / (e_ms * 1e-3), 1)}

    config = workload_config(cfg, run.lens, world, args.cache_fp8)
    run_info = {
        "partition_size": run.dec.partition_size,
        "workspace_bytes": int(run.dec.workspace_bytes),
        "prefix_group_chunks": int(run.meta0.get("num_chunks", 0)),
        "pool": pool_summary(run.dec.alloc.stats()),
        "cow_pairs_in_warmup": warm_cow, "cow_pairs_in_timed_steps": cows,
        "settle_ms": round(settle_ms, 1), "settle_steps": settle_steps,
        "timed_region_retried_for_clocks": retried,
        "kv_cache": ("fp8 e4m3, per-tensor scales %g" % run.kv_scales[0])
                    if args.cache_fp8 else cfg.dtype,
    }
    launches = run.launches_per_step * args.steps
    inp = run.inp
    run.close()

    # ---- the other workloads (N=1, default run only) --------------------------------
    per = None
    if world == 1 and not args.no_per_workload and args.default_shape:
        per = {}
        for name, fp8, ps in PER_WORKLOAD:
            from workloads import CONFIGS
            c = CONFIGS[name] if ps is None else CONFIGS[name].with_(partition_size=ps)
            per[per_workload_key(name, fp8, ps)] = measure_other(
                c, seed, dev, fp8, peak, peak_kind, args.per_workload_ms * 1e-3)

    # ---- CPU baseline: the oracle on the host cores, rank 0 at N=1 only ------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        timer = OracleTimer(cfg, inp)
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

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(elapsed_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "seqs_per_s": round(seqs_per_s, 1),
            "config": config,
            "run_info": run_info,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
            "per_workload": per,
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


def recorded_traffic(cfg, cache_fp8: bool = False):
    """DRAM bytes per decode call from the committed ncu capture of this workload,
    if it was taken on the current kernel sources (else None)."""
    path = os.path.join(HERE, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(cfg.name + ("+fp8_cache" if cache_fp8 else ""))
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
    args.default_shape = (args.workload in (None, HEADLINE) and args.seqs is None
                          and args.pool_blocks is None and args.block_size is None
                          and args.partition_size is None and not args.cache_fp8)
    if args.impl == "reference":
        run_reference(args, cfg)
    elif args.measure == "swap":
        run_swap(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
