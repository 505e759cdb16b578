#!/usr/bin/env python
"""Benchmark: paged single-token decode attention on B200.

One step = one full pass of the hot path over one decode batch: one launch of
the partition kernel with the split reduce folded in (preceded, for batches of
heavy units, by the one-CTA pass that orders the units longest first).  Default workload: the
Qwen3-14B-shaped decode batch (B=64, Hq/Hkv=40/8, D=128, block_size 16, every
seq_len 8192, synthetic bf16 ~N(0,1), tables over a 32768-block pool, 16 splits of
512 tokens, LSE on).  --workload picks another named one.

Prints one JSON line (rank 0).  `value` is achieved algorithmic HBM GB/s of the
whole step: all ranks' bytes per step / the max over ranks of the MEDIAN device
time of a step (seven-sample upper-middle statistics in the pages' CLI; the
median here); the mean, min and max ride beside it.  Timing: W warm-up steps,
then K timed steps, each bracketed by CUDA events on the launching stream, with
an L2 flush between steps outside the events (a 256 MiB write, then a 256 MiB
read so that the written lines are evicted too: every timed launch starts from a
cold L2 holding no dirty data); barrier + synchronize around the timed region.
At N=1 the other named workloads (and every workload on its E4M3 cache) are
then timed the same way, each with its own events, into `workloads`.

--impl reference times the CPU oracle (the reference arm of this path) on the
host cores instead; it never touches the GPU.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--workload", default="qwen14b")
    ap.add_argument("--num-splits", type=int, default=None, help="override the workload's partition count")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-baseline time budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (short profiling runs)")
    ap.add_argument("--batch", type=int, default=None,
                    help="first B sequences of the workload (reduced profiling cases); default: the full batch")
    ap.add_argument("--compact-pool", action="store_true",
                    help="block pool = exactly the blocks the batch uses, no page shared (llama8b: no-alias variant)")
    ap.add_argument("--window", type=int, default=0,
                    help="sliding window: each sequence attends to its last W tokens (pad_decode_ex)")
    ap.add_argument("--sinks", action="store_true", help="per-head attention sink logits (pad_decode_ex)")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay of the end-to-end step")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip timing the other named workloads (the `workloads` table)")
    ap.add_argument("--side-steps", type=int, default=60, help="timed steps per workload of the `workloads` table")
    ap.add_argument("--kv-dtype", default="bf16", choices=["bf16", "e4m3"],
                    help="KV cache element type (e4m3: OCP FP8 E4M3 codes with per-tensor scales)")
    ap.add_argument("--entry", default="default", choices=["default", "tcgen05"],
                    help="tcgen05: every leg calls pad_decode_tcgen05, the tensor-memory kernel (bf16 cache, "
                         "head_dim 128, 17-32 query heads per KV head; no window, sinks or E4M3)")
    args = ap.parse_args()
    if args.entry == "tcgen05" and (args.kv_dtype != "bf16" or args.window or args.sinks):
        ap.error("--entry tcgen05 takes a bf16 cache without --window or --sinks")
    check_gpus(args.gpus, int(os.environ.get("WORLD_SIZE", "1")), ap.error)
    return args


def check_gpus(n, world, error):
    """--gpus N is one rank per GPU: N > 1 needs the N ranks a launcher
    (torch.distributed.run) starts, so a single process never reports n_gpus 1
    for a request of N."""
    if n < 1:
        error(f"--gpus must be >= 1 (got {n})")
    if n != world:
        error(f"--gpus {n} but WORLD_SIZE is {world}: launch one rank per GPU, e.g. "
              f"python -m torch.distributed.run --nproc-per-node {n} bench.py --gpus {n}")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload_config(w, args):
    """The workload both arms run (the same keys in the GPU line and the
    reference line): its shape, lengths, inputs and the options asked for.  The
    GPU arm's launch plan and timing method ride beside it, not in it."""
    cfg = {"workload": w.name, "batch": w.B, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.D,
           "block_size": w.block_size, "max_blocks_per_seq": w.max_blocks_per_seq,
           "kv_tokens": w.kv_tokens(args.window), "seq_len_min": int(w.seq_lens.min()),
           "seq_len_max": int(w.seq_lens.max()), "recipe": w.recipe, "lse": w.want_lse, "seed": w.seed,
           "pool_blocks": w.num_blocks - 1, "num_splits_requested": w.num_splits}
    if args.window:
        cfg["window"] = args.window
    if args.sinks:
        cfg["sinks"] = "one N(0,1) logit per query head"
    if args.kv_dtype == "e4m3":
        cfg["kv_cache"] = f"e4m3, k_scale {w.k_scale:g}, v_scale {w.v_scale:g}"
    return cfg


def plan_summary(w, plan):
    return {"num_splits": plan["num_splits"], "partition_tokens": plan["partition_tokens"],
            "heads_per_tile": plan["heads_per_tile"], "head_tiles": plan["head_tiles"], "ctas": plan["ctas"],
            "warps_per_cta": plan["warps_per_cta"], "ctas_per_sm": plan["ctas_per_sm"], "stages": plan["stages"],
            "stage_tokens": plan["stage_tokens"],
            "launches_per_step": launches_per_step(w, plan)}


def split_scratch_bytes(w, plan, window=0):
    """Bytes of split partials one launch writes and the merge reads back (fp32
    o_s and lse_s of every partition of every sequence with more than one
    non-empty partition): reported beside the algorithmic bytes, not credited."""
    P = plan["partition_tokens"]
    total = 0
    for L in w.seq_lens.tolist():
        lo = max(0, L - window) if window else 0
        ns = (-(-L // P) - lo // P) if L > lo else 0
        if ns > 1:
            total += 2 * ns * w.Hq * (w.D + 1) * 4
    return total


def launches_per_step(w, plan):
    """Kernel launches of one decode call: the partition (or tcgen05) kernel,
    preceded by the one-CTA unit-schedule pass when the plan orders its units --
    visible as a workspace larger than the partials."""
    r = lambda x: -(-x // 256) * 256
    S = plan["num_splits"]
    partials = r(w.B * w.Hq * S * w.D * 4) + r(w.B * w.Hq * S * 4) if S > 1 else 0
    return 2 if plan["workspace_bytes"] > partials else 1


def sink_logits(w, on):
    """The per-head sink logits --sinks runs with (both arms): seeded N(0,1)."""
    return np.random.default_rng(w.seed).standard_normal(w.Hq).astype(np.float32) if on else None


def cpu_baseline(w, budget_s, runs_max=50, prefix=None, window=0, sinks=None):
    """Time the oracle as it stands on this host's cores on a bounded sample,
    plus a one-thread figure (on the whole batch, or on its first sequences
    when that would take more than a few seconds; `prefix(k)` builds that batch)."""
    import oracle
    threads = oracle.default_threads()
    bytes_per = w.algorithmic_bytes(window=window, sinks=sinks is not None)
    times = []
    t_all = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        oracle.decode_workload(w, nthreads=threads, window=window, sinks=sinks)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_all > budget_s or len(times) >= runs_max:
            break
    med = statistics.median(times)
    one = None
    est1 = med * threads  # rough one-thread time of the whole batch
    w1 = w if est1 <= 4.0 or prefix is None else prefix(max(1, int(w.B * 4.0 / est1)))
    t0 = time.perf_counter()
    oracle.decode_workload(w1, nthreads=1, window=window, sinks=sinks)
    t1 = time.perf_counter() - t0
    one = {"value": round(w1.algorithmic_bytes(window=window, sinks=sinks is not None) / t1 / 1e9, 4), "unit": "GB/s",
           "cores": 1,
           "sample": (f"whole {w.name} batch" if w1 is w else f"first {w1.B} of {w.B} {w.name} sequences")
                     + f", one run, {t1 * 1e6:.0f} us"}
    return {"value": round(bytes_per / med / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"whole {w.name} batch, {len(times)} run(s), median {med * 1e6:.0f} us/call "
                      f"(double precision, {threads} threads)",
            "us_per_call": round(med * 1e6, 1), "one_thread": one}


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running (reads only)."""

    def __init__(self, index, period=0.002):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        names = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
                 "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                    get = getattr(self._nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                        self._nv.nvmlDeviceGetCurrentClocksThrottleReasons
                    r = get(self._h)
                    for n, bit in names.items():
                        if r & bit:
                            self.reasons.add(n)
                except Exception:
                    pass
                time.sleep(self.period)

        self._t = threading.Thread(target=run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def traffic_from_profiles(workload, kernel_sha, kernel="partition_kernel"):
    """ncu dram bytes per launch recorded under profiles/, if taken on this kernel source."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    try:
        txt = open(path).read()
    except OSError:
        return None
    vals = dict(line.split(":", 1) for line in txt.splitlines() if line.startswith(("source_sha256:", "dram_bytes_per_launch:")))
    if vals.get("source_sha256", "").strip() != kernel_sha:
        return None
    try:
        return int(vals["dram_bytes_per_launch"].strip())
    except (KeyError, ValueError):
        return None


KERNEL_SOURCES = {
    "partition_kernel": ("pad_partition.cu", "pad_merge.cuh", "pad_device.cuh", "pad_internal.h"),
    "umma_kernel": ("pad_umma.cu", "pad_merge.cuh", "pad_device.cuh", "pad_internal.h"),
}


def kernel_source_sha(kernel="partition_kernel"):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "paged_kv_attention_partition_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def run_reference(args, rank, world):
    import synth
    metric = "decode attention µs/call and achieved HBM GB/s vs B200 peak (1 GPU)"
    if rank != 0:
        return
    w = synth.config(args.workload, batch=args.batch, compact_pool=args.compact_pool, kv_dtype=args.kv_dtype)
    cb = cpu_baseline(w, args.cpu_seconds, prefix=lambda k: synth.config(
        args.workload, batch=k, compact_pool=args.compact_pool, kv_dtype=args.kv_dtype),
        window=args.window, sinks=sink_logits(w, args.sinks))
    us = cb["us_per_call"]
    line = {"impl": "reference", "metric": metric, "value": cb["value"], "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1e3, 4), "us_per_call": us,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded generator, no dataset)", "config": workload_config(w, args),
            "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample", "one_thread")},
            "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def rank_seed(base_seed, rank):
    """Weak scaling: rank r decodes its own batch of the same shape, drawn with
    seed base + 1000 r (rank 0 keeps the named workload's own seed)."""
    return base_seed + 1000 * rank


def max_over_ranks(x, device, world):
    """The largest value of `x` over all ranks (the slowest rank's time)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def max_time_sum_bytes(total_ms, my_bytes, device, world):
    """Whole-job aggregate: (max over ranks of the timed device time, sum over
    ranks of the algorithmic bytes moved).  Every rank must call it."""
    if world == 1:
        return float(total_ms), float(my_bytes)
    import torch
    import torch.distributed as dist
    t_max = max_over_ranks(total_ms, device, world)
    bt = torch.tensor([float(my_bytes)], device=device, dtype=torch.float64)
    dist.all_reduce(bt, op=dist.ReduceOp.SUM)
    return t_max, float(bt.item())


# The `workloads` table: every named workload on both caches, and llama8b's
# no-alias variant (its 4096-block pool is smaller than the pages it needs, so
# some pages are shared; the compact pool gives every page one reader).
SIDE_WORKLOADS = [("tiny", "bf16", False), ("llama8b", "bf16", False), ("llama8b", "bf16", True),
                  ("qwen14b", "bf16", False), ("longctx_d256", "bf16", False), ("ragged_mqa", "bf16", False),
                  ("llama8b", "e4m3", False), ("qwen14b", "e4m3", False), ("longctx_d256", "e4m3", False),
                  ("ragged_mqa", "e4m3", False)]


def time_workload(pad, torch, w, dev, stream, flush_l2, steps, warmup, kv_dtype):
    """Device time of K launches of one workload as the main leg times it (caller
    workspace, L2 flushed between steps outside the events): a dict of the
    median / mean / min / max us per call and the median's GB/s."""
    fp8 = kv_dtype == "e4m3"
    kvt = torch.float8_e4m3fn if fp8 else torch.bfloat16
    q = torch.from_numpy(w.q).view(torch.bfloat16).to(dev)
    k = torch.from_numpy(w.k_cache).view(kvt).to(dev)
    v = torch.from_numpy(w.v_cache).view(kvt).to(dev)
    tables, lens = torch.from_numpy(w.block_tables).to(dev), torch.from_numpy(w.seq_lens).to(dev)
    plan = pad.pad_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks_per_seq,
                               num_splits=w.num_splits, device=dev.index, kv_dtype=kv_dtype)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev) if w.want_lse else None
    ws = torch.empty(plan["workspace_bytes"] // 4 + 64, dtype=torch.float32, device=dev)
    sc = dict(k_scale=w.k_scale, v_scale=w.v_scale) if fp8 else {}
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    with torch.cuda.stream(stream):
        for i in range(-warmup, steps):
            flush_l2(i)
            if i >= 0:
                ev[i][0].record(stream)
            pad.pad_decode_with_workspace(q, k, v, tables, lens, w.scale, w.num_splits, out, lse, ws, stream, **sc)
            if i >= 0:
                ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if pad.pad_check_device_errors(stream):
        raise SystemExit(f"device error word set on {w.name} ({kv_dtype})")
    ms = [a.elapsed_time(b) for a, b in ev]
    med = statistics.median(ms)
    gbs = w.algorithmic_bytes() / (med / 1e3) / 1e9
    return {"us_per_call": round(med * 1e3, 2), "us_mean": round(statistics.mean(ms) * 1e3, 2),
            "us_min_max": [round(min(ms) * 1e3, 2), round(max(ms) * 1e3, 2)], "GB_s": round(gbs, 1),
            "algorithmic_bytes": w.algorithmic_bytes(), "num_splits": plan["num_splits"],
            "partition_tokens": plan["partition_tokens"], "ctas": plan["ctas"], "steps": steps}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist

    import synth
    import paged_kv_attention_partition_b200 as pad

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    # weak scaling: every rank decodes its own batch of the same shape
    base = synth.config(args.workload, batch=args.batch, compact_pool=args.compact_pool, kv_dtype=args.kv_dtype)
    w = synth.config(args.workload, seed=rank_seed(base.seed, rank), batch=args.batch,
                     compact_pool=args.compact_pool, kv_dtype=args.kv_dtype) if rank else base
    splits = w.num_splits if args.num_splits is None else args.num_splits
    plan = pad.pad_decode_plan(w.B, w.Hq, w.Hkv, w.D, w.block_size, w.max_blocks_per_seq, num_splits=splits,
                               device=local, kv_dtype=args.kv_dtype)
    fp8 = args.kv_dtype == "e4m3"
    S = plan["num_splits"]
    tc = args.entry == "tcgen05"
    kernel = "umma_kernel" if tc else "partition_kernel"

    def dev_bf16(a):
        return torch.from_numpy(a).view(torch.bfloat16).to(dev)

    def dev_kv(a):
        return torch.from_numpy(a).view(torch.float8_e4m3fn if fp8 else torch.bfloat16).to(dev)

    q, k, v = dev_bf16(w.q), dev_kv(w.k_cache), dev_kv(w.v_cache)
    tables = torch.from_numpy(w.block_tables).to(dev)
    lens = torch.from_numpy(w.seq_lens).to(dev)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev) if w.want_lse else None
    # caller-owned partials scratch (contents irrelevant)
    ws = torch.empty(plan["workspace_bytes"] // 4 + 64, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_acc = torch.empty((), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)

    def flush_l2(i):
        flush.fill_(float(i))
        torch.sum(flush_rd, 0, out=flush_acc)

    sinks_dev = torch.from_numpy(sink_logits(w, True)).to(dev) if args.sinks else None

    def decode(q_, tables_, lens_, out_, lse_, stream_):
        # the public one-call API, with the decode options when asked for
        if tc:
            return pad.pad_decode_tcgen05(q_, k, v, tables_, lens_, w.scale, num_splits=splits, out=out_, lse=lse_,
                                          stream=stream_)
        return pad.pad_decode(q_, k, v, tables_, lens_, w.scale, num_splits=splits, out=out_, lse=lse_,
                              stream=stream_, window=args.window, sinks=sinks_dev,
                              k_scale=w.k_scale if fp8 else 0.0, v_scale=w.v_scale if fp8 else 0.0)

    def call(stream_):
        return decode(q, tables, lens, out, lse, stream_)

    def step():
        # the whole hot path: one decode launch (partition + fused reduce; after
        # the unit-schedule pass for heavy units), partials in the caller-owned
        # workspace (the tcgen05 entry: library-owned scratch)
        if tc:
            call(stream)
            return
        pad.pad_decode_with_workspace(q, k, v, tables, lens, w.scale, splits, out, lse, ws, stream,
                                      window=args.window, sinks=sinks_dev, k_scale=w.k_scale if fp8 else 0.0,
                                      v_scale=w.v_scale if fp8 else 0.0)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush_l2(1)
            step()
            call(stream)
    stream.synchronize()

    # ---- timed region: exactly K steps, device events around each launch ----
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                flush_l2(i)
                ev = events[i]
                ev[0].record(stream)
                step()
                ev[1].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    step_ms = [e[0].elapsed_time(e[1]) for e in events]
    part_ms = step_ms  # the step is the partition kernel's launch (and the schedule pass, if any)
    alg_bytes = w.algorithmic_bytes(window=args.window, sinks=args.sinks)
    # the median step (max over ranks) sets `value`; the mean is reported beside it
    med_ms, all_bytes = max_time_sum_bytes(statistics.median(step_ms), alg_bytes, dev, world)
    total_ms = max_over_ranks(sum(step_ms), dev, world)
    value = all_bytes / (med_ms / 1e3) / 1e9
    value_mean = all_bytes * args.steps / (total_ms / 1e3) / 1e9

    # ---- end to end through the public one-call API, host buffers -----------
    # Per step: pinned host -> device copy of the step's inputs (q, block table,
    # seq_lens; the KV cache stays resident in HBM as in a decode loop), the call,
    # device -> host copy of out and lse.  The inputs share one pinned staging
    # buffer and one device buffer (each tensor at a 256-byte aligned offset), and
    # out and lse share one device buffer, so a step makes one copy each way.
    def pack(parts):
        offs, total = [], 0
        for t in parts:
            offs.append(total)
            total += (t.numel() * t.element_size() + 255) // 256 * 256
        return offs, total

    def view(buf, off, like):
        return buf[off:off + like.numel() * like.element_size()].view(like.dtype).view(like.shape)

    in_parts = [q, tables, lens]
    in_offs, in_total = pack(in_parts)
    din = torch.empty(in_total, dtype=torch.uint8, device=dev)
    hin = torch.zeros(in_total, dtype=torch.uint8).pin_memory()
    for off, t, a in zip(in_offs, in_parts, (w.q, w.block_tables, w.seq_lens)):
        view(hin, off, t).copy_(torch.from_numpy(a).view(t.dtype))
    qe, te, le = (view(din, off, t) for off, t in zip(in_offs, in_parts))
    out_parts = [out] + ([lse] if lse is not None else [])
    out_offs, out_total = pack(out_parts)
    dout = torch.empty(out_total, dtype=torch.uint8, device=dev)
    hout = torch.empty(out_total, dtype=torch.uint8).pin_memory()
    oute = view(dout, out_offs[0], out)
    lsee = view(dout, out_offs[1], lse) if lse is not None else None
    h2d, d2h = in_total, out_total

    def e2e_step(stream_):
        din.copy_(hin, non_blocking=True)
        decode(qe, te, le, oute, lsee, stream_)
        hout.copy_(dout, non_blocking=True)

    e2e_steps = 0 if args.no_e2e else max(10, args.steps // 2)
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(e2e_steps)]
    with torch.cuda.stream(stream):
        for i in range(-3 if e2e_steps else 0, e2e_steps):
            flush_l2(i)
            if i >= 0:
                e2e_ev[i][0].record(stream)
            e2e_step(stream)
            if i >= 0:
                e2e_ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if e2e_steps and not torch.equal(view(hout, out_offs[0], out), out.cpu()):
        raise SystemExit("the end-to-end step's output differs from the kernel leg's")
    e2e_ms = statistics.median([e[0].elapsed_time(e[1]) for e in e2e_ev]) if e2e_steps else float("nan")
    # every rank takes the same collective steps, e2e leg or not
    e2e_med = max_over_ranks(e2e_ms if e2e_steps else 0.0, dev, world)
    e2e_value = all_bytes / (e2e_med / 1e3) / 1e9 if e2e_steps else float("nan")

    # ---- the same end-to-end step captured once as a CUDA graph and replayed
    # (copies in, the call, copies out): what is left of the host's cost.  The
    # library's scratch for this shape and stream exists already, so capture
    # allocates nothing.
    graph_steps = e2e_steps if not args.no_graph else 0
    graph_ms = 0.0
    if graph_steps:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            e2e_step(stream)
        g_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(graph_steps)]
        with torch.cuda.stream(stream):
            for i in range(-3, graph_steps):
                flush_l2(i)
                if i >= 0:
                    g_ev[i][0].record(stream)
                g.replay()
                if i >= 0:
                    g_ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        graph_ms = statistics.median([e[0].elapsed_time(e[1]) for e in g_ev])
        del g
    graph_med = max_over_ranks(graph_ms if graph_steps else 0.0, dev, world)
    graph_value = all_bytes / (graph_med / 1e3) / 1e9 if graph_steps else float("nan")

    errs = pad.pad_check_device_errors(stream)
    if errs:
        raise SystemExit(f"device error word {errs:#x}")

    if rank == 0:
        peak, peak_kind = measured_peaks()
        # the only kernel of the step writes out/lse itself: its algorithmic bytes
        # are the whole call's
        p_bytes = alg_bytes
        p_ms = statistics.median(part_ms)
        achieved = p_bytes / (p_ms / 1e3) / 1e9
        sha = kernel_source_sha(kernel)
        # the recorded ncu traffic is for the named workload at full size, as
        # captured: no window, no sinks
        traffic = (traffic_from_profiles(w.name + ("_e4m3" if fp8 else ""), sha, kernel)
                   if args.batch is None and not args.compact_pool and not args.window and not args.sinks
                   else None)
        kname = f"{kernel}<{w.D},{plan['heads_per_tile']}>"
        api = "pad_decode_tcgen05" if tc else "pad_decode"
        line = {
            "metric": "decode attention µs/call and achieved HBM GB/s vs B200 peak (1 GPU)",
            "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(med_ms, 5), "us_per_call": round(med_ms * 1e3, 2),
            "timing": "value and us_per_call: median step (max over ranks); mean beside it",
            "value_mean": round(value_mean, 2), "us_per_call_mean": round(total_ms / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16",
            "data": "synthetic (seeded counter-based generator; no dataset)",
            "config": workload_config(w, args),
            "plan": {**plan_summary(w, plan), "api": api},
            "l2": (f"flushed between steps outside the timed events: {L2_FLUSH_BYTES >> 20} MiB write, "
                   f"then {L2_FLUSH_BYTES >> 20} MiB read (cold, clean L2)"),
            "hbm_frac_of_peak": round(value / peak, 4),
            "us_per_call_min_max": [round(min(step_ms) * 1e3, 2), round(max(step_ms) * 1e3, 2)],
            "roofline": {"kernel": kname, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "peak_kind": f"{peak_kind} copy bandwidth", "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "algorithmic_bytes_per_launch": p_bytes, "traffic": traffic, "source_sha": sha,
                         "split_scratch_bytes_per_launch": split_scratch_bytes(w, plan, args.window)},
            "e2e": None if not e2e_steps else {
                "value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "us_per_call": round(e2e_med * 1e3, 2), "api": api},
            "e2e_graph": None if not graph_steps else {
                "value": round(graph_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "us_per_call": round(graph_med * 1e3, 2), "api": api + ", replayed as a CUDA graph"},
            # the decode launch, plus the unit-schedule pass when the plan orders
            # its units (its 4-byte-per-CTA order then follows the partials)
            "gpu_launches": args.steps * launches_per_step(w, plan),
            "clocks": clocks.summary(),
        }
        if world == 1 and not args.no_workloads:
            # every named workload (both caches) as a parity-test case would
            # run it, timed in this process after the main leg
            table = {}
            for name, kvd, compact in SIDE_WORKLOADS:
                sw = synth.config(name, compact_pool=compact, kv_dtype=kvd)
                r = time_workload(pad, torch, sw, dev, stream, flush_l2, args.side_steps, 5, kvd)
                r["frac_of_peak"] = round(r["GB_s"] / peak, 4) if name != "tiny" else None
                table[name + ("_compact" if compact else "") + ("_e4m3" if kvd == "e4m3" else "")] = r
                del sw
                torch.cuda.empty_cache()
            line["workloads"] = {"note": f"median of {args.side_steps} launches each (5 warm-up), L2 flushed "
                                         "between launches, caller workspace; frac_of_peak against the same peak "
                                         "(tiny: launch latency only)", **table}
        if world == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline(w, args.cpu_seconds, prefix=lambda k: synth.config(
                args.workload, batch=k, compact_pool=args.compact_pool, kv_dtype=args.kv_dtype),
                window=args.window, sinks=sink_logits(w, args.sinks))
            line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample", "one_thread")}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
