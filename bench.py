"""Benchmark of the paged decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload targets|7b|gqa70b|prefix_cow|long|tiny|prefill]

One step = the whole hot path over one batch: copy-on-write block copies (if
the workload has any), the slot write of the step's new tokens, and decode
attention.  By default (``--workload targets``) the four large decode
workloads are timed one after the other, each for K steps after W warm-up
steps, and one JSON line is printed whose headline is the largest of them,
``long`` (8 sequences x 32768 tokens, 32 query / 8 KV heads, head size 128,
bf16, 16384-block shuffled pool, partitions of 512 tokens merged by
log-sum-exp; 1.07 GB of K/V per step); the records of ``7b``, ``gqa70b`` and
``prefix_cow`` (plain and prefix-deduplicated) sit under ``workloads``.

Metric: effective KV HBM bandwidth in GB/s = algorithmic bytes of the step
(K and V of every live token, q read, out written, plus the slot write's and
copies' bytes) / device time; also seq-steps/s and % of the measured HBM
peak.  Before every timed step the L2 is flushed and left clean (untimed): a
512 MiB buffer is written, then a second 512 MiB buffer is read, so the
written lines are evicted (and written back to HBM) before the step starts
rather than during it.

Under torchrun (N > 1) every rank runs its own independent batch (the path
shards by sequence with no collective): weak scaling, time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention: effective KV HBM GB/s (% of B200 peak); seq-steps/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
SPEC_HBM_GBS = 8000.0     # B200 data-sheet HBM3e bandwidth (context beside the measured peak)
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "decode_traffic.json")
KERNEL_SOURCES = ("paged_kv_cache_456_b200/csrc/decode_kernel.cuh",
                  "paged_kv_cache_456_b200/csrc/decode_bf16.cu",
                  "paged_kv_cache_456_b200/csrc/decode_f32.cu",
                  "paged_kv_cache_456_b200/csrc/ptx.cuh",
                  "paged_kv_cache_456_b200/csrc/pa_internal.h")
# the deduplicated call adds the shared-prefix pass (on the tcgen05 kernel,
# which also runs bf16 prefill)
DEDUP_SOURCES = ("paged_kv_cache_456_b200/csrc/shared_prefix.cu",
                 "paged_kv_cache_456_b200/csrc/tc_attention.cu",
                 "paged_kv_cache_456_b200/csrc/tc.cuh")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description="paged decode benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="targets",
                    help="'targets' (the four large decode workloads, long as the headline) "
                         "or one workload name")
    ap.add_argument("--partition-size", type=int, default=None)
    ap.add_argument("--append", choices=("fused", "separate"), default="fused",
                    help="slot write of the new tokens fused into decode (one call) or as its "
                         "own launch before it")
    ap.add_argument("--dedup", action="store_true",
                    help="prefix-deduplicated decode (pa_decode_shared_prefix): groups of "
                         "sequences sharing leading blocks read them once")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seed", type=int, default=None)
    ap.add_argument("--num-blocks", type=int, default=None,
                    help="pool size override (same lengths; for small profiler captures)")
    return ap.parse_args(argv)


def measured_peaks(key: str = "hbm_gbs"):
    fallback = {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS}[key]
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d[key]), "measured"
    except (OSError, KeyError, ValueError):
        return fallback, "fallback"


def kernel_source_hash(dedup: bool = False) -> str:
    """Hash of the decode kernel's code (with the tensor-core kernels of the
    shared-prefix pass and of prefill: of both) with comments and blank space
    removed, so that a comment edit does not orphan recorded counters."""
    import re
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES + (DEDUP_SOURCES if dedup else ()):
        with open(os.path.join(ROOT, rel)) as f:
            code = f.read()
        code = re.sub(r"/\*.*?\*/", " ", code, flags=re.S)
        code = re.sub(r"//[^\n]*", " ", code)
        h.update(" ".join(code.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current kernel source; else None."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    entry = d.get(workload)
    tc = workload.endswith("+dedup") or workload == "prefill"
    if not entry or entry.get("kernel_source_hash") != kernel_source_hash(tc):
        return None
    return entry.get("dram_bytes_per_launch")


def step_bytes(w, fused: bool = False) -> int:
    """Algorithmic bytes of one step.  Fused, the new rows are read once (as
    decode's live tokens) and only their two cache writes add."""
    append = w.append_bytes() if fused else w.reshape_bytes()
    return w.decode_bytes() + append + w.copy_bytes()


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4}

    def __init__(self, device_index: int, period_s: float = 0.0002):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: report no clocks rather than fail
            self.max_mhz = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                mask = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.ok:
            self._t.join(timeout=2)

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# the CPU oracle as baseline / reference arm
# ---------------------------------------------------------------------------
def sub_workload(w, k: int):
    """The first k sequences of a workload (same pool, same copy pairs)."""
    import dataclasses
    if w.query_start is not None:
        r = int(w.query_start[k])
        return dataclasses.replace(
            w, context_lens=w.context_lens[:k], tables_compact=w.tables_compact[:k], q=w.q[:r],
            query_start=w.query_start[:k + 1], new_key=w.new_key[:r], new_value=w.new_value[:r],
            slot_mapping_compact=w.slot_mapping_compact[:r])
    return dataclasses.replace(
        w, context_lens=w.context_lens[:k], tables_compact=w.tables_compact[:k], q=w.q[:k],
        new_key=None if w.new_key is None else w.new_key[:k],
        new_value=None if w.new_value is None else w.new_value[:k],
        slot_mapping_compact=None if w.slot_mapping_compact is None else w.slot_mapping_compact[:k])


def oracle_sample(w, budget_s: float, repeat: bool = False, fused: bool = True):
    """Time the oracle's whole step on the first k sequences of the workload,
    k grown until one pass takes about budget_s (or all sequences are in);
    with ``repeat``, whole passes are then repeated until budget_s is spent.
    Bytes follow the GPU arm's accounting (``fused``: see step_bytes).
    Returns (GB/s, seconds per pass, k, bytes per pass, threads)."""
    import oracle

    k = 1
    while True:
        ws = sub_workload(w, k)
        t0 = time.perf_counter()
        oracle.workload_step(ws)
        dt = time.perf_counter() - t0
        if dt >= budget_s or k >= w.num_seqs:
            break
        k = min(w.num_seqs, max(k + 1, int(k * min(8.0, budget_s / max(dt, 1e-3)))))
    if repeat and dt < budget_s:
        passes, t0 = 0, time.perf_counter()
        while passes == 0 or time.perf_counter() - t0 < budget_s:
            oracle.workload_step(ws)
            passes += 1
        dt = (time.perf_counter() - t0) / passes
    nbytes = step_bytes(ws, fused)
    return nbytes / dt / 1e9, dt, k, nbytes, oracle.num_threads()


# the four large decode workloads, the headline (the largest) first; the
# default run adds the chunked-prefill workload (tensor-core attention of
# many query rows) as one more record
TARGETS = ("long", "7b", "gqa70b", "prefix_cow")
EXTRAS = ("prefill",)


def workload_names(args):
    return TARGETS + EXTRAS if args.workload == "targets" else (args.workload,)


def run_reference(args, rank: int, world: int):
    """The oracle on the headline workload (a bounded sample of it per step),
    with this arm's metric, unit and config."""
    if rank != 0:
        return
    from paged_kv_cache_456_b200.workloads import build_workload
    import oracle
    name = workload_names(args)[0]
    w = build_workload(name, seed=args.seed, num_blocks=args.num_blocks)
    steps, warm = args.steps, args.warmup
    per_step_budget = max(0.05, 150.0 / max(1, steps + warm))
    _, dt, k, nbytes, threads = oracle_sample(w, per_step_budget,
                                              fused=args.append == "fused")
    ws = sub_workload(w, k)
    for _ in range(warm):
        oracle.workload_step(ws)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle.workload_step(ws)
    elapsed = time.perf_counter() - t0
    value = nbytes * steps / elapsed / 1e9
    sample = (f"first {k} of {w.num_seqs} sequences of the {w.name} workload per step "
              f"({int(w.context_lens[:k].sum())} tokens)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": steps, "warmup": warm,
        "ms_per_step": round(elapsed / steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "seq_steps_per_s": round(k * steps / elapsed, 3),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    if getattr(args, "dedup", False):
        # (the same attention: the oracle reads every sequence's blocks itself)
        line["config"]["dedup"] = True
    print(json.dumps(line), flush=True)


def max_over_ranks(values, device, world: int):
    """Element-wise maximum of ``values`` over all ranks (one all_reduce;
    the identity on a single process)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def workload_config(w):
    return {"workload": w.name, "num_seqs": w.num_seqs, "num_q_heads": w.num_q_heads,
            "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
            "num_blocks": w.num_blocks, "kv_dtype": w.dtype,
            "context_tokens": int(w.context_lens.sum()),
            "max_context_len": int(w.max_context_len),
            "partition_size": int(w.partition_size),
            "l2": "flushed before every timed step: 512 MiB write, then 512 MiB read "
                  "(untimed), leaving L2 cold and clean"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, rank: int, world: int):
    """Time each named workload in turn; rank 0 prints one JSON line: the
    first workload's record as the headline, the others under ``workloads``."""
    import torch

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    names = workload_names(args)
    multi = len(names) > 1
    recs, samples, reasons = {}, [], set()
    max_mhz = None
    for i, name in enumerate(names):
        # (a workload with a shared prefix is also timed deduplicated in the default run)
        modes = [bool(args.dedup)]
        if multi and name == "prefix_cow":
            modes = [False, True]
        for dedup in modes:
            budget = 10.0 if i == 0 else 5.0
            rec, clk = measure(name, args, rank, world, dev, dedup=dedup, cpu_budget=budget)
            samples += clk.samples
            reasons |= clk.reasons
            max_mhz = clk.max_mhz
            if dedup and not modes[0]:
                recs[name]["dedup"] = rec
            else:
                recs[name] = rec
            torch.cuda.empty_cache()
    if rank != 0:
        return
    line = dict(recs[names[0]])
    if multi:
        line["workloads"] = {n: recs[n] for n in names[1:]}
        # clocks over every workload's timed region
        line["clocks"] = {"sm_mhz": statistics.median(samples) if samples else None,
                          "sm_max_mhz": max_mhz, "reasons": sorted(reasons),
                          "samples": len(samples), "per_workload": {
                              n: recs[n]["clocks"] for n in names}}
        line["gpu_launches"] = sum(recs[n]["gpu_launches"] +
                                   recs[n].get("dedup", {}).get("gpu_launches", 0) for n in names)
        line["gpu_launches_headline"] = recs[names[0]]["gpu_launches"]
        line["target"] = {
            "rule": "roofline.frac >= 0.70 of the measured HBM copy peak on the four large "
                    "decode workloads (prefix_cow: by the logical bytes the metric names)",
            "frac": {n: recs[n]["roofline"]["frac"] for n in names if n in TARGETS}}
    print(json.dumps(line), flush=True)


def measure(name, args, rank: int, world: int, dev, dedup: bool = False, cpu_budget: float = 10.0):
    """One workload: W warm-up and K timed steps (L2 flushed before each),
    the end-to-end figure, and on rank 0 at N = 1 the oracle's baseline.
    Returns (record, clock sampler)."""
    import torch
    import torch.distributed as dist
    from paged_kv_cache_456_b200 import ops
    from paged_kv_cache_456_b200.workloads import build_workload, upload

    # rank 0 runs the named workload's own seed; other ranks get independent batches
    seed = args.seed if rank == 0 else (args.seed or 0) + 1000 * rank
    w = build_workload(name, seed=seed, num_blocks=args.num_blocks)
    if args.partition_size is not None:
        w.partition_size = args.partition_size
    t = upload(w, dev)
    stream = torch.cuda.current_stream(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    tdt = t["q"].dtype
    ps = w.partition_size
    prefill = "query_start" in t     # several query tokens per sequence
    rows = t["q"].shape[0]            # query rows: one per sequence in decode
    dedup = dedup and not prefill
    plan = None
    if dedup:
        # the groups come from the host planner once (they change only when
        # requests fork or finish); their arrays are step inputs like the tables
        plan = ops.shared_prefix_plan(w.block_tables, w.context_lens)
        t["group_seqs"], t["group_start"], t["group_blocks"] = plan.to(dev)
    if prefill:
        ws = ops.make_prefill_workspace(w.num_seqs, rows, w.num_q_heads, w.num_kv_heads,
                                        w.head_dim, w.max_context_len, ps, tdt, device=dev)
    elif dedup:
        ws = ops.make_shared_prefix_workspace(w.num_seqs, plan.num_listed, w.num_q_heads,
                                              w.num_kv_heads, w.head_dim, w.max_blocks_per_seq,
                                              w.max_context_len, ps, tdt, device=dev)
    else:
        ws = ops.make_workspace(rows, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                w.max_context_len, ps, tdt, device=dev)
    if prefill:
        cfg = ops.prefill_launch_config(w.num_seqs, rows, w.num_q_heads, w.num_kv_heads,
                                        w.head_dim, w.max_context_len, ps, tdt)
    else:
        cfg = ops.launch_config(rows, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                w.max_context_len, ps, tdt)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    evict = torch.ones(128 << 20, dtype=torch.int32, device=dev)   # 512 MiB, read only

    def flush_l2(s=None):
        with torch.cuda.stream(s or stream):
            flush.fill_(1)
            evict.sum()     # the read pushes the dirty lines of the write out of L2
    fused = "key" in t and args.append == "fused" and not prefill
    # decode is two kernels (the attention pass and the merge pass behind it);
    # so is bf16 prefill (the plan kernel and the tensor-core attention kernel)
    launches_per_step = 2 + ("key" in t and not fused) + ("block_mapping" in t)
    if dedup and plan.num_groups:
        launches_per_step += 3      # the shared-prefix pass: its plan kernel, the pass, the fold

    def step(ev_mid=None):
        if "block_mapping" in t:
            ops.copy_blocks(t["k_cache"], t["v_cache"], t["block_mapping"], err_flag=err)
        if "key" in t and not fused:
            ops.reshape_and_cache(t["key"], t["value"], t["k_cache"], t["v_cache"],
                                  t["slot_mapping"], err_flag=err)
        if ev_mid is not None:
            ev_mid.record(stream)
        if prefill:
            ops.prefill(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                        t["context_lens"], t["query_start"], scale=w.scale,
                        max_context_len=w.max_context_len, workspace=ws, partition_size=ps,
                        err_flag=err)
        elif dedup:
            shared_prefix_call(t, t, w, ws, ps, err, fused, stream)
        elif fused:
            ops.decode_append(t["out"], t["q"], t["key_seq"], t["value_seq"], t["k_cache"],
                              t["v_cache"], t["block_tables"], t["context_lens"], scale=w.scale,
                              max_context_len=w.max_context_len, workspace=ws,
                              partition_size=ps, err_flag=err)
        else:
            ops.decode(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                       t["context_lens"], scale=w.scale, max_context_len=w.max_context_len,
                       workspace=ws, partition_size=ps, err_flag=err)

    for _ in range(max(3, args.warmup)):
        flush_l2()
        step()
    torch.cuda.synchronize(dev)

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        for i in range(K):
            flush_l2()                      # evict the previous step from L2 (untimed)
            ev[i][0].record(stream)
            step(ev[i][1])
            ev[i][2].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    step_ms = [a.elapsed_time(c) for a, b, c in ev]
    dec_ms = [b.elapsed_time(c) for a, b, c in ev]
    total_ms = sum(step_ms)
    timed_err = int(err.item())

    # end to end through the public API: pinned host inputs in, output back
    e2e = end_to_end(w, t, ws, ps, dev, stream, K, args.warmup, fused, dedup, flush_l2)

    # every rank reaches this one collective, errors or not; then all agree
    max_ms, e2e["ms"], e2e["warm_ms"], bad = max_over_ranks(
        [total_ms, e2e["ms"], e2e["warm_ms"], float(timed_err | e2e["err"])], dev, world)
    if bad:
        raise RuntimeError(f"device error flag {int(bad)} during the benchmark (some rank)")

    nbytes = step_bytes(w, fused)
    peak, peak_kind = measured_peaks()
    value = world * nbytes * K / (max_ms * 1e-3) / 1e9
    dec_avg = statistics.mean(dec_ms)
    # the kernel's bytes: the workload's logical bytes (what the metric names);
    # deduplicated, each shared block once (what the call must move)
    dec_bytes = ((w.unique_decode_bytes() if dedup else w.decode_bytes()) +
                 (w.append_bytes() if fused else 0))
    achieved = dec_bytes / (dec_avg * 1e-3) / 1e9
    traffic = recorded_traffic(w.name + ("+dedup" if dedup else ""))
    rec = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(max_ms / K, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if
        w.dtype == "bf16" else "f32", "data": "synthetic", "config": workload_config(w),
        "pct_of_peak": round(100 * value / world / peak, 2),
        "pct_of_spec_8tbs": round(100 * value / world / SPEC_HBM_GBS, 2),
        "seq_steps_per_s": round(world * w.num_seqs * K / (max_ms * 1e-3), 1),
        "append": ("fused into decode" if fused else "separate launch") if "key" in t else "none",
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic, "kernel": "paged_decode_kernel + merge pass",
                     "peak_source": f"{peak_kind} hbm_gbs (burst copy)",
                     "algorithmic_bytes_per_launch": dec_bytes,
                     "launch_ms_mean": round(dec_avg, 5),
                     "launch_ms_median": round(statistics.median(dec_ms), 5),
                     "frac_of_spec_8tbs": round(achieved / SPEC_HBM_GBS, 4)},
        "e2e": {"value": round(world * nbytes * K / (e2e["ms"] * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "ms_per_step": round(e2e["ms"] / K, 5),
                "how": "each step from cold, clean L2 (flushed, untimed): inputs copied from "
                       "pinned host memory, kernels, output copied back, in order on one stream",
                "pipelined_warm": {
                    "value": round(world * nbytes * K / (e2e["warm_ms"] * 1e-3) / 1e9, 2),
                    "ms_per_step": round(e2e["warm_ms"] / K, 5),
                    "how": "steps back to back, no flush, copies double-buffered on two copy "
                           "streams overlapping the previous step's kernels"}},
        "gpu_launches": launches_per_step * K,
        "launch": cfg,
        "clocks": clocks.summary(),
    }
    if traffic:
        rec["roofline"]["traffic_over_algorithmic"] = round(traffic / dec_bytes, 4)
    if w.name == "prefix_cow" and not dedup:
        # shared blocks are read from HBM about once and then from L2: the
        # logical rate is L2 -> SM bandwidth; the HBM view divides the unique bytes
        ub = w.unique_decode_bytes() + (w.append_bytes() if fused else 0)
        rec["roofline"]["unique_bytes_per_launch"] = ub
        rec["roofline"]["hbm_frac_by_unique_bytes"] = round(ub / (dec_avg * 1e-3) / 1e9 / peak, 4)
    if dedup:
        rec["config"]["dedup"] = True
        rec["roofline"]["kernel"] = ("shared-prefix pass (tc_attention_kernel, tcgen05, its "
                                     "plan kernel and tc_fold_kernel) + paged_decode_kernel + "
                                     "merge pass (the deduplicated decode call)")
        rec["roofline"]["logical_bytes_per_launch"] = w.decode_bytes()
        rec["dedup"] = {"groups": plan.num_groups, "listed": plan.num_listed,
                        "shared_blocks": [int(b) for b in plan.blocks[:8]],
                        "logical_kv_bytes": w.decode_bytes(),
                        "unique_kv_bytes": w.unique_decode_bytes()}
    if prefill:
        # many query columns share each K/V tile: a dense contraction, set
        # against the tensor roofline by its attention FLOPs
        fl = w.attention_flops()
        tpk, tkind = measured_peaks("bf16_tflops")
        tf = fl / (dec_avg * 1e-3) / 1e12
        rec["roofline"].update({"kernel": "tc_attention_kernel (tcgen05) + its plan kernel"
                                if w.dtype == "bf16" else "paged_decode_kernel + merge pass",
                                "bound": "tensor", "achieved": round(tf, 2), "peak": tpk,
                                "unit": "TFLOP/s", "frac": round(tf / tpk, 4),
                                "peak_source": f"{tkind} bf16_tflops (burst cuBLAS GEMM)",
                                "algorithmic_flops_per_launch": fl,
                                "hbm_view_gbs": round(achieved, 2)})
        rec["query_rows"] = rows
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not dedup:
        gbs, dt, k, nb, threads = oracle_sample(w, budget_s=cpu_budget, repeat=True, fused=fused)
        rec["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads,
                               "kind": "oracle",
                               "sample": f"first {k} of {w.num_seqs} sequences of the {w.name} "
                                         f"step ({dt:.2f} s per pass, repeated for "
                                         f"{cpu_budget:.0f} s)"}
    del t, ws, flush, evict
    return rec, clocks


def shared_prefix_call(d, t, w, ws, ps, err, fused, stream):
    """The deduplicated decode call: inputs from d (step inputs), cache from t."""
    from paged_kv_cache_456_b200 import ops
    ops.decode_shared_prefix(t["out"] if d is t else d["_out"], d["q"], t["k_cache"],
                             t["v_cache"], d["block_tables"], d["context_lens"],
                             (d["group_seqs"], d["group_start"], d["group_blocks"]),
                             scale=w.scale, max_context_len=w.max_context_len, workspace=ws,
                             key=d["key_seq"] if fused else None,
                             value=d["value_seq"] if fused else None, partition_size=ps,
                             err_flag=err, stream=stream)


def end_to_end(w, t, ws, ps, dev, stream, K, warmup, fused, dedup, flush_l2):
    """The step through the public API with the step's inputs in pinned host
    memory: every step copies its inputs (q, the new K/V or slot ids, block
    tables, lengths, copy pairs) host to device in one transfer, runs the
    kernels, and copies the output back.  The KV pool itself is resident
    device state and is not copied.

    Two figures: ``ms`` times each step alone from a cold, clean L2 (flushed
    as for the device-timed steps, outside the events), copies and kernels
    in order on one stream -- the figure comparable with the device-timed
    step; ``warm_ms`` runs the steps back to back as a serving loop would,
    the copies on two copy streams, double-buffered, so that step i's
    transfers overlap step i-1's kernels (and L2 stays warm)."""
    import torch
    from paged_kv_cache_456_b200 import ops

    step_inputs = ("q", "key_seq", "value_seq") if fused else ("q", "key", "value", "slot_mapping")
    names = [n for n in step_inputs + ("block_tables", "context_lens", "block_mapping",
                                       "query_start", "group_seqs", "group_start",
                                       "group_blocks") if n in t]
    # one pinned staging buffer holding every input, 256-byte aligned pieces
    offs, size = {}, 0
    for n in names:
        offs[n] = size
        size += -(-(t[n].numel() * t[n].element_size()) // 256) * 256
    h_in = torch.empty(size, dtype=torch.uint8).pin_memory()
    for n in names:
        nb = t[n].numel() * t[n].element_size()
        h_in[offs[n]:offs[n] + nb].copy_(t[n].cpu().contiguous().view(-1).view(torch.uint8))
    d_in = [torch.empty(size, dtype=torch.uint8, device=dev) for _ in range(2)]

    def views(buf):
        return {n: buf[offs[n]:offs[n] + t[n].numel() * t[n].element_size()].view(t[n].dtype)
                .view(t[n].shape) for n in names}

    dv = [views(d_in[0]), views(d_in[1])]
    out = [torch.empty_like(t["out"]) for _ in range(2)]
    h_out = [torch.empty(t["out"].shape, dtype=t["out"].dtype).pin_memory() for _ in range(2)]
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    h2d, d2h = size, h_out[0].numel() * h_out[0].element_size()
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, computed, out_read = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def kernels(d, o, s):
        if "block_mapping" in d:
            ops.copy_blocks(t["k_cache"], t["v_cache"], d["block_mapping"], err_flag=err, stream=s)
        if "key" in d:
            ops.reshape_and_cache(d["key"], d["value"], t["k_cache"], t["v_cache"],
                                  d["slot_mapping"], err_flag=err, stream=s)
        if "query_start" in d:
            ops.prefill(o, d["q"], t["k_cache"], t["v_cache"], d["block_tables"],
                        d["context_lens"], d["query_start"], scale=w.scale,
                        max_context_len=w.max_context_len, workspace=ws, partition_size=ps,
                        err_flag=err, stream=s)
        elif dedup:
            shared_prefix_call(dict(d, _out=o), t, w, ws, ps, err, fused, s)
        elif fused:
            ops.decode_append(o, d["q"], d["key_seq"], d["value_seq"], t["k_cache"],
                              t["v_cache"], d["block_tables"], d["context_lens"], scale=w.scale,
                              max_context_len=w.max_context_len, workspace=ws,
                              partition_size=ps, err_flag=err, stream=s)
        else:
            ops.decode(o, d["q"], t["k_cache"], t["v_cache"], d["block_tables"],
                       d["context_lens"], scale=w.scale, max_context_len=w.max_context_len,
                       workspace=ws, partition_size=ps, err_flag=err, stream=s)

    def one(i):
        b = i % 2
        d = dv[b]
        up.wait_event(computed[b])           # buffer b's previous step has read its inputs
        with torch.cuda.stream(up):
            d_in[b].copy_(h_in, non_blocking=True)
            in_ready[b].record(up)
        stream.wait_event(in_ready[b])
        stream.wait_event(out_read[b])       # out[b]'s previous result has left the device
        kernels(d, out[b], stream)
        computed[b].record(stream)
        down.wait_event(computed[b])
        with torch.cuda.stream(down):
            h_out[b].copy_(out[b], non_blocking=True)
            out_read[b].record(down)

    # -- cold, serial: each step alone, L2 flushed before it (untimed) ----------
    for i in range(max(3, warmup)):
        flush_l2()
        d_in[0].copy_(h_in, non_blocking=True)
        kernels(dv[0], out[0], stream)
        h_out[0].copy_(out[0], non_blocking=True)
    torch.cuda.synchronize(dev)
    marks = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(K)]
    for i in range(K):
        flush_l2()
        marks[i][0].record(stream)
        d_in[0].copy_(h_in, non_blocking=True)
        kernels(dv[0], out[0], stream)
        h_out[0].copy_(out[0], non_blocking=True)
        marks[i][1].record(stream)
    torch.cuda.synchronize(dev)
    cold_ms = sum(a.elapsed_time(z) for a, z in marks)
    bad = int(err.item())
    if not bad and not torch.equal(h_out[0].view(torch.uint8), t["out"].cpu().view(torch.uint8)):
        bad = 1 << 30   # the end-to-end output differs from the device-timed run's

    # -- warm, pipelined: back to back, copies overlapping the previous step ---
    for i in range(max(3, warmup)):
        one(i)
    torch.cuda.synchronize(dev)
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(K):
        one(i)
    stream.wait_event(out_read[(K - 1) % 2])  # the last result is on the host
    z.record(stream)
    torch.cuda.synchronize(dev)
    bad |= int(err.item())
    if not bad and not torch.equal(h_out[(K - 1) % 2].view(torch.uint8),
                                   t["out"].cpu().view(torch.uint8)):
        bad = 1 << 30
    return {"ms": cold_ms, "warm_ms": a.elapsed_time(z), "h2d": h2d, "d2h": d2h, "err": bad}


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
