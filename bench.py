#!/usr/bin/env python
"""Benchmark one decode step of one attention layer: copy-on-write block
copies, KV append and paged decode, on the Llama-2-7B-shaped layer (32 query
heads = 32 KV heads, head_dim 128, fp16, block size 16, batch 64 per GPU,
context lengths uniform in [512, 4096], random block placement).

Prints one JSON line (rank 0). `value` is KV-path throughput in GB/s: the
algorithmic bytes of a step (unique KV bytes read by decode, query, output,
block-table entries and lengths, plus the append's and copies' bytes) over
the device-timed step; `roofline` relates the decode call's own bytes and
time to the measured HBM copy bandwidth; `e2e` repeats the measurement with
the step's inputs copied from pinned host memory and the output read back
inside the timed region; `cpu_baseline` times the float64 CPU oracle on the
host's cores on the same inputs.

L2 is flushed between timed steps, outside the timed events: a 256 MiB
buffer (twice the L2) is written, then another one is read, so every step
reads its KV cache from HBM and starts with clean lines in L2 (a write alone
would leave the step to pay the write-back of the flush's dirty lines). The
line also carries the same measurement without the flush (`unflushed`). At
one GPU the line adds `other_configs`: the 70B-shaped shared-prefix layer,
the 128K-token long context at batch 1 and 4 and the FP8 cache with beam
forks, each timed the same way in the same run, with its decode roofline,
clocks and a check of sampled outputs against the oracle.

Multi-GPU (torchrun): every rank runs its own independent batch of the same
shape (sequences are independent; no data-path collective), so per-GPU work
is fixed ("weak" scaling); the step time is the max over ranks.

`--impl reference` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged-decode KV GB/s and % of B200 HBM peak; decode attn tokens/s per layer"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20  # written, then another as large read, between timed steps
# measured beside the headline at one GPU: (family, batch; None = the family's)
OTHER_CONFIGS = [("llama2_70b_prefix", None), ("long_context", 1), ("long_context", 4),
                 ("fp8_beams", None)]
SPEC_HBM_GBS = 8000.0
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "pa_decode_llama2_7b.md")
# the sources of the plain decode's kernels (main + split-K merge): the
# committed DRAM counters stay valid while these are unchanged
KERNEL_SOURCES = ["paged_kv_cache_410_b200/csrc/pa_common.cuh",
                  "paged_kv_cache_410_b200/csrc/pa_decode.cuh"]


# ---------------------------------------------------------------- helpers ---

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def rank_seed_offset(rank: int) -> int:
    """Each rank draws its own batch: the family's seed plus 1000 * rank."""
    return 1000 * rank


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def make_workload(name: str, rank: int, batch: int | None):
    from paged_kv_cache_410_b200 import workloads as W
    fam = W.FAMILIES[name]
    import inspect
    kw = {}
    params = inspect.signature(fam).parameters
    if batch is not None:
        kw["batch"] = batch
        if "beam_groups" in params:  # as many 4-beam groups as the batch holds, up to 16
            kw["beam_groups"] = min(params["beam_groups"].default,
                                    batch // params["beam_width"].default)
    seed = params["seed"].default
    if seed is None:  # fp8 family derives its seed from the block size
        seed = W.SEED_BASE + 5 + params["block_size"].default
    kw["seed"] = seed + rank_seed_offset(rank)
    return W.make(name, **kw)


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current kernel sources for this workload; else None."""
    try:
        text = open(PROFILE_SUMMARY).read()
    except OSError:
        return None
    def field(k):
        m = re.search(rf"^{k}:\s*(\S+)", text, re.M)
        return m.group(1) if m else None
    if field("workload") != workload_name or field("kernel_source_sha256") != kernel_source_hash():
        return None
    v = field("dram_bytes_per_full_launch")
    return float(v) if v else None


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except OSError:
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu_index), "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        def reader():
            for line in self.proc.stdout:
                self.lines.append(line.strip())
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ------------------------------------------------------------ CPU oracle ---

_ORACLE_CACHES = {}


def oracle_caches(w):
    """The oracle's copy of the workload's caches, made once per workload (set-up,
    not timed): the 16-bit pools as drawn, or an E4M3 pool that the oracle's own
    append fills from the workload's history tokens."""
    if id(w) not in _ORACLE_CACHES:
        if w.cache_dtype == "e4m3":
            import oracle
            shape = (w.num_blocks, w.block_size, w.num_kv_heads, w.head_dim)
            kc, vc = np.zeros(shape, np.uint8), np.zeros(shape, np.uint8)
            oracle.append_kv(w.fill_k, w.fill_v, w.io_dtype, w.fill_slots, kc, vc, "e4m3",
                             w.block_size, w.k_inv_scale, w.v_inv_scale)
        else:
            kc, vc = w.k_pool, w.v_pool
        _ORACLE_CACHES[id(w)] = (w, kc, vc)
    return _ORACLE_CACHES[id(w)][1:]


def oracle_step_time(w, seqs, reps=1, window=0):
    """Seconds for `reps` oracle passes over the sampled sequences: their
    copy-on-write pairs, the append of their new tokens and their decode
    (over the last `window` tokens when window > 0). Also returns the sample
    and the last pass's float64 output [n, Hq, D]."""
    import oracle
    from paged_kv_cache_410_b200 import workloads as W
    s = W.subset(w, seqs)
    kc, vc = oracle_caches(w)  # each pass rewrites the same slots and blocks
    t0 = time.perf_counter()
    for _ in range(reps):
        if len(s.copy_pairs):
            oracle.copy_blocks(s.copy_pairs, kc, vc, s.cache_dtype)
        oracle.append_kv(s.k_new, s.v_new, s.io_dtype, s.slot_mapping, kc, vc, s.cache_dtype,
                         s.block_size, s.k_inv_scale, s.v_inv_scale)
        out = oracle.decode(s.q, s.io_dtype, kc, vc, s.cache_dtype, s.block_tables,
                            s.context_lens, s.scale, k_scale=s.k_scale, v_scale=s.v_scale,
                            window=window)
    return time.perf_counter() - t0, s, out


def cpu_baseline(w, target_s=12.0, window=0):
    """Oracle throughput on a bounded sample: whole passes over the batch (or
    the first sequences of it) repeated until about `target_s` seconds.
    Returns the JSON object, the sampled sequence indices and the oracle's
    output for them."""
    import oracle
    from paged_kv_cache_410_b200 import accounting as A
    t1, _, _ = oracle_step_time(w, np.arange(1), window=window)
    per_seq = max(t1, 1e-4)
    n = int(min(w.batch, max(1, target_s / per_seq)))
    seqs = np.arange(n)
    t, s, out = oracle_step_time(w, seqs, window=window)
    reps = max(1, int(target_s / max(t, 1e-6)))
    if reps > 1:
        t, s, out = oracle_step_time(w, seqs, reps, window=window)
    nbytes = A.step_bytes(s, window=window)["total"] * reps
    return {"value": nbytes / t / 1e9, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{n} of {w.batch} sequences x {reps} passes (copies + append + decode), "
                      f"{t:.1f} s, float64 C oracle, OpenMP over (sequence, head)",
            "seconds": t, "tokens_per_s_per_layer": n * reps / t}, seqs, out


# decode tolerance on max-abs error against the float64 oracle, by output dtype
TOLERANCE = {"f16": 2e-3, "bf16": 1e-2}


def parity_summary(got: np.ndarray, want: np.ndarray, io_dtype: str,
                   against: str = "float64 CPU oracle, same inputs, the cpu_baseline sample") -> dict:
    """Max-abs error of the GPU output (float64 [n, Hq, D]) against the
    oracle's for the same sequences."""
    diff = np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))
    err = float(diff.max()) if diff.size else 0.0
    finite = math.isfinite(err)
    tol = TOLERANCE[io_dtype]
    return {"max_abs_err": err if finite else None, "tolerance": tol,
            "sequences": int(got.shape[0]), "ok": bool(finite and err <= tol),
            "against": against}


def parity_sample(w, n: int) -> np.ndarray:
    """Up to n sequences for a bench-side check: the shortest and the longest,
    the first beam group when the batch has one, then evenly spaced ones."""
    if n >= w.batch:
        return np.arange(w.batch)
    must = {int(np.argmin(w.context_lens)), int(np.argmax(w.context_lens))}
    if "beam_groups" in w.meta:
        must |= {0, 1, 2, 3}
    rest = [int(i) for i in np.linspace(0, w.batch - 1, n) if int(i) not in must]
    return np.array(sorted(must | set(rest[:max(0, n - len(must))])))


# ----------------------------------------------------------------- main ----

def cascade_blocks(args, w) -> int:
    """Shared-prefix blocks the step decodes through the cascade (0: none)."""
    if args.cascade != "auto" or args.window or args.fused:
        return 0
    return int(w.meta.get("shared_prefix_blocks", 0))


def decode_label(args, spb: int) -> str:
    return ("append fused into decode" if args.fused else
            f"sliding window {args.window}" if args.window else
            f"shared-prefix cascade ({spb} blocks)" if spb else
            "whole history")


def l2_note(flushed: bool, w) -> str:
    elt = 1 if w.cache_dtype == "e4m3" else 2
    pool_gb = 2 * w.num_blocks * w.block_size * w.num_kv_heads * w.head_dim * elt / 1e9
    if flushed:
        return (f"flushed: between timed steps, outside the timed events, a {L2_FLUSH_BYTES >> 20} "
                "MiB buffer (twice the L2) is written and another one read; step time = sum of "
                f"the per-step event intervals (pool {pool_gb:.2f} GB)")
    return f"not flushed: steps back to back (pool {pool_gb:.2f} GB)"


def base_line(args, w, n_gpus, spb=0):
    return {"metric": METRIC, "unit": UNIT, "n_gpus": n_gpus, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.cache_dtype, "data": "synthetic",
            "config": {"workload": w.name, "batch_per_gpu": w.batch,
                       "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
                       "head_dim": w.head_dim, "block_size": w.block_size,
                       "context_lens": f"{int(w.context_lens.min())}..{int(w.context_lens.max())}"
                                       f" (mean {float(w.context_lens.mean()):.0f})",
                       "kv_cache_dtype": w.cache_dtype, "io_dtype": w.io_dtype,
                       "parallelism": f"independent batch per GPU x{n_gpus}",
                       "l2": l2_note(not args.no_flush, w),
                       "decode": decode_label(args, spb)}}


def run_reference(args):
    rank, local_rank, world = dist_env()
    if rank != 0:
        return 0
    w = make_workload(args.workload, 0, args.batch)
    from paged_kv_cache_410_b200 import accounting as A
    import oracle
    oracle.build()
    # per-step sample sized so warmup + steps fit in about two minutes
    budget = min(10.0, 120.0 / max(1, args.steps + args.warmup))
    t1, _, _ = oracle_step_time(w, np.arange(1), window=args.window)
    n = int(min(w.batch, max(1, budget / max(t1, 1e-4))))
    seqs = np.arange(n)
    for _ in range(args.warmup):
        oracle_step_time(w, seqs, window=args.window)
    times = []
    s = None
    for _ in range(args.steps):
        t, s, _ = oracle_step_time(w, seqs, window=args.window)
        times.append(t)
    total = sum(times)
    nbytes = A.step_bytes(s, window=args.window)["total"] * args.steps
    value = nbytes / total / 1e9
    # the same config object as the GPU arm's line for the same flags (the
    # oracle has no cascade or fused form: it computes the same result)
    line = base_line(args, w, world, cascade_blocks(args, w))
    line["dtype"] = "f64"
    line.update({"impl": "reference", "value": value, "ms_per_step": 1e3 * total / args.steps,
                 "tokens_per_s_per_layer": n * args.steps / total,
                 "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                                  "kind": "oracle",
                                  "sample": f"{n} of {w.batch} sequences per step "
                                            "(copies + append + decode), float64 C oracle"},
                 "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                         "d2h_bytes_per_step": 0},
                 "gpu_launches": 0})
    print(json.dumps(line), flush=True)
    return 0


def make_step(args, w, dev, spb):
    from paged_kv_cache_410_b200.session import DecodeStep
    return DecodeStep(w, dev, partition_tokens=args.partition_tokens, shared_prefix_blocks=spb,
                      window=args.window, fused=args.fused)


def decode_plan(args, w, step, spb):
    """(partition tokens, partitions, decode launches, kernel description).
    A split decode of more than one sequence launches the work-list plan
    kernel, the decode and the split-K merge; one partition, the decode
    alone."""
    from paged_kv_cache_410_b200 import binding as B
    split = lambda n: (n > 1) * (2 + (w.batch > 1)) or 1  # noqa: E731
    if args.window:
        span = min(w.max_context, args.window + 15)
        pt = args.partition_tokens or B.pa_decode_partition_tokens(w.batch, span, step.cache)
        n = max(1, math.ceil(span / pt))
        return pt, n, split(n), (f"pa_decode_sliding_window (window {args.window}; "
                                 "main + split-K reduce)")
    if spb:
        pt = args.partition_tokens or B.pa_decode_shared_prefix_partition_tokens(
            w.batch, w.num_q_heads, w.max_context, spb, step.cache)
        n = max(1, math.ceil((w.max_context - spb * w.block_size) / pt))
        return pt, n, 3 if w.cache_dtype != "e4m3" else 2, \
            "pa_decode_shared_prefix (prefix + suffix + merge kernels)"
    pt = args.partition_tokens or B.pa_decode_partition_tokens(w.batch, w.max_context, step.cache)
    n = max(1, math.ceil(w.max_context / pt))
    name = ("pa_append_decode (append fused into decode; main + split-K reduce)" if args.fused
            else "pa_decode (main + split-K reduce)")
    if (not args.fused and w.batch == 1 and n > 1 and pt >= 1024 and w.cache_dtype != "e4m3"
            and w.block_size >= 16):
        # steal mode; the rows merge inside the (cooperative) launch when the
        # grid fits on the GPU at once: 3 CTAs per SM at head_dim 128 (66 KB
        # of shared memory, up to 168 registers), 4 at 64 (up to 128)
        import torch
        sms = torch.cuda.get_device_properties(step.q.device).multi_processor_count
        groups = w.num_kv_heads * -(-(w.num_q_heads // w.num_kv_heads) // 16)
        if n * groups <= sms * (3 if w.head_dim == 128 else 4) and 3 * groups * 8 <= (
                256 + -(-n * 8 // 256) * 256):
            return pt, n, 1, "pa_decode (steal mode, rows merged in the launch)"
        return pt, n, 2, "pa_decode (steal mode + split-K reduce)"
    return pt, n, split(n), name


class L2Flush:
    """Two buffers of L2_FLUSH_BYTES: `run()` writes the first and reads the
    second, so that L2 ends up holding clean lines of neither the step's
    data nor dirty ones whose write-back the next step would pay."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
        self.n = 0

    def run(self):
        self.n += 1
        self.w.fill_(self.n & 255)
        self.sink = self.r.sum()


def timed_steps(step, steps: int, fused: bool, stream, flush=None):
    """Record `steps` steps (copy, append, decode) on `stream` with a pair of
    events around each step and each decode call; with `flush` (an L2Flush),
    L2 is flushed before each step, outside its events. Returns the event
    pairs; read them after a synchronize."""
    import torch
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev_step = [(ev(), ev()) for _ in range(steps)]
    ev_dec = [(ev(), ev()) for _ in range(steps)]
    call = step.append_decode if fused else step.decode
    for i in range(steps):
        if flush is not None:
            flush.run()
        ev_step[i][0].record(stream)
        step.copy()
        if not fused:
            step.append()
        ev_dec[i][0].record(stream)
        call()
        ev_dec[i][1].record(stream)
        ev_step[i][1].record(stream)
    return ev_step, ev_dec


def elapsed(pairs):
    return [a.elapsed_time(b) for a, b in pairs]


def peak_gbs():
    peaks = measured_peaks()
    if peaks and peaks.get("hbm_gbs"):
        return float(peaks["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    return FALLBACK_HBM_GBS, "fallback (no MEASURED_PEAKS.json)"


def measure_other(args, name, batch, dev, stream, local_rank, peak):
    """One more workload in the same run: warm-up, then steps timed with the
    L2 flushed between them; its decode roofline, clocks, and sampled outputs
    checked against the oracle."""
    import torch
    from paged_kv_cache_410_b200 import accounting as A
    t_gen = time.perf_counter()
    w = make_workload(name, 0, batch)
    t_gen = time.perf_counter() - t_gen
    spb = int(w.meta.get("shared_prefix_blocks", 0))
    from paged_kv_cache_410_b200.session import DecodeStep
    step = DecodeStep(w, dev, shared_prefix_blocks=spb)
    sb = A.step_bytes(w)
    db = A.decode_bytes(w)
    pt, n_parts, dec_launches, kname = decode_plan(
        argparse.Namespace(window=0, fused=False, partition_tokens=0), w, step, spb)
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize(dev)
    if step.device_errors():
        raise RuntimeError(f"{name}: device bounds error during warm-up")
    flush = L2Flush(dev)
    steps = args.other_steps
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.25)
    ev_step, ev_dec = timed_steps(step, steps, False, stream, flush)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    step_ms, dec_ms = elapsed(ev_step), elapsed(ev_dec)
    errs = step.device_errors()
    del flush
    dmean = statistics.mean(dec_ms)
    achieved = sb["decode"] / (dmean * 1e-3) / 1e9
    res = {"workload": w.name, "batch": w.batch, "num_q_heads": w.num_q_heads,
           "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
           "kv_cache_dtype": w.cache_dtype, "io_dtype": w.io_dtype,
           "context_lens": f"{int(w.context_lens.min())}..{int(w.context_lens.max())} "
                           f"(mean {float(w.context_lens.mean()):.0f})",
           "decode": f"shared-prefix cascade ({spb} blocks)" if spb else "whole history",
           "kernel": kname, "partition_tokens": pt, "partitions": n_parts,
           "steps": steps, "l2": "flushed between steps",
           "decode_bytes": sb["decode"], "kv_unique_bytes": db["kv_unique"],
           "kv_logical_bytes": db["kv_logical"],
           "decode_ms_mean": dmean, "decode_ms_median": statistics.median(dec_ms),
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                        "frac": achieved / peak},
           "logical_gbs": (db["total_logical"]) / (dmean * 1e-3) / 1e9,
           "step_ms_mean": statistics.mean(step_ms),
           "step_gbs": sb["total"] / (statistics.mean(step_ms) * 1e-3) / 1e9,
           "tokens_per_s_per_layer": w.batch / (dmean * 1e-3),
           "gpu_launches_per_step": 1 + dec_launches + math.ceil(len(w.copy_pairs) / 256),
           "clocks": clk, "device_errors": errs, "workload_gen_s": t_gen}
    if not args.no_cpu_baseline:
        try:
            seqs = parity_sample(w, args.other_parity_seqs)
            _, _, want = oracle_step_time(w, seqs)
            got = step.out.double().cpu().numpy()[seqs]
            res["parity"] = parity_summary(got, want, w.io_dtype,
                                           "float64 CPU oracle, same inputs, sampled sequences")
        except Exception as e:  # report, never lose the measured line
            res["parity"] = {"error": repr(e)}
    _ORACLE_CACHES.pop(id(w), None)
    del step
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    import torch.distributed as dist
    rank, local_rank, world = dist_env()
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)

    from paged_kv_cache_410_b200 import accounting as A
    from paged_kv_cache_410_b200 import build as libbuild
    if not os.path.exists(libbuild.LIB):
        raise RuntimeError("libpagedattn.so is not built; run __graft_entry__.build()")

    w = make_workload(args.workload, rank, args.batch)
    spb = cascade_blocks(args, w)
    step = make_step(args, w, dev, spb)
    stream = torch.cuda.current_stream(dev)
    sb = A.step_bytes(w, window=args.window, fused=args.fused)
    plan_pt, n_parts, decode_launches, decode_name = decode_plan(args, w, step, spb)
    launches_per_step = (0 if args.fused else 1) + decode_launches + math.ceil(
        len(w.copy_pairs) / 256)
    timed_bytes = sb["append_decode"] if args.fused else sb["decode"]

    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize(dev)
    if step.device_errors():
        raise RuntimeError("device bounds error during warm-up")

    # ---- device-timed steps: L2 flushed between steps (default), then the
    # same steps back to back ----
    flush = None if args.no_flush else L2Flush(dev)
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.25)  # let the sampler start before the timed region
    ev_step, ev_dec = timed_steps(step, args.steps, args.fused, stream, flush)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    step_ms, decode_ms = elapsed(ev_step), elapsed(ev_dec)
    # back to back, no flush (the step reads more than L2 holds for the
    # default workload, so the two should agree)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    ev_dec_nf = None
    if flush is not None:
        del flush
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        t_start.record(stream)
        _, ev_dec_nf = timed_steps(step, args.steps, args.fused, stream, None)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    clk = clocks.stop()
    ms_total = max_over_ranks(sum(step_ms), dev)
    ms_per_step = ms_total / args.steps
    total_bytes = sum_over_ranks(sb["total"], dev) * args.steps
    value = total_bytes / (ms_total * 1e-3) / 1e9
    tokens_per_s = sum_over_ranks(w.batch, dev) * args.steps / (ms_total * 1e-3)

    # ---- end to end: host inputs -> device -> host output, every step ----
    pinned = {k: getattr(step, k).cpu().pin_memory()
              for k in ("q", "k_new", "v_new", "slot_mapping", "block_tables", "context_lens")}
    out_host = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = out_host.numel() * out_host.element_size()
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    for _ in range(2):
        for k, t in pinned.items():
            getattr(step, k).copy_(t, non_blocking=True)
        step.run()
        out_host.copy_(step.out, non_blocking=True)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        for k, t in pinned.items():
            getattr(step, k).copy_(t, non_blocking=True)
        step.run()
        out_host.copy_(step.out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_value = sum_over_ranks(sb["total"], dev) * e2e_steps / (e2e_ms * 1e-3) / 1e9
    errs = step.device_errors()

    # ---- roofline of the decode call ----
    peak, peak_src = peak_gbs()
    dec_ms = statistics.mean(decode_ms)
    achieved = timed_bytes / (dec_ms * 1e-3) / 1e9
    # the committed ncu counters cover the plain whole-history decode only
    traffic = None if (args.window or args.fused or spb) else recorded_traffic(w.name)

    line = base_line(args, w, world, spb)
    line.update({
        "value": value, "ms_per_step": ms_per_step,
        "tokens_per_s_per_layer": tokens_per_s,
        "frac_of_hbm_peak": value / peak,
        "frac_of_hbm_spec_8tbs": value / SPEC_HBM_GBS,
        "roofline": {"bound": "hbm", "kernel": decode_name,
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": peak_src,
                     "algorithmic_bytes_per_launch": timed_bytes,
                     "decode_ms_mean": dec_ms, "decode_ms_median": statistics.median(decode_ms),
                     "partition_tokens": plan_pt, "partitions": n_parts},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps},
        "gpu_launches": launches_per_step * args.steps,
        "bytes_per_step": sb,
        "clocks": clk,
        "device_errors": errs,
    })
    if ev_dec_nf is not None:
        nf_ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
        nf_dec = statistics.mean(elapsed(ev_dec_nf))
        line["unflushed"] = {
            "value": total_bytes / (nf_ms * 1e-3) / 1e9, "ms_per_step": nf_ms / args.steps,
            "decode_ms_mean": nf_dec,
            "roofline_achieved": timed_bytes / (nf_dec * 1e-3) / 1e9,
            "roofline_frac": timed_bytes / (nf_dec * 1e-3) / 1e9 / peak,
            "note": "the same steps back to back, without the L2 flush"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        cb, seqs, want = cpu_baseline(w, window=args.window)
        line["cpu_baseline"] = cb
        try:  # the GPU's output for the sampled sequences (last e2e step, same inputs)
            got = step.out.double().cpu().numpy()[seqs]
            line["parity"] = parity_summary(got, want, w.io_dtype)
        except Exception as e:  # report, never lose the measured line
            line["parity"] = {"error": repr(e)}
    if world == 1 and not args.no_other_configs:
        del step
        _ORACLE_CACHES.clear()
        torch.cuda.empty_cache()
        line["other_configs"] = {}
        for name, batch in OTHER_CONFIGS:
            if name == args.workload and batch == args.batch:
                continue
            key = name if batch is None else f"{name}_b{batch}"
            try:
                line["other_configs"][key] = measure_other(args, name, batch, dev, stream,
                                                           local_rank, peak)
            except Exception as e:  # report, never lose the headline
                line["other_configs"][key] = {"error": repr(e)}
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(
        description="Time one decode step of one attention layer (block copies, KV append, "
                    "paged decode) and print one JSON line.")
    ap.add_argument("--gpus", type=int, default=1, help="GPUs (one process each, torchrun)")
    ap.add_argument("--steps", type=int, default=2000, help="timed steps")
    ap.add_argument("--warmup", type=int, default=20, help="untimed steps first (>= 3)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours",
                    help="the CUDA library, or the float64 CPU oracle")
    ap.add_argument("--workload", default="llama2_7b",
                    choices=["tiny_mha", "llama2_7b", "llama2_70b_prefix", "long_context",
                             "fp8_beams"],
                    help="input family (its shapes and seed)")
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per GPU (default: the family's)")
    ap.add_argument("--partition-tokens", type=int, default=0,
                    help="split-K partition length (0: the library's choice)")
    ap.add_argument("--e2e-steps", type=int, default=200,
                    help="steps of the end-to-end measurement (host copies included)")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle baseline and its parity check")
    ap.add_argument("--window", type=int, default=0,
                    help="sliding-window decode over the last WINDOW tokens (0: whole history)")
    ap.add_argument("--fused", action="store_true",
                    help="append each sequence's new token inside the decode launch "
                         "(pa_append_decode) instead of a separate pa_append_kv")
    ap.add_argument("--cascade", choices=["auto", "off"], default="auto",
                    help="decode a workload whose sequences share prefix blocks through "
                         "pa_decode_shared_prefix (auto) or plain pa_decode (off)")
    ap.add_argument("--no-flush", action="store_true",
                    help="time the steps back to back, without the L2 flush between them")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="measure the headline workload only (at one GPU the line otherwise "
                         "adds the other benchmark families)")
    ap.add_argument("--other-steps", type=int, default=100,
                    help="timed steps of each other workload")
    ap.add_argument("--other-parity-seqs", type=int, default=16,
                    help="sequences of each other workload checked against the oracle")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
