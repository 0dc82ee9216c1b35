"""Benchmark of the exact attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
    python bench.py --peak        (bf16 / e4m3 dense matmul peaks of GPU 0)

One step = one attn_fwd call (every stage of the forward: tile schedule,
TMA loads, S = Q K^T, online softmax, O += P V, epilogue) over one batch of
the workload's seeded synthetic inputs, already resident in HBM.  Each step
is timed with CUDA events on the launching stream; between steps a 256 MiB
buffer is written to flush the 126 MB L2 and the SM clock is probed (both
untimed).  Prints one JSON line.  The default workload is the largest
one-GPU configuration (bf16 causal + window 4096, N = 16384); its line also
carries per_config, the throughput-vs-sequence-length curve over all five
forward configurations (N = 128 ... 16384), each timed the same way.
Other workloads: decode_* time one attn_fwd_decode call per step (key-range
and combine kernels); bf16_doccausal_* one attn_fwd_masked call (tile-range
pre-pass and the range variant of the forward kernel); bwd_* one attn_bwd
call (stats pass, dK/dV kernel, dQ kernel) after an untimed forward.
The line's e2e figure feeds the same call from pinned host memory and reads
the results back, every step's copies inside the timed region: pipelined
over three streams (copies in, compute, copies out; two device buffer sets)
for the forward workloads, one stream for decode and backward.

Multi-GPU: one process per GPU.  Under torchrun WORLD_SIZE must equal
--gpus; without torchrun, --gpus N > 1 relaunches the command as a torchrun
job of N ranks.  Each rank runs its own replica of the workload
(independent problems, no collective on the data path) or, with --shard
heads, its block of the workload's heads; the barrier and the
max-over-ranks reduction are the only communication.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_78_b200 import accounting  # noqa: E402
from exact_io_aware_78_b200.inputs import (BWD_WORKLOADS, CURVE_WORKLOADS, DECODE_WORKLOADS,  # noqa: E402
                                           DEFAULT_BENCH_WORKLOAD, WORKLOADS, decode_workload_inputs, head_shard,
                                           make_grad_output, shard_inputs, workload_inputs)

METRIC = "attention fwd TFLOP/s (and % of B200 dense BF16/FP8 peak) vs seq len, 1 GPU"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# The sources behind each kind of workload's kernels and launch code; a
# recorded ncu traffic figure is valid only while their hash is unchanged.
KERNEL_SOURCES = {
    "prefill": ["exact_io_aware_78_b200/csrc/attn_fwd_kernel.cuh", "exact_io_aware_78_b200/csrc/sm100_ptx.cuh",
                "exact_io_aware_78_b200/csrc/exactattn.cu"],
    "decode": ["exact_io_aware_78_b200/csrc/decode_tc_kernel.cuh", "exact_io_aware_78_b200/csrc/decode_kernel.cuh",
               "exact_io_aware_78_b200/csrc/decode_api.cuh", "exact_io_aware_78_b200/csrc/attn_fwd_kernel.cuh",
               "exact_io_aware_78_b200/csrc/sm100_ptx.cuh"],
    "backward": ["exact_io_aware_78_b200/csrc/attn_bwd_kernel.cuh", "exact_io_aware_78_b200/csrc/backward_api.cuh",
                 "exact_io_aware_78_b200/csrc/attn_fwd_kernel.cuh", "exact_io_aware_78_b200/csrc/sm100_ptx.cuh"],
}
METRIC_BWD = "attention bwd TFLOP/s (5 products of 2*d FLOPs per attended pair), 1 GPU"


def kernel_source_hash(kind: str = "prefill") -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def load_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu
    summary, or None when there is none or the kernel changed since."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        data = json.load(f)
    ent = data.get(workload)
    kind = ("decode" if workload.startswith("decode_") else "backward" if workload.startswith("bwd_")
            else "prefill")
    if not ent or ent.get("kernel_source_hash") != kernel_source_hash(kind):
        return None
    return ent.get("dram_bytes_per_launch")


LEAD_FLUSHES = 8


def queue_ahead(flush):
    """Untimed device work (L2 flushes, ~70 us each) queued just before the
    first timed step, so that the host enqueues the timed steps ahead of the
    device from the start: the host side of each call (argument marshalling,
    tensor-map encoding, launch) then never leaves the device idle after a
    step's start event, whatever the number of timed steps."""
    for _ in range(LEAD_FLUSHES):
        flush.zero_()


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.bus = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            self.bus = getattr(props, "pci_bus_id", None)
        except Exception:
            pass

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        rows = [r.split(", ") for r in out.strip().splitlines() if r.strip()]
        if not rows:
            return None
        bus_ids = sorted({r[0] for r in rows})
        if self.bus is not None:
            mine = [r for r in rows if r[0].lower().endswith(str(self.bus).lower()[-12:])]
            rows = mine or rows
        elif len(bus_ids) > 1:
            # pick the busiest GPU (highest median clock) when the mapping is unknown
            by = {b: [float(r[1]) for r in rows if r[0] == b] for b in bus_ids}
            best = max(by, key=lambda b: statistics.median(by[b]))
            rows = [r for r in rows if r[0] == best]
        sm = [float(r[1]) for r in rows]
        mx = max(float(r[2]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": reasons, "samples": len(sm),
                "power_w_max": max(float(r[3]) for r in rows)}


def init_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def dist_max(x: float, world: int, device) -> float:
    """Maximum of x over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_step: float, steps: int, world: int, max_total_ms: float) -> float:
    """Whole-job throughput: every rank runs `steps` steps of its own replica
    (weak scaling), timed by the slowest rank."""
    return flops_per_step * world * steps / (max_total_ms * 1e-3) / 1e12


def sharded_tflops(job_flops_per_step: float, steps: int, max_total_ms: float) -> float:
    """Whole-job throughput when the ranks split one problem's heads (strong
    scaling): the full problem's FLOPs per step over the slowest rank's time."""
    return job_flops_per_step * steps / (max_total_ms * 1e-3) / 1e12


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


# ------------------------------------------------------------ CPU oracle arm
def pairs_for_rows(rows, N: int, causal: bool, window: int, key_lo=None, key_hi=None) -> int:
    """Attended (query, key) pairs of the given query rows (key_lo, key_hi:
    this batch's per-row key ranges, length N, or None)."""
    r = np.asarray(rows, dtype=np.int64)
    hi = np.minimum(r + 1, N) if causal else np.full_like(r, N)
    lo = np.maximum(r - window + 1, 0) if window > 0 else np.zeros_like(r)
    if key_lo is not None:
        lo = np.maximum(lo, np.asarray(key_lo, dtype=np.int64)[r])
        hi = np.minimum(hi, np.asarray(key_hi, dtype=np.int64)[r])
    return int(np.maximum(hi - lo, 0).sum())


class OracleSampler:
    """Times the float64 oracle on consecutive 128-row chunks of the
    workload's (b, h) heads, continuing where the previous call stopped."""

    CHUNK = 128

    def __init__(self, w):
        from oracle import dequantize_per_head  # CPU baseline leg only

        self.w = w
        inp = workload_inputs(w)
        if w.dtype == "fp8":
            self.qkv = [dequantize_per_head(inp[n].view(torch.uint8).numpy(), inp[n + "_scale"].numpy())
                        for n in "qkv"]
        else:
            self.qkv = [inp[n].to(torch.float64).numpy() for n in "qkv"]
        self.ranges = (None, None) if inp.get("key_lo") is None else (inp["key_lo"].numpy(), inp["key_hi"].numpy())
        self.cursor = 0
        self.chunks_per_head = (w.N + self.CHUNK - 1) // self.CHUNK

    def run(self, budget_s: float):
        """Returns (seconds, attended FLOPs covered, rows done)."""
        from oracle import attention_ref  # CPU baseline leg only

        w = self.w
        g = w.Hq // w.Hkv
        q, k, v = self.qkv
        flops = 0.0
        rows_done = 0
        t0 = time.perf_counter()
        while True:
            idx = self.cursor % (w.B * w.Hq * self.chunks_per_head)
            self.cursor += 1
            bh, c = divmod(idx, self.chunks_per_head)
            b, h = divmod(bh, w.Hq)
            rows = list(range(c * self.CHUNK, min(w.N, (c + 1) * self.CHUNK)))
            lo, hi = self.ranges
            lo_b = None if lo is None else lo[b:b + 1]
            hi_b = None if hi is None else hi[b:b + 1]
            attention_ref(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, h // g:h // g + 1],
                          v[b:b + 1, :, h // g:h // g + 1], w.causal, w.window, w.scale, rows=rows,
                          key_lo=lo_b, key_hi=hi_b)
            flops += 4.0 * w.d * pairs_for_rows(rows, w.N, w.causal, w.window,
                                                None if lo is None else lo[b], None if hi is None else hi[b])
            rows_done += len(rows)
            if time.perf_counter() - t0 >= budget_s:
                break
        return time.perf_counter() - t0, flops, rows_done


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


class DecodeOracleSampler:
    """Times the float64 decode oracle one (b, h) head at a time (its Nq
    query rows against the whole cache), continuing where it stopped."""

    def __init__(self, w):
        inp = decode_workload_inputs(w)
        self.w = w
        self.qkv = [inp[n].to(torch.float64).numpy() for n in "qkv"]
        self.cursor = 0

    def run(self, budget_s: float):
        """Returns (seconds, attended FLOPs covered, query rows done)."""
        from oracle import attention_kv_ref  # CPU baseline leg only

        w = self.w
        q, k, v = self.qkv
        pairs = accounting.decode_pairs(w.Nq, w.Nk, w.causal, w.window)
        flops = 0.0
        rows_done = 0
        t0 = time.perf_counter()
        while True:
            b, h = divmod(self.cursor % (w.B * w.Hq), w.Hq)
            self.cursor += 1
            kh = h // w.group
            attention_kv_ref(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, kh:kh + 1], v[b:b + 1, :, kh:kh + 1],
                             w.causal, w.window, w.scale)
            flops += 4.0 * w.d * pairs
            rows_done += w.Nq
            if time.perf_counter() - t0 >= budget_s:
                break
        return time.perf_counter() - t0, flops, rows_done


def is_decode(w) -> bool:
    return w.name in DECODE_WORKLOADS


def is_backward(w) -> bool:
    return w.name in BWD_WORKLOADS


class BackwardOracleSampler:
    """Times the float64 backward oracle one (b, h) query head at a time
    (with its key/value head), continuing where it stopped."""

    def __init__(self, w):
        inp = workload_inputs(w)
        self.w = w
        self.qkv = [inp[n].to(torch.float64).numpy() for n in "qkv"]
        self.do = make_grad_output(w.B, w.N, w.Hq, w.d, w.seed + 3).to(torch.float64).numpy()
        self.ranges = (None, None) if inp.get("key_lo") is None else (inp["key_lo"].numpy(), inp["key_hi"].numpy())
        self.cursor = 0

    def run(self, budget_s: float):
        """Returns (seconds, backward FLOPs covered, query rows done)."""
        from oracle import attention_bwd_ref  # CPU baseline leg only

        w = self.w
        q, k, v = self.qkv
        lo, hi = self.ranges
        flops = 0.0
        rows_done = 0
        t0 = time.perf_counter()
        while True:
            b, h = divmod(self.cursor % (w.B * w.Hq), w.Hq)
            self.cursor += 1
            kh = h // w.group
            lo_b = None if lo is None else lo[b:b + 1]
            hi_b = None if hi is None else hi[b:b + 1]
            attention_bwd_ref(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, kh:kh + 1], v[b:b + 1, :, kh:kh + 1],
                              self.do[b:b + 1, :, h:h + 1], w.causal, w.window, w.scale, key_lo=lo_b, key_hi=hi_b)
            pairs = (accounting.attended_pairs(w.N, w.causal, w.window) if lo is None else
                     accounting.range_pairs(lo_b, hi_b, w.causal, w.window))
            flops += 10.0 * w.d * pairs
            rows_done += w.N
            if time.perf_counter() - t0 >= budget_s:
                break
        return time.perf_counter() - t0, flops, rows_done


def run_reference(args, w, world, rank):
    if rank != 0:
        print(f"reference arm: rank {rank} of {world} exits without work", file=sys.stderr, flush=True)
        return
    times = []
    flops_done = 0.0
    rows_total = 0
    per_step_budget = min(20.0, args.ref_seconds / max(1, args.steps + args.warmup))
    sampler = (DecodeOracleSampler(w) if is_decode(w) else BackwardOracleSampler(w) if is_backward(w)
               else OracleSampler(w))
    for i in range(args.warmup + args.steps):
        dt, fl, rows = sampler.run(per_step_budget)
        if i >= args.warmup:
            times.append(dt)
            flops_done += fl
            rows_total += rows
    value = flops_done / sum(times) / 1e12
    unit_desc = ("query rows (all Nq rows of consecutive (b,h) heads)" if is_decode(w) else
                 "query rows (all N rows of consecutive (b,h) heads, backward)" if is_backward(w) else
                 "query rows (128-row chunks of consecutive (b,h) heads)")
    sample = (f"{rows_total} {unit_desc} of {w.name} over "
              f"{args.steps} steps of ~{per_step_budget:.3g} s, numpy float64 two-pass oracle; "
              f"TFLOP/s counts attended-pair FLOPs")
    line = {
        "impl": "reference", "metric": METRIC_BWD if is_backward(w) else METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": any_line_config(w, world, args.shard),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": host_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w) -> dict:
    if is_decode(w):
        return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
                "causal": w.causal, "window": w.window, "input_dtype": "bf16"}
    cfg = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
           "causal": w.causal, "window": w.window, "input_dtype": w.dtype}
    if w.mask:
        cfg["row_ranges"] = f"{w.mask} of {w.mask_min}-{w.mask_max} tokens"
    return cfg


# ------------------------------------------------------------- CUDA arm
PROBE_CYCLES = (50_000, 250_000)


def sm_clock_probe(stream):
    """Queue an in-stream SM clock measurement: two spin kernels of known
    SM-clock cycle counts between events.  The difference of their durations
    cancels the fixed launch cost; returns the three events."""
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    ev[0].record(stream)
    torch.cuda._sleep(PROBE_CYCLES[0])
    ev[1].record(stream)
    torch.cuda._sleep(PROBE_CYCLES[1])
    ev[2].record(stream)
    return ev


def probe_mhz(ev) -> float:
    dt_ms = ev[1].elapsed_time(ev[2]) - ev[0].elapsed_time(ev[1])
    return (PROBE_CYCLES[1] - PROBE_CYCLES[0]) / (dt_ms * 1e3) if dt_ms > 0 else float("nan")


def time_steps(step, flush, stream, dev, args, world, rank, local, check_error):
    """W untimed warm-up steps, then exactly K steps each between CUDA events
    on the launching stream, L2 flushed (untimed) before each.  After each
    timed step (outside its events) an SM clock probe runs, so every step has
    the SM clock it ran at.  Returns (per-step ms, nvidia-smi clock record,
    per-step probed SM MHz)."""
    for _ in range(args.warmup):
        flush.zero_()
        step()
    check_error("warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(local) if rank == 0 else None
    barrier(world)
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    queue_ahead(flush)
    probes = []
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
        probes.append(sm_clock_probe(stream))
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = sampler.stop() if sampler else None
    check_error("the timed region")
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    return step_ms, clocks, [probe_mhz(ev) for ev in probes]


def with_probe(clocks, mhz, ms_per_step):
    """The nvidia-smi record plus the probed SM clock of the timed steps (and
    the SM cycles per step it implies)."""
    out = dict(clocks) if clocks else {}
    m = statistics.median(mhz)
    out["sm_mhz_probe_median"] = m
    out["sm_mhz_probe_min"] = min(mhz)
    out["sm_cycles_per_step"] = ms_per_step * 1e-3 * m * 1e6
    out["probe"] = "torch.cuda._sleep spin kernels after each timed step (outside its events)"
    return out


def fp8_peak_record():
    """The e4m3 dense matmul peak measured on a B200 of this machine (committed
    summary of `python bench.py --peak`), or None."""
    path = os.path.join(ROOT, "profiles", "peaks_fp8.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        return json.load(f)


def prefill_roofline(w, launch_ms, peaks, peak_kind):
    """Roofline of the attention kernel for one workload: tensor-bound at
    4*d FLOPs per attended pair against the dense peak of its input format,
    except the tiny fp32 case, which launch latency bounds (reported as
    algorithmic GB/s against the copy bandwidth)."""
    flops = accounting.flops(w)
    nbytes = accounting.algorithmic_bytes(w)
    if w.dtype == "fp32" and w.N <= 256:
        achieved = nbytes / (launch_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": load_traffic(w.name),
                "peak_source": f"{peak_kind} HBM copy bandwidth (launch-latency bound: 2 launches)",
                "algorithmic_bytes": nbytes, "kernel_source_hash": kernel_source_hash()}
    achieved = flops / (launch_ms * 1e-3) / 1e12
    peak, peak_sustained = peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]
    note = f"{peak_kind} bf16 burst (kernel timed alone)"
    if w.dtype == "fp8":
        rec = fp8_peak_record()
        if rec:
            peak, peak_sustained = rec["fp8_tflops"], rec["fp8_tflops_sustained"]
            note = "measured e4m3 burst (torch._scaled_mm 8192^3 on a B200 of this pool, profiles/peaks_fp8.json)"
        else:
            peak, peak_sustained = 2 * peak, 2 * peak_sustained
            note = f"{peak_kind} bf16 burst x 2 (nominal fp8/bf16 dense ratio)"
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": load_traffic(w.name), "peak_source": note, "peak_sustained": peak_sustained,
            "frac_sustained": achieved / peak_sustained, "algorithmic_bytes": nbytes,
            "kernel_source_hash": kernel_source_hash()}


def _timing_config(world: int, shard: str) -> dict:
    return {"l2": "flushed between timed steps (256 MiB write, untimed)",
            "host": f"{LEAD_FLUSHES} untimed L2 flushes queued before the first timed step",
            "parallelism": (f"head shards x{world}" if shard == "heads" else
                            f"replicas x{world}" if world > 1 else "single GPU")}


def line_config(w, world: int, shard: str) -> dict:
    """The `config` object of a forward line; both arms print the same one."""
    return {**workload_config(w), "flops_per_step": accounting.flops(w),
            "flops_half_square_per_step": accounting.flops_half_square(w), **_timing_config(world, shard)}


def bwd_line_config(w, world: int, shard: str) -> dict:
    return {**workload_config(w), "pass": "backward", "flops_per_step": accounting.bwd_flops(w),
            **_timing_config(world, shard)}


def decode_line_config(w, world: int, shard: str) -> dict:
    return {**workload_config(w), "flops_per_step": accounting.decode_flops(w), **_timing_config(world, shard)}


def any_line_config(w, world: int, shard: str) -> dict:
    if is_decode(w):
        return decode_line_config(w, world, shard)
    if is_backward(w):
        return bwd_line_config(w, world, shard)
    return line_config(w, world, shard)


class PrefillProblem:
    """Device buffers and the step (one attn_fwd, or attn_fwd_masked with
    per-row key ranges) of one forward workload, this rank's shard of it
    with --shard heads."""

    def __init__(self, w_job, args, world, rank, dev, stream):
        import exact_io_aware_78_b200 as ea

        self.w_job = w = w_job
        inp = workload_inputs(w_job)
        if args.shard == "heads":
            w, q_lo, q_hi, kv_lo, kv_hi = head_shard(w_job, world, rank)
            inp = shard_inputs(inp, q_lo, q_hi, kv_lo, kv_hi)
        self.w, self.inp = w, inp
        self.q, self.k, self.v = (inp[n].to(dev) for n in "qkv")
        self.scales = [None if inp[n + "_scale"] is None else inp[n + "_scale"].to(dev) for n in "qkv"]
        self.masked = inp.get("key_lo") is not None
        self.key_lo, self.key_hi = ((inp[n].to(dev) for n in ("key_lo", "key_hi")) if self.masked
                                    else (None, None))
        o_dtype = torch.float32 if w.dtype == "fp32" else torch.bfloat16
        self.o = torch.empty((w.B, w.N, w.Hq, w.d), device=dev, dtype=o_dtype)
        self.lse = torch.empty((w.B, w.Hq, w.N), device=dev, dtype=torch.float32)
        self.stream = stream
        self.ea = ea
        # fp32: + the split kernel; row ranges: + the tile-range kernel
        self.launches = 1 + int(w.dtype == "fp32") + int(self.masked)

    def buffers(self):
        """This problem's device tensors by name (inputs, then O and LSE)."""
        return {"q": self.q, "k": self.k, "v": self.v, "key_lo": self.key_lo, "key_hi": self.key_hi, "o": self.o,
                "lse": self.lse}

    def step(self, bufs=None):
        """One forward on the stream, on this problem's buffers or on another
        set of the same shapes (bufs, as buffers() names them)."""
        w, ea = self.w, self.ea
        b = self.buffers() if bufs is None else bufs
        if self.masked:
            ea.attn_fwd_masked(b["q"], b["k"], b["v"], b["o"], b["lse"], b["key_lo"], b["key_hi"], w.causal,
                               w.window, w.scale, *self.scales, stream=self.stream)
        else:
            ea.attn_fwd(b["q"], b["k"], b["v"], b["o"], b["lse"], w.causal, w.window, w.scale, *self.scales,
                        stream=self.stream)

    def check_error(self, where):
        st, code, site = self.ea.attn_get_last_error(self.stream)
        if st != 0:
            raise RuntimeError(f"device error {code} at site {site} during {where}")


def pipelined_e2e(pb, stream, dev, steps):
    """Time `steps` forward steps fed from pinned host memory, copies in, compute and copies out on three
    streams with two alternating device buffer sets (after two untimed steps); returns (total ms, the
    (device, host) input pairs of one set, the host O and LSE buffers)."""
    inp = pb.inp
    names = ["q", "k", "v"] + (["key_lo", "key_hi"] if pb.masked else [])
    host = {n: inp[n].pin_memory() for n in names}
    oh = torch.empty(pb.o.shape, dtype=pb.o.dtype).pin_memory()
    lh = torch.empty(pb.lse.shape, dtype=torch.float32).pin_memory()
    sets = [pb.buffers()]
    sets.append({n: (None if t is None else torch.empty_like(t)) for n, t in sets[0].items()})
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        torch.cuda.synchronize(dev)
        es = torch.cuda.Event(enable_timing=True)
        ee = torch.cuda.Event(enable_timing=True)
        es.record(s_in)
        for i in range(n):
            j = i % 2
            b = sets[j]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[j])  # step i-2 has read this set's inputs
                for nm in names:
                    b[nm].copy_(host[nm], non_blocking=True)
                in_done[j].record(s_in)
            stream.wait_event(in_done[j])
            if i >= 2:
                stream.wait_event(out_done[j])  # step i-2's outputs have left this set
            pb.step(b)
            comp_done[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[j])
                oh.copy_(b["o"], non_blocking=True)
                lh.copy_(b["lse"], non_blocking=True)
                out_done[j].record(s_out)
        ee.record(s_out)
        ee.synchronize()
        return es.elapsed_time(ee)

    run(2)
    total = run(steps)
    pb.check_error("pipelined end-to-end steps")
    return total, [(sets[0][nm], host[nm]) for nm in names], oh, lh


def job_value(pb, args, world, total_ms, steps):
    if args.shard == "heads":
        return sharded_tflops(accounting.flops(pb.w_job), steps, total_ms)
    return job_tflops(accounting.flops(pb.w), steps, world, total_ms)


def curve_entry(pb, args, world, rank, local, dev, flush, peaks, peak_kind):
    """One point of the throughput-vs-sequence-length curve, timed exactly as
    the line's own workload (same K, W, flushes and clock probes)."""
    step_ms, clocks, mhz = time_steps(pb.step, flush, pb.stream, dev, args, world, rank, local, pb.check_error)
    total_ms = dist_max(sum(step_ms), world, dev)
    launch_ms = statistics.mean(step_ms)
    w = pb.w_job
    entry = {"workload": w.name, "N": w.N, "input_dtype": w.dtype, "value": job_value(pb, args, world, total_ms,
                                                                                    args.steps),
             "unit": "TFLOP/s", "ms_per_step": total_ms / args.steps,
             "roofline": prefill_roofline(pb.w, launch_ms, peaks, peak_kind),
             "gpu_launches": args.steps * pb.launches,
             "clocks": with_probe(clocks, mhz, launch_ms)}
    return entry


def run_cuda(args, w, world, rank, local):
    import exact_io_aware_78_b200 as ea

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    ea.load_library()
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    peaks, peak_kind = load_peaks()
    pb = PrefillProblem(w, args, world, rank, dev, stream)
    step_ms, clocks, mhz = time_steps(pb.step, flush, stream, dev, args, world, rank, local, pb.check_error)
    total_ms = dist_max(sum(step_ms), world, dev)
    value = job_value(pb, args, world, total_ms, args.steps)

    # e2e: the public API fed from pinned host memory as a user streaming batches runs it -- step i's inputs
    # are copied in on one stream while step i-1 computes and step i-2's outputs are copied out on a third
    # stream, two device buffer sets alternating.  Every step's copies lie inside the timed region, which runs
    # from the first copy in to the last copy out.
    e2e_steps = max(3, min(args.steps, 50))
    e2e_ms_total, host_in, oh, lh = pipelined_e2e(pb, stream, dev, e2e_steps)
    e2e_total = dist_max(e2e_ms_total, world, dev)
    e2e_value = job_value(pb, args, world, e2e_total, e2e_steps)
    h2d = sum(src.numel() * src.element_size() for _, src in host_in)
    d2h = oh.numel() * oh.element_size() + lh.numel() * 4
    launch_ms = statistics.mean(step_ms)
    w_job = pb.w_job
    top = {"workload": w_job.name, "N": w_job.N, "input_dtype": w_job.dtype, "value": value, "unit": "TFLOP/s",
           "ms_per_step": total_ms / args.steps, "roofline": prefill_roofline(pb.w, launch_ms, peaks, peak_kind),
           "gpu_launches": args.steps * pb.launches, "clocks": with_probe(clocks, mhz, launch_ms)}
    launches = pb.launches
    del pb, host_in, oh, lh

    # The rest of the curve: every forward configuration, each timed the same way.
    curve = None
    if args.curve == "on" or (args.curve == "auto" and w.name == DEFAULT_BENCH_WORKLOAD):
        curve = []
        for name in CURVE_WORKLOADS:
            if name == w.name:
                curve.append(top)
                continue
            other = PrefillProblem(WORKLOADS[name], args, world, rank, dev, stream)
            curve.append(curve_entry(other, args, world, rank, local, dev, flush, peaks, peak_kind))
            del other
            torch.cuda.empty_cache()

    if rank != 0:
        return
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "strong" if args.shard == "heads" else "weak",
        "vs_baseline": None,
        "dtype": {"bf16": "bf16", "fp8": "e4m3", "fp32": "bf16x3 (fp32 in/out)"}[w_job.dtype],
        "data": "synthetic",
        "config": line_config(w_job, world, args.shard),
        "roofline": top["roofline"],
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "mode": "pipelined: step i's copies in, step i-1's compute and step i-2's copies out on three streams, "
                        "two device buffer sets; timed from the first copy in to the last copy out"},
        "gpu_launches": args.steps * launches,
        "clocks": top["clocks"],
    }
    if curve is not None:
        line["per_config"] = curve
    if world == 1 and not args.no_cpu_baseline:
        dt, fl, rows = OracleSampler(w_job).run(args.cpu_seconds)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": host_cores(), "kind": "oracle",
                                "sample": f"{rows} query rows (128-row chunks of consecutive (b,h) heads) of "
                                          f"{w_job.name} in {dt:.1f} s, numpy float64 two-pass oracle; TFLOP/s "
                                          f"counts attended-pair FLOPs"}
    print(json.dumps(line), flush=True)


def run_backward_cuda(args, w, world, rank, local):
    """One backward step (attn_bwd: the stats pass, the dK/dV kernel and the
    dQ kernel) per timed iteration; O and LSE come from one untimed forward."""
    import exact_io_aware_78_b200 as ea

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    ea.load_library()
    w_job = w
    inp = workload_inputs(w)
    inp["do"] = make_grad_output(w.B, w.N, w.Hq, w.d, w.seed + 3)
    if args.shard == "heads":
        w, q_lo, q_hi, kv_lo, kv_hi = head_shard(w_job, world, rank)
        do_full = inp["do"]
        inp = shard_inputs(inp, q_lo, q_hi, kv_lo, kv_hi)
        inp["do"] = do_full[:, :, q_lo:q_hi].contiguous()
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    masked = inp.get("key_lo") is not None
    key_lo, key_hi = (inp[n].to(dev) for n in ("key_lo", "key_hi")) if masked else (None, None)
    o, lse = ea.forward(q, k, v, causal=w.causal, window=w.window, scale=w.scale, key_lo=key_lo, key_hi=key_hi)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        if masked:
            ea.attn_bwd_masked(q, k, v, o, lse, do, dq, dk, dv, key_lo, key_hi, w.causal, w.window, w.scale,
                               stream=stream)
        else:
            ea.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, w.causal, w.window, w.scale, stream=stream)

    def check_error(where):
        st, code, site = ea.attn_get_last_error(stream)
        if st != 0:
            raise RuntimeError(f"device error {code} at site {site} during {where}")

    step_ms, clocks, mhz = time_steps(step, flush, stream, dev, args, world, rank, local, check_error)
    total_ms = dist_max(sum(step_ms), world, dev)
    flops = accounting.bwd_flops(w)
    if args.shard == "heads":
        value = sharded_tflops(accounting.bwd_flops(w_job), args.steps, total_ms)
    else:
        value = job_tflops(flops, args.steps, world, total_ms)

    # e2e: the public call with the step's inputs copied from pinned host memory
    host_in = [(t, t.cpu().pin_memory()) for t in (q, k, v, o, lse, do) + ((key_lo, key_hi) if masked else ())]
    host_out = [(t, torch.empty(t.shape, dtype=t.dtype).pin_memory()) for t in (dq, dk, dv)]
    e2e_steps = max(3, min(args.steps, 50))
    es = torch.cuda.Event(enable_timing=True)
    ee = torch.cuda.Event(enable_timing=True)
    e2e_ms = []
    for i in range(e2e_steps + 2):
        flush.zero_()
        es.record(stream)
        for dst, src in host_in:
            dst.copy_(src, non_blocking=True)
        step()
        for src, dst in host_out:
            dst.copy_(src, non_blocking=True)
        ee.record(stream)
        ee.synchronize()
        if i >= 2:
            e2e_ms.append(es.elapsed_time(ee))
    e2e_total = dist_max(sum(e2e_ms), world, dev)
    if args.shard == "heads":
        e2e_value = sharded_tflops(accounting.bwd_flops(w_job), e2e_steps, e2e_total)
    else:
        e2e_value = job_tflops(flops, e2e_steps, world, e2e_total)
    h2d = sum(src.numel() * src.element_size() for _, src in host_in)
    d2h = sum(dst.numel() * dst.element_size() for _, dst in host_out)

    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    launch_ms = statistics.mean(step_ms)
    achieved = flops / (launch_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC_BWD,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "strong" if args.shard == "heads" else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": bwd_line_config(w_job, world, args.shard),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "traffic": load_traffic(w.name),
                     "peak_source": f"{peak_kind} bf16 burst (kernel timed alone)",
                     "peak_sustained": peaks["bf16_tflops_sustained"],
                     "frac_sustained": achieved / peaks["bf16_tflops_sustained"],
                     "algorithmic_bytes": accounting.bwd_bytes(w),
                     "kernel_source_hash": kernel_source_hash("backward"),
                     "note": "achieved over the whole step (stats pass + dK/dV kernel + dQ kernel)"},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        # stats pass, dK/dV and dQ kernels; row ranges: + the two tile-table kernels
        "gpu_launches": args.steps * (5 if masked else 3),
        "clocks": with_probe(clocks, mhz, launch_ms),
    }
    if world == 1 and not args.no_cpu_baseline:
        dt, fl, rows = BackwardOracleSampler(w).run(args.cpu_seconds)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": host_cores(), "kind": "oracle",
                                "sample": f"{rows} query rows (all rows of consecutive (b,h) heads) of {w.name} "
                                          f"in {dt:.1f} s, numpy float64 backward oracle; TFLOP/s counts 10*d "
                                          f"FLOPs per attended pair"}
    print(json.dumps(line), flush=True)


def run_decode_cuda(args, w, world, rank, local):
    """A decode step (attn_fwd_decode): Nq new query rows per (b, h) against a
    cache of Nk keys.  HBM-bound, so the roofline is the measured copy
    bandwidth over the step's algorithmic bytes (Q, the visible K/V rows, O,
    LSE, each moved once); the value is still attended-pair TFLOP/s."""
    import exact_io_aware_78_b200 as ea

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    ea.load_library()
    w_job = w
    inp = decode_workload_inputs(w)
    if args.shard == "heads":
        w, q_lo, q_hi, kv_lo, kv_hi = head_shard(w_job, world, rank)
        inp = shard_inputs(inp, q_lo, q_hi, kv_lo, kv_hi)
    q, k, v = (inp[n].to(dev) for n in "qkv")
    o = torch.empty((w.B, w.Nq, w.Hq, w.d), device=dev, dtype=torch.bfloat16)
    lse = torch.empty((w.B, w.Hq, w.Nq), device=dev, dtype=torch.float32)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ea.attn_fwd_decode(q, k, v, o, lse, w.causal, w.window, w.scale, 0, stream=stream)

    def check_error(where):
        st, code, site = ea.attn_get_last_error(stream)
        if st != 0:
            raise RuntimeError(f"device error {code} at site {site} during {where}")

    step_ms, clocks, mhz = time_steps(step, flush, stream, dev, args, world, rank, local, check_error)
    total_ms = dist_max(sum(step_ms), world, dev)
    flops = accounting.decode_flops(w)
    if args.shard == "heads":
        value = sharded_tflops(accounting.decode_flops(w_job), args.steps, total_ms)
    else:
        value = job_tflops(flops, args.steps, world, total_ms)

    # e2e: the public call with the step's inputs copied from pinned host memory
    qh, kh, vh = (inp[n].pin_memory() for n in "qkv")
    oh = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    lh = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    es = torch.cuda.Event(enable_timing=True)
    ee = torch.cuda.Event(enable_timing=True)
    e2e_ms = []
    for i in range(e2e_steps + 2):
        flush.zero_()
        es.record(stream)
        q.copy_(qh, non_blocking=True)
        k.copy_(kh, non_blocking=True)
        v.copy_(vh, non_blocking=True)
        step()
        oh.copy_(o, non_blocking=True)
        lh.copy_(lse, non_blocking=True)
        ee.record(stream)
        ee.synchronize()
        if i >= 2:
            e2e_ms.append(es.elapsed_time(ee))
    e2e_total = dist_max(sum(e2e_ms), world, dev)
    if args.shard == "heads":
        e2e_value = sharded_tflops(accounting.decode_flops(w_job), e2e_steps, e2e_total)
    else:
        e2e_value = job_tflops(flops, e2e_steps, world, e2e_total)
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size() + lh.numel() * 4

    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    launch_ms = statistics.mean(step_ms)
    nbytes = accounting.decode_bytes(w)
    achieved = nbytes / (launch_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "strong" if args.shard == "heads" else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": decode_line_config(w_job, world, args.shard),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": load_traffic(w.name),
                     "peak_source": f"{peak_kind} HBM copy bandwidth", "algorithmic_bytes": nbytes,
                     "kernel_source_hash": kernel_source_hash("decode")},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * 2,  # key-range kernel + combine kernel
        "clocks": with_probe(clocks, mhz, launch_ms),
    }
    if world == 1 and not args.no_cpu_baseline:
        dt, fl, rows = DecodeOracleSampler(w).run(args.cpu_seconds)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": host_cores(), "kind": "oracle",
                                "sample": f"{rows} query rows (all Nq rows of consecutive (b,h) heads) of "
                                          f"{w.name} in {dt:.1f} s, numpy float64 two-pass oracle; TFLOP/s "
                                          f"counts attended-pair FLOPs"}
    print(json.dumps(line), flush=True)


def world_from_env():
    return int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0"))


def resolve_launch(gpus: int, env) -> str:
    """How to honour --gpus N: "run" in this process (one GPU, or already one
    rank of a torchrun job of N), "spawn" N ranks from here (N > 1 and no
    torchrun environment); a torchrun job of another size is an error."""
    if gpus < 1:
        raise ValueError("--gpus must be >= 1")
    if "WORLD_SIZE" in env:
        world = int(env["WORLD_SIZE"])
        if world != gpus:
            raise ValueError(f"--gpus {gpus} but WORLD_SIZE={world}: launch as many ranks as --gpus asks for")
        return "run"
    return "spawn" if gpus > 1 else "run"


def spawn_ranks(gpus: int) -> int:
    """Relaunch this command as a torchrun job of `gpus` ranks on this node
    (one process per GPU, rendezvous on 127.0.0.1); returns its exit code."""
    import socket
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def measure_peaks(args):
    """Dense matmul peaks on this GPU for the roofline denominators: torch
    bf16 matmul and e4m3 torch._scaled_mm (bf16 output, unit scales) at
    8192^3.  Burst: best of 10 single calls, each followed by an SM clock
    probe, taken for both formats (after a short idle, twice) before any
    long load; sustained: back-to-back calls for about --peak-seconds each,
    with nvidia-smi clocks sampled meanwhile.  Prints one JSON line."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    n = 8192
    g = torch.Generator(device="cpu")
    g.manual_seed(88)
    a = torch.randn(n, n, generator=g).to(dev)
    b = torch.randn(n, n, generator=g).to(dev)
    a16, b16 = a.to(torch.bfloat16), b.to(torch.bfloat16)
    a8 = a.clamp(-448, 448).to(torch.float8_e4m3fn)
    b8 = b.clamp(-448, 448).to(torch.float8_e4m3fn).t().contiguous().t()  # column-major, as _scaled_mm wants
    one = torch.ones((), device=dev, dtype=torch.float32)
    del a, b
    stream = torch.cuda.current_stream(dev)
    kinds = {"bf16": lambda: torch.matmul(a16, b16),
             "fp8": lambda: torch._scaled_mm(a8, b8, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)}
    flop = 2.0 * n ** 3
    out = {"what": "dense matmul peaks, 8192^3", "gpu": torch.cuda.get_device_name(dev)}
    best = {k: float("inf") for k in kinds}
    mhz = {k: [] for k in kinds}
    for rnd in range(2):
        for name, fn in kinds.items():
            time.sleep(1.0)
            for _ in range(3):
                fn()
            torch.cuda.synchronize(dev)
            for _ in range(10):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                ev = sm_clock_probe(stream)
                torch.cuda.synchronize(dev)
                t = e0.elapsed_time(e1)
                if t < best[name]:
                    best[name] = t
                mhz[name].append(probe_mhz(ev))
    for name, fn in kinds.items():
        out[f"{name}_tflops"] = flop / (best[name] * 1e-3) / 1e12
        out[f"{name}_burst_sm_mhz_probe_median"] = statistics.median(mhz[name])
    for name, fn in kinds.items():
        time.sleep(2.0)
        sampler = ClockSampler(0)
        sampler.start()
        t_end = time.perf_counter() + args.peak_seconds
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        calls = 0
        while time.perf_counter() < t_end:
            for _ in range(20):
                fn()
            calls += 20
            torch.cuda.synchronize(dev)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        out[f"{name}_tflops_sustained"] = flop * calls / (e0.elapsed_time(e1) * 1e-3) / 1e12
        out[f"{name}_sustained_clocks"] = sampler.stop()
    out["fp8_over_bf16_burst"] = out["fp8_tflops"] / out["bf16_tflops"]
    out["fp8_over_bf16_sustained"] = out["fp8_tflops_sustained"] / out["bf16_tflops_sustained"]
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1,
                    help="GPUs of this node; without a torchrun environment N > 1 relaunches this command as a "
                         "torchrun job of N ranks")
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_BENCH_WORKLOAD,
                    choices=sorted(WORKLOADS) + sorted(DECODE_WORKLOADS) + sorted(BWD_WORKLOADS))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="with several GPUs: each runs its own replica of the workload (weak scaling), or the "
                         "GPUs split the workload's heads (strong scaling; Hkv must divide by the GPU count)")
    ap.add_argument("--curve", default="auto", choices=["auto", "on", "off"],
                    help="add per_config: every forward configuration timed the same way (auto: with the "
                         "default workload)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="host time for the cpu_baseline sample of the CUDA arm")
    ap.add_argument("--ref-seconds", type=float, default=150.0,
                    help="total host time budget of the --impl reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--peak", action="store_true",
                    help="measure the bf16 and e4m3 dense matmul peaks of GPU 0 instead (one JSON line)")
    ap.add_argument("--peak-seconds", type=float, default=4.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.peak:
        measure_peaks(args)
        return
    try:
        how = resolve_launch(args.gpus, os.environ)
    except ValueError as e:
        ap.error(str(e))
    if how == "spawn":
        sys.exit(spawn_ranks(args.gpus))
    w = {**WORKLOADS, **DECODE_WORKLOADS, **BWD_WORKLOADS}[args.workload]
    if args.impl == "reference":
        # host-only: rank 0 times the oracle, other ranks exit without work
        world, rank = world_from_env()
        run_reference(args, w, world, rank)
        return
    world, rank, local = init_dist()
    try:
        (run_decode_cuda if is_decode(w) else run_backward_cuda if is_backward(w) else run_cuda)(
            args, w, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
