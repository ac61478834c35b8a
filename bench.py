#!/usr/bin/env python3
"""Benchmark of the quantized-gradient-aggregation hot path on B200.

One step = one pass of the error-feedback 2-bit path of the VGG16-sized
workload: each of W = 8 simulated workers quantizes its own n = 138,357,544
element fp32 gradient against its own residual (fused add / code / residual
update / pack, ``qga_quantize_2bit``), then the 8 packed streams are merged
into one fp32 aggregate (``qga_dequant_accumulate_2bit``).  Gradients are
seeded Laplace(0, 1e-3) draws, 5 iterations' worth resident in HBM and
cycled, residuals carried from step to step; thresholds +-2e-3.

``value`` is gradient elements aggregated per second over the whole job
(W * n per step per GPU), timed with CUDA events on the launching stream,
max over ranks.  Every buffer is larger than L2, so no flush is needed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qga|reference]

``--impl reference`` times the CPU oracle (single-threaded C) as it stands on
a bounded sample of the same workload.  Under torchrun with N > 1 each rank
runs its own replica (weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "2-bit quantize+residual+pack Gelem/s and HBM GB/s (% of peak), n=138M fp32"
WORKLOAD = "vgg16-8w"
QUANT_BYTES_PER_ELEM = 12.25        # read g 4 + read r 4 + write r 4 + write codes 0.25
FALLBACK_HBM_GBS = 6650.0
TS_PAIRS = ((4, 8), (2, 4))          # QSGD-MN-TS rows: (coarse bits, fine bits)

# dram__bytes_read.sum + dram__bytes_write.sum per element of one launch of
# the quantize kernel, captured at n = 34,589,386
# (profiles/quantize_2bit_kernel_fp32_vgg16.md) and scaled by elements to the
# full launch; keyed by the code hash of the sources that kernel is compiled
# from, and reported as null once they have changed since the capture.
MEASURED_TRAFFIC = {"a9972aea59c8a86c": 10.739}   # 1.486 GB per launch of n = 138,357,544
QUANT_SOURCES = ("qga_common.cuh", "qga_2bit_tiles.cuh", "qga_2bit.cu")

# ALU-pipe thread instructions per element (ncu sm__inst_executed_pipe_alu.sum
# x 32 / elements, captured at n = 2^25, profiles/row_kernels_quarter_size.md)
# of the integer-bound QSGD quantizers, keyed by the code hash of their
# sources; a row's "alu" object is null once the sources have changed.
QSGD_SOURCES = ("qga_common.cuh", "qga_qsgd_level.cuh", "qga_qsgd.cu")
TS_SOURCES = ("qga_common.cuh", "qga_qsgd_level.cuh", "qga_qsgd_ts.cu")
MEASURED_ALU = {
    "6043dbb4f8cc3ed9": {"b2": 12.78, "b4": 12.88, "b8": 13.58},
    "cec14726e428f3f1": {"b4_8": 23.03, "b2_4": 21.50},
}
ALU_CLOCK_MHZ = 1965.0   # clocks.max.sm of the B200


def alu_bound(instr_per_elem, elems, seconds, sms):
    """The ALU-pipe roofline of an integer-bound kernel: one warp-instruction
    every other cycle per SM sub-partition (4 per SM) at the maximum SM
    clock; returns the bound's time and the fraction of it achieved."""
    if instr_per_elem is None:
        return None
    per_s = sms * 4 * 0.5 * ALU_CLOCK_MHZ * 1e6   # warp-instructions per second
    bound = elems * instr_per_elem / 32 / per_s
    return {"alu_instr_per_elem": instr_per_elem, "bound_us": bound * 1e6, "frac": bound / seconds,
            "clock_mhz": ALU_CLOCK_MHZ, "sms": sms}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=300)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["qga", "reference"], default="qga")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--reduce-form", choices=["pair", "fused"], default="pair",
                   help="the reducing worker's step: quantize + merge (pair) or one fused launch")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-rows", action="store_true",
                   help="skip the per-kernel timings of the other hot-path rows")
    # smaller cases of the same step, for profiler captures (not bench lines)
    p.add_argument("--n", type=int, default=None, help="elements per worker (default: workload n)")
    p.add_argument("--iterations", type=int, default=None, help="resident gradient sets")
    p.add_argument("--rows-scale", type=int, default=1,
                   help="divide the per-row workloads' sizes by this (profiler captures)")
    p.add_argument("--rows-reps", type=int, default=20,
                   help="timed launches per row (1 with --rows-warmup 0: each row kernel once, "
                        "for profiler captures)")
    p.add_argument("--rows-warmup", type=int, default=3)
    return p.parse_args()


def _code_only(text):
    """C/C++ source without its comments and blank lines: the part that can
    change a kernel (string and character literals are kept as they are)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            i = text.find("\n", i)
            i = n if i < 0 else i
        elif text.startswith("/*", i):
            i = text.find("*/", i + 2)
            i = n if i < 0 else i + 2
        else:
            out.append(c)
            i += 1
    lines = [ln.rstrip() for ln in "".join(out).splitlines()]
    return "\n".join(ln for ln in lines if ln)


def csrc_hash(names=None):
    """Hash of the CUDA sources' code, comments excluded (all files, or the
    named ones): it changes exactly when a kernel may have changed."""
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "quantized_gradient_aggregation_b200", "csrc")
    paths = sorted(glob.glob(os.path.join(pkg, "*.cu*"))) if names is None else \
        [os.path.join(pkg, x) for x in names]
    for path in paths:
        with open(path, encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload_config(w, n_gpus, reduce_form="pair"):
    last = (f"then worker 0 (the reducing worker) quantizes its own gradient and all {w.workers} "
            "records are merged" + (" in one launch" if reduce_form == "fused" else ""))
    return {
        "workload": (f"{w.name}: W={w.workers} simulated workers x n={w.n:,} fp32, "
                     f"g~Laplace(0,{w.scale:g}) (seeded synthetic, {w.iterations} iterations "
                     f"resident and cycled), residual carried, thresholds {w.neg_thr:g}/{w.pos_thr:g}; "
                     f"step = quantize of workers 1..{w.workers - 1}, {last}"),
        "n": w.n,
        "workers": w.workers,
        "l2": "every buffer (553 MB per gradient) is larger than the 126 MB L2; no flush",
        "parallelism": f"replicas x{n_gpus} (weak scaling, no data-path collective)",
    }


# ------------------------------------------------------------- ranks ----

def max_over_ranks(values, world, device="cpu"):
    """Elementwise max of per-rank timings over all ranks (the slowest rank
    sets the job's time).  Every rank must call it, in the same order."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_gelem_per_s(world, workers, n, steps, ms):
    """Whole-job throughput: gradient elements of every simulated worker on
    every rank, over the slowest rank's time."""
    return world * workers * n * steps / (ms * 1e-3) / 1e9


# ------------------------------------------------------------ clocks ----

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_id):
        self.out = tempfile.TemporaryFile(mode="w+")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_id}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.seek(0)
        sm, smax, reasons, n = [], [], set(), 0
        for line in self.out:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            n += 1
            for name, flag in zip(self.REASONS, parts[5:9]):
                if flag.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": n}


def gpu_id_for(dev_index):
    import torch
    props = torch.cuda.get_device_properties(dev_index)
    uuid = getattr(props, "uuid", None)
    if uuid is not None:
        s = str(uuid)
        return s if s.startswith("GPU-") else "GPU-" + s
    return str(dev_index)


# ------------------------------------------------------------ oracle ----

def oracle_step_sample(n_s, seed=0):
    """Host inputs for a bounded sample of the workload (first n_s elements
    of each worker's gradient)."""
    import numpy as np
    import workloads
    w = workloads.WORKLOADS[WORKLOAD]
    grads = [workloads.gradient(w, k, 0, device="cpu", n=n_s).numpy() for k in range(w.workers)]
    res = [np.zeros(n_s, np.float32) for _ in range(w.workers)]
    return w, grads, res


def time_oracle(n_s, min_seconds, max_steps=None, warmup=0):
    """Oracle steps (W quantizes + 1 merge) on n_s elements per worker."""
    import oracle
    L = oracle.lib()
    w, grads, res = oracle_step_sample(n_s)
    ptrs = (ctypes.c_void_p * w.workers)()

    def step():
        recs = []
        for k in range(w.workers):
            c, res[k] = oracle.quantize_2bit(grads[k], res[k], w.neg_thr, w.pos_thr, L)
            recs.append(c)
        oracle.dequant_accumulate_2bit(recs, n_s, L)

    for _ in range(warmup):
        step()
    t0 = time.perf_counter()
    steps = 0
    while True:
        step()
        steps += 1
        el = time.perf_counter() - t0
        if (max_steps is not None and steps >= max_steps) or (max_steps is None and el >= min_seconds):
            break
    el = time.perf_counter() - t0
    del ptrs
    return steps, el, w


def cpu_baseline(n_s=1 << 24, min_seconds=10.0):
    steps, el, w = time_oracle(n_s, min_seconds)
    elems = steps * w.workers * n_s
    return {"value": elems / el / 1e9, "unit": "Gelem/s", "cores": 1, "kind": "oracle",
            "sample": (f"{steps} oracle steps of {w.workers} workers x {n_s:,} elements "
                       f"(first {n_s:,} of each worker's gradient) quantize + merge, "
                       f"{el:.1f} s single-threaded; host has {len(os.sched_getaffinity(0))} cores")}


def run_reference(args, rank, world):
    if rank != 0:
        return
    # per-step sample sized so the whole run stays near a minute (the oracle
    # takes about 15 ns per element per worker, merge included)
    budget_s = 60.0 / max(1, args.steps + args.warmup)
    n_s = int(min(1 << 22, max(1 << 14, budget_s / (8 * 15e-9)))) & ~15
    steps, el, w = time_oracle(n_s, 0.0, max_steps=args.steps, warmup=args.warmup)
    value = steps * w.workers * n_s / el / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "Gelem/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded Laplace draws)", "config": workload_config(w, args.gpus),
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "Gelem/s", "cores": 1, "kind": "oracle",
                         "sample": (f"each step: {w.workers} workers x first {n_s:,} elements of "
                                    "the workload, quantize + merge, single-threaded C oracle; host "
                                    f"has {len(os.sched_getaffinity(0))} cores")},
        "e2e": {"value": value, "unit": "Gelem/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------- GPU ----

def run_qga(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import quantized_gradient_aggregation_b200 as q
    import workloads

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = workloads.WORKLOADS[WORKLOAD]
    if args.n is not None or args.iterations is not None:
        import dataclasses
        w = dataclasses.replace(w, n=args.n or w.n, iterations=args.iterations or w.iterations,
                                name=w.name + "-reduced")
    n, W, iters = w.n, w.workers, w.iterations
    L = q.lib()

    grads = [[workloads.gradient(w, k, it, device=dev) for k in range(W)] for it in range(iters)]
    res = [torch.zeros(n, device=dev) for _ in range(W)]
    words = q.qga_2bit_words(n)
    comprs = [torch.empty(words, dtype=torch.int32, device=dev) for _ in range(W)]
    out = torch.empty(n, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    cptrs = (ctypes.c_void_p * W)(*[c.data_ptr() for c in comprs])
    cpp = ctypes.cast(cptrs, ctypes.POINTER(ctypes.c_void_p))
    neg, pos = w.neg_thr, w.pos_thr

    def quant(it, k):
        st = L.qga_quantize_2bit(ctypes.c_void_p(grads[it][k].data_ptr()),
                                 ctypes.c_void_p(res[k].data_ptr()),
                                 ctypes.c_void_p(comprs[k].data_ptr()), n, neg, pos, sp)
        if st:
            raise q.QGAError(st, "qga_quantize_2bit")

    def reduce_fused(it):
        # worker 0 is the reducing worker ([MX] Local kvstore): its own quantize
        # and the merge of all W records in one launch
        st = L.qga_quantize_merge_2bit(ctypes.c_void_p(grads[it][0].data_ptr()),
                                       ctypes.c_void_p(res[0].data_ptr()), n, neg, pos, cpp, W, 0,
                                       ctypes.c_void_p(out.data_ptr()), sp)
        if st:
            raise q.QGAError(st, "qga_quantize_merge_2bit")

    def reduce_pair(it):
        # the same results from two launches: worker 0's quantize, then the merge
        quant(it, 0)
        st = L.qga_dequant_accumulate_2bit(cpp, W, ctypes.c_void_p(out.data_ptr()), n, sp)
        if st:
            raise q.QGAError(st, "qga_dequant_accumulate_2bit")

    # The reducing worker's step (both forms give the same bits) is timed in
    # the form given by --reduce-form: by default the pair, measured faster on
    # B200 (391.6 against 404.4 us at n = 138M, W = 8).  Both forms are also
    # timed alone after the timed region and reported.
    reduce_form = args.reduce_form
    reduce = reduce_fused if reduce_form == "fused" else reduce_pair

    def barrier():
        if world > 1:
            dist.barrier()

    sampler = ClockSampler(gpu_id_for(local_rank))
    time.sleep(0.3)
    for s in range(args.warmup):
        for k in range(1, W):
            quant(s % iters, k)
        reduce(s % iters)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()

    K = args.steps
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    q_ev = [(ev(), ev()) for _ in range(K * (W - 1))]
    m_ev = [(ev(), ev()) for _ in range(K)]
    start, end = ev(), ev()
    start.record(stream)
    for s in range(K):
        it = (args.warmup + s) % iters
        for k in range(1, W):
            a, b = q_ev[s * (W - 1) + k - 1]
            a.record(stream)
            quant(it, k)
            b.record(stream)
        a, b = m_ev[s]
        a.record(stream)
        reduce(it)
        b.record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()

    total_ms = start.elapsed_time(end)
    quant_ms = statistics.fmean(a.elapsed_time(b) for a, b in q_ev)
    merge_ms = statistics.fmean(a.elapsed_time(b) for a, b in m_ev)
    total_ms, quant_ms, merge_ms = max_over_ranks([total_ms, quant_ms, merge_ms], world, dev)

    trial = {}
    for name, fn in (("fused", reduce_fused), ("pair", reduce_pair)):
        trial[name] = _time_launches(stream, lambda fn=fn: fn(0), 10, nvtx="reducing_worker_" + name) * 1e6
    e2e = None if args.no_e2e else run_e2e(args, w, grads[0], res, comprs, out, quant, reduce,
                                           stream, world, dev, reduce_form)
    del grads, res, comprs, out
    torch.cuda.empty_cache()
    rows = None if args.no_rows else time_rows(dev, stream, measured_peaks()[0], reps=args.rows_reps,
                                               scale=max(1, args.rows_scale), warmup=args.rows_warmup)

    if rank != 0:
        return
    peak, peak_kind = measured_peaks()
    quant_gbs = QUANT_BYTES_PER_ELEM * n / (quant_ms * 1e-3) / 1e9
    merge_gbs = (QUANT_BYTES_PER_ELEM + 0.25 * (W - 1) + 4) * n / (merge_ms * 1e-3) / 1e9
    traffic_per_elem = MEASURED_TRAFFIC.get(csrc_hash(QUANT_SOURCES))
    line = {
        "metric": METRIC,
        "value": job_gelem_per_s(world, W, n, K, total_ms),
        "unit": "Gelem/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": total_ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded Laplace(0,1e-3) gradients generated on the GPU)",
        "config": workload_config(w, world, reduce_form),
        "roofline": {"bound": "hbm", "kernel": "qga_quantize_2bit (quantize_2bit_words_kernel)",
                     "achieved": quant_gbs, "peak": peak, "unit": "GB/s", "frac": quant_gbs / peak,
                     "peak_source": f"{peak_kind} HBM copy rate",
                     "bytes_per_elem": QUANT_BYTES_PER_ELEM, "elems_per_launch": n,
                     "avg_launch_us": quant_ms * 1e3,
                     "traffic": None if traffic_per_elem is None else traffic_per_elem * n},
        "kernels": {
            "quantize_2bit": {"us": quant_ms * 1e3, "gelem_s": n / (quant_ms * 1e-3) / 1e9,
                              "gb_s": quant_gbs, "frac_of_peak": quant_gbs / peak,
                              "frac_of_8TBs": quant_gbs / 8000.0},
            "reducing_worker_step_w8": {"us": merge_ms * 1e3, "form": reduce_form,
                                       "gelem_s": n / (merge_ms * 1e-3) / 1e9,
                                       "gb_s": merge_gbs, "frac_of_peak": merge_gbs / peak,
                                       "frac_of_8TBs": merge_gbs / 8000.0,
                                       "bytes_per_elem": QUANT_BYTES_PER_ELEM + 0.25 * (W - 1) + 4},
        },
        "gpu_launches": K * (W + (reduce_form == "pair")),
        "reducing_worker_step": {"timed_form": reduce_form,
                                 "alone_us_after_timed_region": trial,
                                 "forms": {"fused": "qga_quantize_merge_2bit (one launch)",
                                           "pair": "qga_quantize_2bit + qga_dequant_accumulate_2bit"}},
        "clocks": clocks,
        "csrc": csrc_hash(),
        "quantize_sources": csrc_hash(QUANT_SOURCES),
    }
    if rows is not None:
        line["kernels"].update(rows)
        line["gpu_launches_rows"] = sum(r.get("launches", 0) for r in rows.values())
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)


def _time_launches(stream, fn, reps, warmup=3, nvtx="row"):
    """Average device time of fn() (one or more kernel launches) over reps,
    CUDA events on the launching stream.  The timed launches sit in an NVTX
    range named ``nvtx`` (a profiler can select them by it)."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push(nvtx)
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps * 1e-3


def _row(seconds, elems, bytes_per_elem, peak, launches, **extra):
    gbs = bytes_per_elem * elems / seconds / 1e9
    d = {"us": seconds * 1e6, "gelem_s": elems / seconds / 1e9, "gb_s": gbs,
         "bytes_per_elem": bytes_per_elem, "frac_of_peak": gbs / peak, "frac_of_8TBs": gbs / 8000.0,
         "launches": launches}
    d.update(extra)
    return d


def time_rows(dev, stream, peak, reps=20, scale=1, warmup=3):
    """Device time of every other row of the hot path, each on its own
    workload at full size (inputs resident, larger than L2); ``scale`` > 1
    shrinks the flat workloads for profiler captures only."""
    import torch

    import quantized_gradient_aggregation_b200 as q
    import workloads
    rows = {}
    L = q.lib()
    sp = ctypes.c_void_p(stream.cuda_stream)
    vp = ctypes.c_void_p

    def ok(st, name):
        if st:
            raise q.QGAError(st, name)

    # dequantize of one VGG16-sized record
    w = workloads.WORKLOADS[WORKLOAD]
    n = w.n // scale
    g = workloads.gradient(w, 0, 0, device=dev, n=n)
    r = torch.zeros(n, device=dev)
    c = torch.empty(q.qga_2bit_words(n), dtype=torch.int32, device=dev)
    q.qga_quantize_2bit(g, r, c, w.neg_thr, w.pos_thr)
    out = torch.empty(n, device=dev)
    t = _time_launches(stream, lambda: ok(L.qga_dequantize_2bit(vp(c.data_ptr()), vp(out.data_ptr()),
                                                                n, sp), "dequantize"), reps, warmup)
    rows["dequantize_2bit"] = _row(t, n, 4.25, peak, reps + warmup, workload=f"vgg16 record, n={n:,}")

    # the reducing worker's fused step: quantize worker 0, merge 8 records
    # (the other workers' records from their own gradients)
    others = []
    for k in range(1, w.workers):
        gk = workloads.gradient(w, k, 0, device=dev, n=n)
        rk = torch.zeros(n, device=dev)
        ck = torch.empty_like(c)
        q.qga_quantize_2bit(gk, rk, ck, w.neg_thr, w.pos_thr)
        others.append(ck)
        del gk, rk
    c_own = torch.empty_like(c)
    rarr = (ctypes.c_void_p * w.workers)(*[x.data_ptr() for x in [c_own] + others])
    rp = ctypes.cast(rarr, ctypes.POINTER(ctypes.c_void_p))
    t = _time_launches(stream, lambda: ok(L.qga_quantize_merge_2bit(
        vp(g.data_ptr()), vp(r.data_ptr()), n, w.neg_thr, w.pos_thr, rp, w.workers, 0,
        vp(out.data_ptr()), sp), "quantize_merge"), reps, warmup)
    rows["quantize_merge_2bit_w8_alone"] = _row(t, n, 12.25 + 0.25 * (w.workers - 1) + 4, peak,
                                                reps + warmup,
                                                workload=f"vgg16 worker 0 + 7 received records, n={n:,}")
    # the merge alone (A8): 8 records
    t = _time_launches(stream, lambda: ok(L.qga_dequant_accumulate_2bit(
        rp, w.workers, vp(out.data_ptr()), n, sp), "merge"), reps, warmup)
    rows["dequant_accumulate_2bit_w8"] = _row(t, n, 0.25 * w.workers + 4, peak, reps + warmup,
                                              workload=f"8 records of n={n:,}")
    del c, others, c_own

    # dense ternary records (5 codes per byte): quantize and the 8-worker merge
    ct = [torch.empty(q.qga_ternary_words(n), dtype=torch.int32, device=dev) for _ in range(w.workers)]
    t = _time_launches(stream, lambda: ok(L.qga_quantize_ternary(
        vp(g.data_ptr()), vp(r.data_ptr()), vp(ct[0].data_ptr()), n, w.neg_thr, w.pos_thr, sp),
        "quantize_ternary"), reps, warmup)
    rows["quantize_ternary"] = _row(t, n, 12.2, peak, reps + warmup, workload=f"vgg16 gradient, n={n:,}")
    for k in range(1, w.workers):
        gk = workloads.gradient(w, k, 0, device=dev, n=n)
        rk = torch.zeros(n, device=dev)
        q.qga_quantize_ternary(gk, rk, ct[k], w.neg_thr, w.pos_thr)
        del gk, rk
    tarr = (ctypes.c_void_p * w.workers)(*[cc.data_ptr() for cc in ct])
    tp = ctypes.cast(tarr, ctypes.POINTER(ctypes.c_void_p))
    t = _time_launches(stream, lambda: ok(L.qga_dequant_accumulate_ternary(
        tp, w.workers, vp(out.data_ptr()), n, sp), "merge_ternary"), reps, warmup)
    rows["dequant_accumulate_ternary_w8"] = _row(t, n, 0.2 * w.workers + 4, peak, reps + warmup,
                                                 workload=f"8 dense records of n={n:,}")
    del g, r, out, ct

    # BERT-Base bucket: quantize (bf16 grad) and 4-worker merge
    wb = workloads.WORKLOADS["bert-bucket-4w"]
    sizes = workloads.bert_base_sizes()
    total = sum(sizes)
    words = q.qga_2bit_bucket_words(sizes)
    comprs, tables, keep = [], [], []
    neg = pos = None
    for k in range(wb.workers):
        grads = workloads.bert_bucket(wb, k, 0, device=dev)
        if neg is None:
            neg, pos = workloads.bert_thresholds(grads)
        res = [torch.zeros(s, device=dev) for s in sizes]
        tables.append(q.make_bucket_table(grads, res, neg, pos))
        keep.append((grads, res))
        comprs.append(torch.empty(words, dtype=torch.int32, device=dev))
    T = len(sizes)

    def quant_bucket(k=0):
        ok(L.qga_quantize_2bit_bucket(tables[k], T, q.QGA_DTYPE_BF16, vp(comprs[k].data_ptr()), sp),
           "quantize_bucket")
    for k in range(wb.workers):
        quant_bucket(k)
    t = _time_launches(stream, quant_bucket, reps, warmup)
    rows["quantize_2bit_bucket_bf16"] = _row(t, total, 10.25, peak, reps + warmup + wb.workers,
                                             workload="BERT-Base bucket, 197 bf16 tensors, "
                                                      "109,480,704 elements")
    out = torch.empty(total, device=dev)
    arr = (ctypes.c_void_p * wb.workers)(*[cc.data_ptr() for cc in comprs])
    pp = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    nn = (ctypes.c_int64 * T)(*sizes)
    t = _time_launches(stream, lambda: ok(L.qga_dequant_accumulate_2bit_bucket(
        pp, wb.workers, nn, T, vp(out.data_ptr()), sp), "merge_bucket"), reps, warmup)
    rows["dequant_accumulate_2bit_bucket_w4"] = _row(t, total, 0.25 * wb.workers + 4, peak, reps + warmup,
                                                     workload="BERT-Base bucket, 4 workers")
    del keep, comprs, out, tables

    # the single-tensor bf16 quantize on one flat gradient of the bucket's size
    gb = workloads.normal(total, wb.scale, torch.Generator(device=dev).manual_seed(7), dev,
                          dtype=torch.bfloat16)
    rb = torch.zeros(total, device=dev)
    cb = torch.empty(q.qga_2bit_words(total), dtype=torch.int32, device=dev)
    t = _time_launches(stream, lambda: ok(L.qga_quantize_2bit_bf16(
        vp(gb.data_ptr()), vp(rb.data_ptr()), vp(cb.data_ptr()), total, neg[0], pos[0], sp),
        "quantize_bf16"), reps, warmup)
    rows["quantize_2bit_bf16"] = _row(t, total, 10.25, peak, reps + warmup,
                                      workload=f"one flat bf16 gradient, n={total:,}")
    del gb, rb, cb

    # QSGD-MaxNorm: max over 8 workers, quantize per b, merge of 8
    wq = workloads.WORKLOADS["qsgd-128M-8w"]
    nq, Wq = wq.n // scale, wq.workers
    grads = [workloads.gradient(wq, k, 0, device=dev, n=nq) for k in range(Wq)]
    M = torch.empty(1, device=dev)
    garr = (ctypes.c_void_p * Wq)(*[gg.data_ptr() for gg in grads])
    gp = ctypes.cast(garr, ctypes.POINTER(ctypes.c_void_p))
    t = _time_launches(stream, lambda: ok(L.qga_qsgd_mn_max(gp, Wq, nq, vp(M.data_ptr()), sp),
                                          "qsgd_max"), reps, warmup)
    rows["qsgd_mn_max_w8"] = _row(t, nq * Wq, 4.0, peak, reps + warmup,
                                  workload=f"8 x {nq:,} fp32 (0.1% outliers of 50)")
    out = torch.empty(nq, device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    alu_q = MEASURED_ALU.get(csrc_hash(QSGD_SOURCES), {})
    alu_ts = MEASURED_ALU.get(csrc_hash(TS_SOURCES), {})
    for b in wq.bits:
        cq = [torch.empty(q.qga_qsgd_words(nq, b), dtype=torch.int32, device=dev) for _ in range(Wq)]

        def quant_q(k=0, b=b, cq=cq):
            ok(L.qga_qsgd_mn_quantize(vp(grads[k].data_ptr()), vp(cq[k].data_ptr()), nq, b,
                                      workloads.QSGD_SEED_BASE + k, vp(M.data_ptr()), sp),
               "qsgd_quantize")
        for k in range(Wq):
            quant_q(k)
        t = _time_launches(stream, quant_q, reps, warmup)
        rows[f"qsgd_mn_quantize_b{b}"] = _row(t, nq, 4 + b / 8, peak, reps + warmup + Wq,
                                              workload=f"{nq:,} fp32, b={b}",
                                              alu=alu_bound(alu_q.get(f"b{b}"), nq, t, sms))
        carr = (ctypes.c_void_p * Wq)(*[cc.data_ptr() for cc in cq])
        cp = ctypes.cast(carr, ctypes.POINTER(ctypes.c_void_p))
        t = _time_launches(stream, lambda: ok(L.qga_qsgd_mn_dequant_accumulate(
            cp, Wq, vp(out.data_ptr()), nq, b, sp), "qsgd_merge"), reps, warmup)
        rows[f"qsgd_mn_dequant_accumulate_b{b}_w8"] = _row(t, nq, Wq * b / 8 + 4, peak, reps + warmup,
                                                          workload=f"8 records of {nq:,}, b={b}")
        del cq

    # QSGD-MN-TS: coarse scale M with b1 bits, fine scale M / s1 with b2 bits
    for b1, b2 in TS_PAIRS:
        words = q.qga_qsgd_mnts_words(nq, b1, b2)
        ct = [torch.empty(words, dtype=torch.int32, device=dev) for _ in range(Wq)]

        def quant_ts(k=0, b1=b1, b2=b2, ct=ct):
            ok(L.qga_qsgd_mnts_quantize(vp(grads[k].data_ptr()), vp(ct[k].data_ptr()), nq, b1, b2,
                                        workloads.QSGD_SEED_BASE + k, vp(M.data_ptr()), sp),
               "qsgd_mnts_quantize")
        for k in range(Wq):
            quant_ts(k)
        t = _time_launches(stream, quant_ts, reps, warmup)
        rows[f"qsgd_mnts_quantize_b{b1}_{b2}"] = _row(t, nq, 4 + (b1 + b2) / 8, peak, reps + warmup + Wq,
                                                      workload=f"{nq:,} fp32, b1={b1}, b2={b2}",
                                                      alu=alu_bound(alu_ts.get(f"b{b1}_{b2}"), nq, t, sms))
        carr = (ctypes.c_void_p * Wq)(*[cc.data_ptr() for cc in ct])
        cp = ctypes.cast(carr, ctypes.POINTER(ctypes.c_void_p))
        t = _time_launches(stream, lambda: ok(L.qga_qsgd_mnts_dequant_accumulate(
            cp, Wq, vp(out.data_ptr()), nq, b1, b2, sp), "qsgd_mnts_merge"), reps, warmup)
        rows[f"qsgd_mnts_dequant_accumulate_b{b1}_{b2}_w8"] = _row(
            t, nq, Wq * (b1 + b2) / 8 + 4, peak, reps + warmup, workload=f"8 records of {nq:,}, b1={b1}, b2={b2}")
        del ct

    # GRandK-MaxNorm: the same gradients, K = 10000 shared coordinates
    K = workloads.GRANDK_K
    index = torch.from_numpy(workloads.grandk_index(nq, K)).to(dev)
    ip = vp(index.data_ptr())
    t = _time_launches(stream, lambda: ok(L.qga_grandk_mn_max(gp, Wq, nq, ip, K, vp(M.data_ptr()), sp),
                                          "grandk_max"), reps, warmup)
    rows["grandk_mn_max_w8"] = _row(t, K * Wq, 4.0, peak, reps + warmup, bound="latency",
                                    workload=f"8 x {nq:,} fp32, K = {K:,} kept coordinates")
    for b in wq.bits:
        ck = [torch.empty(q.qga_qsgd_words(K, b), dtype=torch.int32, device=dev) for _ in range(Wq)]

        def quant_k(k=0, b=b, ck=ck):
            ok(L.qga_grandk_mn_quantize(vp(grads[k].data_ptr()), nq, ip, K, vp(ck[k].data_ptr()), b,
                                        workloads.QSGD_SEED_BASE + k, vp(M.data_ptr()), sp),
               "grandk_quantize")
        for k in range(Wq):
            quant_k(k)
        t = _time_launches(stream, quant_k, reps, warmup)
        rows[f"grandk_mn_quantize_b{b}"] = _row(t, K, 4 + 8 + b / 8, peak, reps + warmup + Wq,
                                                bound="latency", workload=f"K = {K:,} of {nq:,}, b={b}")
        carr = (ctypes.c_void_p * Wq)(*[cc.data_ptr() for cc in ck])
        cp = ctypes.cast(carr, ctypes.POINTER(ctypes.c_void_p))
        # the merge clears the n-element result (cudaMemsetAsync), then scatters K values
        t = _time_launches(stream, lambda: ok(L.qga_grandk_mn_dequant_accumulate(
            cp, Wq, ip, K, vp(out.data_ptr()), nq, b, sp), "grandk_merge"), reps, warmup)
        rows[f"grandk_mn_dequant_accumulate_b{b}_w8"] = _row(
            t, nq, 4 + (K * (8 + 4 + Wq * b / 8)) / nq, peak, reps + warmup, bound="hbm (clear of out)",
            workload=f"8 records of K = {K:,}, out of {nq:,}")
        del ck
    del grads, out, index
    torch.cuda.empty_cache()
    return rows


def run_e2e(args, w, dev_grads, res, comprs, out, quant, reduce, stream, world, dev, reduce_form):
    """Same step with the gradients arriving from pinned host memory and the
    aggregate read back, copies inside the timed region.  Uploads run on one
    copy stream, so worker k's upload overlaps the quantize of the worker
    before it; the aggregate's download runs on another, so that it overlaps
    the next step's uploads (PCIe carries both directions at once).  Events
    order every reuse of a buffer.  Worker 0, the reducing worker, comes
    last: its quantize and the merge are one launch."""
    import torch
    n, W = w.n, w.workers
    host = [torch.empty(n, dtype=torch.float32, pin_memory=True) for _ in range(W)]
    for k in range(W):
        host[k].copy_(dev_grads[k], non_blocking=False)
    host_out = torch.empty(n, dtype=torch.float32, pin_memory=True)
    copy_stream = torch.cuda.Stream(device=dev)
    down_stream = torch.cuda.Stream(device=dev)
    K = max(3, min(args.steps, 10))
    landed = [torch.cuda.Event() for _ in range(W)]
    consumed = [torch.cuda.Event() for _ in range(W)]
    merged = torch.cuda.Event()
    downloaded = torch.cuda.Event()
    for e in consumed:
        e.record(stream)
    downloaded.record(stream)

    def step():
        for k in list(range(1, W)) + [0]:
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(consumed[k])      # previous quantize of worker k is done
                dev_grads[k].copy_(host[k], non_blocking=True)
                landed[k].record(copy_stream)
            stream.wait_event(landed[k])
            if k:
                quant(0, k)
            else:
                stream.wait_event(downloaded)            # previous aggregate has left the device
                reduce(0)
                merged.record(stream)
            consumed[k].record(stream)
        with torch.cuda.stream(down_stream):
            down_stream.wait_event(merged)
            host_out.copy_(out, non_blocking=True)
            downloaded.record(down_stream)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    copy_stream.wait_event(a)
    for _ in range(K):
        step()
    stream.wait_event(downloaded)
    b.record(stream)
    torch.cuda.synchronize()
    (ms,) = max_over_ranks([a.elapsed_time(b)], world, dev)
    return {"value": job_gelem_per_s(world, W, n, K, ms), "unit": "Gelem/s",
            "h2d_bytes_per_step": W * n * 4, "d2h_bytes_per_step": n * 4, "steps": K,
            "path": ("pinned host gradients -> cudaMemcpyAsync (copy stream) -> qga_quantize_2bit x7 -> "
                     + ("qga_quantize_2bit + qga_dequant_accumulate_2bit" if reduce_form == "pair"
                        else "qga_quantize_merge_2bit") + " (worker 0) -> pinned host aggregate (download stream)")}


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_qga(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
