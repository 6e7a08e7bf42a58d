#!/usr/bin/env python
"""Benchmark of the QLoRA linear layer on B200.

One step = the whole hot path over one batch of synthetic input, for every
projection of the workload: blockwise NF4 quantisation with double
quantisation of W0, the fused forward (Y = X W^T + s X A^T B^T, W rebuilt in
shared memory) and the backward (dX, dA, dB).  With several ranks each rank
runs the layer set on its own token batch (data parallel, weak scaling) and the
adapter gradients dA, dB are summed over ranks with NCCL, as a data-parallel
training step would.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints one JSON line on rank 0.  `value` is the fwd+bwd TFLOP/s of the whole
job (algorithmic flops 4Mdk + 6Mr(d+k) per projection, summed over ranks,
divided by the device time of K steps, max over ranks).  `--impl reference`
times the CPU oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from bit_quantized_lora_02_b200 import synth  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# workload arithmetic
# ---------------------------------------------------------------------------
def flops_fwd(M, d, k, r):
    return 2 * M * d * k + 2 * M * r * (d + k)


def flops_bwd(M, d, k, r):
    return 2 * M * d * k + 4 * M * r * (d + k)


def main_fwd_flops(M, d, k, r):      # the fused forward GEMM: X W^T + T_s B^T
    return 2 * M * d * k + 2 * M * d * r


def main_bwd_flops(M, d, k, r):      # the fused backward GEMM: dY W + U_s A
    return 2 * M * d * k + 2 * M * k * r


def nf4_bytes(d, k):
    n = d * k
    nb = -(-n // 64)
    return (n + 1) // 2 + nb + 4 * (-(-nb // 256)) + 4


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _code_only(src):
    """Source text without comments and blank or trailing space, so that a
    comment edit does not count as a kernel change."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def kernel_source_hash():
    """Hash of the code the many-token GEMM kernels are built from (the
    kernels whose DRAM traffic profiles/traffic_*.txt records)."""
    h = hashlib.sha256()
    for name in ("qlora_gemm.cu", "qlora_device.cuh", "qlora_internal.h", "nf4_scale.cuh", "nf4_table.h"):
        with open(os.path.join(ROOT, "bit_quantized_lora_02_b200", "csrc", name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def read_traffic(kernel_class, workload):
    """DRAM bytes per launch from the committed ncu summary for this kernel
    class and workload, or None when there is none or the kernel sources
    changed since those counters were taken."""
    p = os.path.join(ROOT, "profiles", f"traffic_{kernel_class}_{workload}.txt")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            if "=" in line and not line.startswith("#"):
                key, v = line.split("=", 1)
                vals[key.strip()] = v.strip()
    if vals.get("source_hash") != kernel_source_hash():
        return None
    try:
        return float(vals["bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for rec in csv.reader(io.StringIO(out)):
            if len(rec) < 10:
                continue
            rec = [x.strip() for x in rec]
            try:
                ts = time.mktime(time.strptime(rec[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                frac = float("0." + rec[0].split(".")[1]) if "." in rec[0] else 0.0
                rows.append((ts + frac, float(rec[2]), float(rec[3]), rec[6:10]))
            except (ValueError, IndexError):
                continue
        inside = [r for r in rows if self.t0 is not None and self.t0 - 0.06 <= r[0] <= self.t1 + 0.06]
        use = inside or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median([r[1] for r in use]) if use else None,
                "sm_max_mhz": max(r[2] for r in use) if use else None,
                "reasons": reasons, "samples": len(use), "samples_in_window": len(inside)}


# ---------------------------------------------------------------------------
# CPU oracle sample (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
class OracleSample:
    """The CPU oracle on frac^2 of one step, with the step's mix of work: per
    projection it quantises and reconstructs frac^2 of W0's rows (NF4 + double
    quantisation + dequantisation) and runs the fp64 forward+backward of frac of
    the tokens against frac of the output rows (frac^2 of the flops).  Only the
    work actually done is credited, so the rate is the oracle's own, and the
    host time stays bounded on the largest workloads."""

    def __init__(self, work, frac=0.125):
        from oracle import qlora_oracle as O
        self.O = O
        self.M, self.r, self.alpha = work["m"], work["r"], work["alpha"]
        self.p = work.get("dropout", 0.0)
        self.frac = frac
        self.Ms = max(1, int(self.M * frac))
        self.prepared = []
        for pi, (name, d, k) in enumerate(work["proj"]):
            rows = max(1, int(d * frac))                 # output rows of the fwd+bwd sample
            qrows = max(1, int(d * frac * frac))         # rows quantised inside the timed region
            W0 = synth.weight(d, k, seed=pi)[:rows].copy()
            What = O.dequantize_tensor(O.quantize_tensor(W0.reshape(-1), True)).reshape(rows, k)
            dY = synth.grad_output(self.Ms, d, pi)[:, :rows].copy()
            B = synth.lora_b(d, self.r, pi)[:rows].copy()
            self.prepared.append((rows, k, W0[:qrows].copy(), What, synth.activations(self.Ms, k, pi), dY,
                                  synth.lora_a(self.r, k, pi), B))
        self.desc = (f"{frac * frac:g} of one step: per projection NF4+DQ quantise/dequantise of {frac * frac:g} of "
                     f"W0's rows, fp64 fwd+bwd of {self.Ms} of {self.M} tokens against {frac:g} of the output rows "
                     f"(numpy)")

    def run(self):
        """Returns (seconds, credited fwd+bwd flops)."""
        O, r, alpha = self.O, self.r, self.alpha
        t0 = time.perf_counter()
        flops = 0.0
        for pi, (rows, k, W0q, What, X, dY, A, B) in enumerate(self.prepared):
            O.dequantize_tensor(O.quantize_tensor(W0q.reshape(-1), True))
            if self.p:
                keep = O.dropout_keep(self.Ms, k, self.p, 1234, pi)
                O.qlora_forward_dropout(X, What, A, B, alpha, r, keep, self.p)
                O.qlora_backward_dropout(dY, X, What, A, B, alpha, r, keep, self.p)
            else:
                O.qlora_forward(X, What, A, B, alpha, r)
                O.qlora_backward(dY, X, What, A, B, alpha, r)
            flops += flops_fwd(self.Ms, rows, k, r) + flops_bwd(self.Ms, rows, k, r)
        return time.perf_counter() - t0, flops


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_ours(args, work, wl_name):
    import torch
    import torch.distributed as dist

    import bit_quantized_lora_02_b200 as Q

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from bit_quantized_lora_02_b200.dp import GradBucket, max_over_ranks as dp_max

    M, r, alpha = work["m"], work["r"], work["alpha"]
    projs = work["proj"]
    drop_p = work.get("dropout", 0.0)
    step_no = [0]          # the dropout generator's offset: a new mask every step (and projection)
    # Units of the step: a single projection, or (grouped workloads) the
    # projections that share X (q, k, v; gate, up), run as one grouped layer.
    units = work.get("groups") or [[pi] for pi in range(len(projs))]
    # adapter gradients of every projection in one flat fp32 bucket (one all-reduce per step)
    shapes = []
    for u in units:
        k = projs[u[0]][2]
        shapes += [(len(u) * r, k), (sum(projs[pi][1] for pi in u), r)]
    bucket = GradBucket(shapes, dev)
    bufs = []
    h2d_bytes = d2h_bytes = 0
    for ui, u in enumerate(units):
        p0 = u[0]
        ds = [projs[pi][1] for pi in u]
        d, k = sum(ds), projs[p0][2]
        tok_seed = p0 + 1000 * rank         # each rank has its own token batch
        host = {"A": np.concatenate([synth.lora_a(r, k, seed=pi) for pi in u]),
                "B": np.concatenate([synth.lora_b(projs[pi][1], r, seed=pi) for pi in u]),
                "X": synth.activations(M, k, seed=tok_seed), "dY": synth.grad_output(M, d, seed=tok_seed)}
        for j, pi in enumerate(u):
            host[f"W0_{j}"] = synth.weight(projs[pi][1], k, seed=pi)
        b = {"d": d, "k": k, "name": "+".join(projs[pi][0] for pi in u), "n": len(u)}
        for key, arr in host.items():
            pinned = torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16).pin_memory()
            b["h_" + key] = pinned
            b[key] = pinned.to(dev, non_blocking=True)
            h2d_bytes += pinned.numel() * 2
        if len(u) > 1:
            b["g"] = Q.nf4_alloc_group(ds, k, True, dev)
            b["qparts"] = b["g"].parts
        else:
            b["q"] = Q.nf4_alloc(d, k, True, dev)
            b["qparts"] = [b["q"]]
        b["qws"] = torch.empty(max(max(Q.qlora_nf4_sizes(x, k, 64, True)[1] for x in ds), 16), dtype=torch.uint8,
                               device=dev)
        b["Y"] = torch.empty(M, d, dtype=torch.bfloat16, device=dev)
        b["T"] = torch.empty(M, Q.qlora_rank_pad(len(u) * r), dtype=torch.bfloat16, device=dev)
        b["dX"] = torch.empty(M, k, dtype=torch.bfloat16, device=dev)
        b["dA"] = bucket.views[2 * ui]
        b["dB"] = bucket.views[2 * ui + 1]
        if len(u) > 1:
            nws = max(Q.qlora_grouped_workspace_size(M, b["g"], r, False),
                      Q.qlora_grouped_workspace_size(M, b["g"], r, True))
        else:
            wsz = Q.qlora_linear_dropout_workspace_size if drop_p else Q.qlora_linear_workspace_size
            nws = max(wsz(M, d, k, r, False), wsz(M, d, k, r, True))
        b["ws"] = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
        for key in ("Y", "dX", "dA", "dB"):
            b["h_" + key] = torch.empty(b[key].shape, dtype=b[key].dtype, pin_memory=True)
            d2h_bytes += b[key].numel() * b[key].element_size()
        bufs.append(b)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def unit_step(ui, b):
        drop = (drop_p, 1234 + rank, step_no[0] * len(bufs) + ui) if drop_p else None
        for j, part in enumerate(b["qparts"]):
            Q.nf4_quantize(b[f"W0_{j}"], True, out=part, workspace=b["qws"], stream=stream)
        if b["n"] > 1:
            Q.qlora_linear_fwd_grouped(b["X"], b["g"], b["A"], b["B"], alpha, r=r, Y=b["Y"], T_save=b["T"],
                                       workspace=b["ws"], stream=stream)
            Q.qlora_linear_bwd_grouped(b["dY"], b["X"], b["g"], b["A"], b["B"], alpha, r=r, T_save=b["T"],
                                       dX=b["dX"], dA=b["dA"], dB=b["dB"], workspace=b["ws"], stream=stream)
        else:
            Q.qlora_linear_fwd(b["X"], b["q"], b["A"], b["B"], alpha, Y=b["Y"], T_save=b["T"],
                               workspace=b["ws"], stream=stream, dropout=drop)
            Q.qlora_linear_bwd(b["dY"], b["X"], b["q"], b["A"], b["B"], alpha, T_save=b["T"], dX=b["dX"],
                               dA=b["dA"], dB=b["dB"], workspace=b["ws"], stream=stream, dropout=drop)

    def step():
        for ui, b in enumerate(bufs):
            unit_step(ui, b)
        step_no[0] += 1
        if world > 1:
            bucket.allreduce()

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return dp_max(x, dev)

    # correctness guard before timing: the device status word must be clean
    step()
    torch.cuda.synchronize()
    assert Q.qlora_device_status() == 0

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)

    def timed_steps():
        barrier()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(ev0.elapsed_time(ev1))

    # the headline: K steps with nothing but the library's launches in the stream
    clocks.mark("t0")
    ms_total = timed_steps()
    # the same K steps again with an event pair around every launch, for the
    # per-kernel breakdown and the roofline of the dominant kernel
    Q.qlora_profile_read()                  # reset launch counters
    Q.qlora_profile_enable(True)
    ms_profiled = timed_steps()
    Q.qlora_profile_enable(False)
    clocks.mark("t1")
    clk = clocks.stop()
    kms, klaunch = Q.qlora_profile_read()
    ms_step = ms_total / args.steps
    assert Q.qlora_device_status() == 0

    step_flops = sum(flops_fwd(M, d, k, r) + flops_bwd(M, d, k, r) for _, d, k in projs)
    value = world * step_flops / (ms_step * 1e-3) / 1e12

    # End to end through the public API with host buffers.  Copies run on
    # their own streams so that they overlap the layer's kernels: unit i's
    # inputs go up while unit i-1 computes, and its Y, dX come down while unit
    # i+1 computes (both directions of the link at once); the adapter
    # gradients come down after the step's all-reduce.  A unit's input
    # buffers are refilled only after its kernels of the previous step have
    # read them, and its outputs are rewritten only after they came down.
    e2e_steps = max(1, min(args.steps, 5))
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    n_units = len(bufs)
    used = [None] * n_units          # compute of unit i (previous step) finished with its inputs
    fetched = [None] * n_units       # unit i's outputs (previous step) are on the host
    bucket_fetched = [None]

    def ev(st):
        e = torch.cuda.Event()
        e.record(st)
        return e

    def step_e2e():
        for ui, b in enumerate(bufs):
            with torch.cuda.stream(s_in):
                if used[ui] is not None:
                    s_in.wait_event(used[ui])
                for key in b:
                    if key.startswith("h_") and key[2:] in ("A", "B", "X", "dY") or key.startswith("h_W0_"):
                        b[key[2:]].copy_(b[key], non_blocking=True)
                ready = ev(s_in)
            stream.wait_event(ready)
            if fetched[ui] is not None:
                stream.wait_event(fetched[ui])
            if ui == 0 and bucket_fetched[0] is not None:
                stream.wait_event(bucket_fetched[0])
            unit_step(ui, b)
            used[ui] = ev(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(used[ui])
                for key in ("Y", "dX"):
                    b["h_" + key].copy_(b[key], non_blocking=True)
                fetched[ui] = ev(s_out)
        step_no[0] += 1
        if world > 1:
            bucket.allreduce()
        reduced = ev(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(reduced)
            for b in bufs:
                for key in ("dA", "dB"):
                    b["h_" + key].copy_(b[key], non_blocking=True)
            bucket_fetched[0] = ev(s_out)

    step_e2e()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for _ in range(e2e_steps):
        step_e2e()
    stream.wait_event(ev(s_in))
    stream.wait_event(ev(s_out))
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1)) / e2e_steps
    e2e_value = world * step_flops / (e2e_ms * 1e-3) / 1e12

    # roofline of the dominant kernel (device time over the timed region)
    peaks, peaks_src = load_peaks()
    algo = {
        "fwd_gemm": sum(main_fwd_flops(M, d, k, r) for _, d, k in projs) * args.steps,
        "bwd_gemm": sum(main_bwd_flops(M, d, k, r) for _, d, k in projs) * args.steps,
    }
    dom = max(kms, key=lambda c: kms[c])
    roofline = None
    if dom in algo and kms[dom] > 0:
        achieved = algo[dom] / (kms[dom] * 1e-3) / 1e12
        # the timed region lasts about a second at full clocks, so the burst
        # figure is the denominator; the sustained one is given beside it
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        sustained = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        launches = max(klaunch[dom], 1)
        traffic = read_traffic(dom, wl_name)
        roofline = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                    "peak_source": f"{peaks_src} bf16 dense, burst",
                    "frac_of_sustained": round(achieved / sustained, 4),
                    "traffic": traffic, "launches": klaunch[dom],
                    "avg_launch_ms": round(kms[dom] / launches, 4)}

    result = {
        "metric": "QLoRA linear fwd+bwd TFLOP/s (NF4 double-quant base, LoRA adapters), step = quantize+fwd+bwd",
        "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded numpy: W0~N(0,0.02), A~N(0,1/r), B~N(0,0.01), X,dY~N(0,1))",
        "config": {"workload": wl_name, "tokens_per_rank": M, "rank": r, "alpha": alpha,
                   "projections": [f"{n}:{d}x{k}" for n, d, k in projs], "nf4_blocksize": 64,
                   "double_quant": True, "lora_dropout": drop_p,
                   "grouped": [[projs[pi][0] for pi in u] for u in units if len(u) > 1],
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "l2": "working set per step larger than L2 (no explicit flush)"},
        "breakdown_ms_per_step": {c: round(v / args.steps, 4) for c, v in kms.items()},
        "profiled_ms_per_step": round(ms_profiled / args.steps, 4),
        "gpu_launches": int(sum(klaunch.values())),
        "roofline": roofline,
        "clocks": clk,
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 3),
                "copies": "host-to-device and device-to-host on their own streams, overlapping the kernels",
                "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = OracleSample(work)
        dt, fl, reps = 0.0, 0.0, 0
        while reps == 0 or dt < 10.0:      # about 10 s of host work, at least one sample
            t, f = sample.run()
            dt, fl, reps = dt + t, fl + f, reps + 1
        result["cpu_baseline"] = {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cpu_cores(),
                                  "kind": "oracle", "sample": f"{reps} x ({sample.desc})", "seconds": round(dt, 3)}
    if rank == 0 and world == 1 and not args.no_secondary:
        # the weight-bound and quantisation workloads, timed call by call (L2
        # flushed in between) in the same run, so the line carries them too
        del bufs, bucket
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        result["secondary"] = {}
        for wl in ("decode_28672x8192", "quant_sweep"):
            sec = secondary_results(args, wl, iters=5)
            result["secondary"][wl] = {"metric": sec["metric"], "value": sec["value"], "unit": sec["unit"],
                                       "results": sec["results"]}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def run_reference(args, work, wl_name):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    sample = OracleSample(work)
    desc = sample.desc
    times, fl = [], 0.0
    for i in range(args.warmup + args.steps):
        dt, fl = sample.run()
        if i >= args.warmup:
            times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = fl / (ms * 1e-3) / 1e12
    result = {
        "impl": "reference",
        "metric": "QLoRA linear fwd+bwd TFLOP/s (NF4 double-quant base, LoRA adapters), step = quantize+fwd+bwd",
        "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy)",
        "config": {"workload": wl_name, "tokens_per_rank": work["m"], "rank": work["r"], "alpha": work["alpha"],
                   "projections": [f"{n}:{d}x{k}" for n, d, k in work["proj"]], "sample": desc},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


# ---------------------------------------------------------------------------
# secondary workloads (not the default line): decode-like forward and the
# quantisation sweep, each timed kernel by kernel with L2 flushed in between
# ---------------------------------------------------------------------------
def _timed(fn, iters, flush, stream):
    """Median device ms of fn() over `iters` runs; `flush` (outside the
    events) evicts L2 before each run."""
    import torch
    times = []
    for _ in range(iters):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def run_secondary(args, wl_name):
    print(json.dumps(secondary_results(args, wl_name)), flush=True)


def secondary_results(args, wl_name, iters=None):
    import torch

    import bit_quantized_lora_02_b200 as Q
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks, src = load_peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    flush_buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    clean_buf = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def flush():
        flush_buf.zero_()
        # reading a second buffer larger than L2 writes the flush's dirty lines
        # back now (outside the timed region) and leaves L2 holding clean,
        # unrelated data, so the timed call pays for no write-backs but its own
        clean_buf.sum()

    def dev_bits(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    results = []
    iters = iters or max(args.steps, 5)
    if wl_name == "decode_28672x8192":
        work = synth.WORKLOADS[wl_name]
        r, alpha = work["r"], work["alpha"]
        for pi, (name, d, k) in enumerate(work["proj"]):
            W = dev_bits(synth.weight(d, k, seed=pi))
            q = Q.nf4_quantize(W, True)
            del W
            A, B = dev_bits(synth.lora_a(r, k, seed=pi)), dev_bits(synth.lora_b(d, r, seed=pi))
            for M in work["m"]:
                X = dev_bits(synth.activations(M, k, seed=pi))
                Y = torch.empty(M, d, dtype=torch.bfloat16, device=dev)
                T = torch.empty(M, Q.qlora_rank_pad(r), dtype=torch.bfloat16, device=dev)
                ws = torch.empty(max(Q.qlora_linear_workspace_size(M, d, k, r, False), 16), dtype=torch.uint8,
                                 device=dev)
                fn = lambda: Q.qlora_linear_fwd(X, q, A, B, alpha, Y=Y, T_save=T, workspace=ws, stream=stream)  # noqa: E731
                for _ in range(args.warmup):
                    fn()
                ms = _timed(fn, iters, flush, stream)
                Q.qlora_profile_read()
                Q.qlora_profile_enable(True)
                _timed(fn, iters, flush, stream)
                Q.qlora_profile_enable(False)
                kms, kn = Q.qlora_profile_read()
                nf4 = nf4_bytes(d, k)
                act = 2 * (M * k + M * d + r * k + d * r)
                fl = flops_fwd(M, d, k, r)
                main_ms = kms["fwd_gemm"] / max(kn["fwd_gemm"], 1)
                results.append({"proj": f"{name}:{d}x{k}", "M": M, "ms": round(ms, 4),
                                "nf4_weight_gbs": round(nf4 / (ms * 1e-3) / 1e9, 1),
                                "nf4_weight_frac_hbm": round(nf4 / (ms * 1e-3) / 1e9 / hbm, 4),
                                "bytes_gbs": round((nf4 + act) / (ms * 1e-3) / 1e9, 1),
                                "tflops": round(fl / (ms * 1e-3) / 1e12, 2),
                                "main_kernel_ms": round(main_ms, 4),
                                "main_kernel_nf4_gbs": round(nf4 / (main_ms * 1e-3) / 1e9, 1) if main_ms else None,
                                "launches": int(sum(kn.values())) // iters})
        metric, unit = "QLoRA decode-like forward NF4-weight GB/s (M in 1,8,32,128)", "GB/s"
        value = statistics.median([x["nf4_weight_gbs"] for x in results if x["M"] <= 32])
    elif wl_name == "quant_sweep":
        for pi, (name, d, k) in enumerate(synth.WORKLOADS[wl_name]["proj"]):
            W = dev_bits(synth.weight(d, k, seed=pi, outliers=True))
            n = d * k
            nblk = -(-n // 64)
            for dq in (1, 2, 0):   # Int8 constants, E4M3 constants, DQ off
                q = Q.nf4_alloc(d, k, dq, dev)
                wsz = Q.qlora_nf4_sizes(d, k, 64, dq)[1]
                qws = torch.empty(max(wsz, 16), dtype=torch.uint8, device=dev)
                out = torch.empty(d, k, dtype=torch.bfloat16, device=dev)
                fq = lambda: Q.nf4_quantize(W, dq, out=q, workspace=qws, stream=stream)  # noqa: E731
                fd = lambda: Q.nf4_dequantize(q, out=out, stream=stream)  # noqa: E731
                for _ in range(args.warmup):
                    fq()
                    fd()
                mq = _timed(fq, iters, flush, stream)
                md = _timed(fd, iters, flush, stream)
                consts = (nblk + 4 * (-(-nblk // 256)) + 4) if dq else 4 * nblk
                qbytes = 2 * n + (n + 1) // 2 + consts + (2 * nblk * 2 if dq else 0)   # + bf16 scale scratch write/read
                dbytes = (n + 1) // 2 + consts + 2 * n
                results.append({"proj": f"{name}:{d}x{k}", "double_quant": bool(dq),
                                "dq_format": ("off", "int8", "fp8")[dq],
                                "quantize_ms": round(mq, 4), "quantize_gbs": round(qbytes / (mq * 1e-3) / 1e9, 1),
                                "quantize_frac_hbm": round(qbytes / (mq * 1e-3) / 1e9 / hbm, 4),
                                "dequantize_ms": round(md, 4), "dequantize_gbs": round(dbytes / (md * 1e-3) / 1e9, 1),
                                "dequantize_frac_hbm": round(dbytes / (md * 1e-3) / 1e9 / hbm, 4)})
        metric, unit = "NF4 quantize GB/s (4096x11008, double quant)", "GB/s"
        value = [x for x in results if x["proj"].startswith("rect") and x["dq_format"] == "int8"][0]["quantize_gbs"]
    elif wl_name == "merge_sweep":
        work = synth.WORKLOADS[wl_name]
        r, alpha = work["r"], work["alpha"]
        for pi, (name, d, k) in enumerate(work["proj"]):
            q = Q.nf4_quantize(dev_bits(synth.weight(d, k, seed=pi)), True)
            A = dev_bits(synth.lora_a(r, k, seed=pi))
            B = dev_bits(synth.lora_b(d, r, seed=pi))
            out = torch.empty(d, k, dtype=torch.bfloat16, device=dev)
            fm = lambda: Q.qlora_lora_merge(q, A, B, alpha, out=out, stream=stream)  # noqa: E731
            for _ in range(args.warmup):
                fm()
            mm = _timed(fm, iters, flush, stream)
            n = d * k
            nblk = n // 64
            # algorithmic bytes: codes + c2 + c1 + mean read, merged bf16 written, adapters read once
            mbytes = n // 2 + nblk + 4 * (-(-nblk // 256)) + 4 + 2 * n + 2 * r * (d + k)
            results.append({"proj": f"{name}:{d}x{k}", "r": r, "merge_ms": round(mm, 4),
                            "merge_gbs": round(mbytes / (mm * 1e-3) / 1e9, 1),
                            "merge_frac_hbm": round(mbytes / (mm * 1e-3) / 1e9 / hbm, 4)})
        metric, unit = "LoRA merge GB/s (W_merged = W^ + (alpha/r) B A, 11008x4096, r=64)", "GB/s"
        value = [x for x in results if x["proj"].startswith("gate")][0]["merge_gbs"]
    else:
        raise SystemExit(f"unknown secondary workload {wl_name}")
    del flush_buf, clean_buf
    torch.cuda.empty_cache()
    return {"metric": metric, "value": value, "unit": unit, "n_gpus": 1, "workload": wl_name,
            "hbm_peak_gbs": hbm, "peak_source": src,
            "l2": f"flushed ({2 * L2_BYTES >> 20} MiB write, then {2 * L2_BYTES >> 20} MiB read of a second "
                  "buffer so that no dirty lines remain) before every run",
            "iters": iters, "results": results}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="llama65b_block_m8192",
                    choices=("llama7b_proj_set_m4096", "llama65b_block_m8192", "proj_q_4096", "tiny_512",
                             "llama7b_proj_set_m4096_dropout", "llama65b_block_m8192_dropout",
                             "llama7b_proj_set_m4096_grouped", "llama65b_block_m8192_grouped",
                             "decode_28672x8192", "quant_sweep", "merge_sweep"))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the decode and quantisation workloads appended to the default line")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.workload in ("decode_28672x8192", "quant_sweep", "merge_sweep"):
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "secondary workloads are measured for this arm only"}))
            return
        run_secondary(args, args.workload)
        return
    work = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, work, args.workload)
    else:
        run_ours(args, work, args.workload)


if __name__ == "__main__":
    main()
