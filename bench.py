#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200: TFLOP/s of a GPT-style attention training step.

A step is one pass of the whole path over one batch of synthetic input: the forward (O and LSE) and the
recomputation backward (preprocess, main dK/dV/dQ kernel, dQ conversion) for B=4, H=32, Sq=Sk=8192, D=128,
bf16, causal, with q, k, v and dO iid N(0,1) from a fixed seed. FLOPs: forward 4*B*H*D*pairs, backward
10*B*H*D*pairs (five products, the recomputed Q K^T included), pairs = S(S+1)/2 visible (query, key) pairs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload gpt|long|...]

Prints one JSON line (rank 0). ``value`` is the whole-job TFLOP/s from CUDA events with the inputs resident
in HBM (1.07 GB per step, larger than the 126 MB L2); ``e2e`` is the same metric through the public Python API
with pinned host inputs copied in and the gradients copied out every step (two buffer sets on separate upload,
compute and download streams, so step i+1's upload and step i-1's download overlap step i); ``roofline``
rates the dominant kernel against the measured bf16 peak, and ``roofline.mufu`` its exponentials against the
MUFU bound (16 per cycle per SM), which binds the head-dim-64 forward; ``clocks`` summarises nvidia-smi samples
taken in the timed region (or, for a region shorter than the sampling period, the samples on either side);
``cpu_baseline`` times the fp64 CPU oracle on a bounded row sample.
With N > 1 (torchrun) every GPU runs its own replica of the workload (weak scaling, no collective on the data
path) and the time is the maximum over ranks. ``--impl reference`` times the oracle itself as the reference
arm (rank 0 only).
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
NOMINAL_BF16_TFLOPS = 2250.0
# MUFU (special-function unit) roofline: 16 exponentials per cycle per SM, 148 SMs, at the top SM clock
# (`clocks.max.sm`, 1965 MHz on these B200s, used when no clock was sampled).
MUFU_EXP_PER_CYCLE_SM = 16
N_SMS = 148
NOMINAL_SM_MHZ = 1965.0
_COMMON_SOURCES = ["exact_io_aware_76_b200/csrc/sm100.cuh", "exact_io_aware_76_b200/csrc/tmem_ldst.inc",
                   "exact_io_aware_76_b200/csrc/dropout.cuh"]
KERNEL_SOURCES = {
    "fa_bwd_main": ["exact_io_aware_76_b200/csrc/fa_bwd128.cuh", "exact_io_aware_76_b200/csrc/fa_bwd.cuh"] + _COMMON_SOURCES,
    "fa_fwd": ["exact_io_aware_76_b200/csrc/fa_fwd.cuh"] + _COMMON_SOURCES,
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gpt")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--batch", type=int, default=None, help="override B (smaller cases for profiling)")
    ap.add_argument("--heads", type=int, default=None, help="override H (smaller cases for profiling)")
    ap.add_argument("--variant", choices=["plain", "fp8", "dropout"], default="plain",
                    help="fp8: the e4m3 forward alone; dropout: forward + backward with dropout_p 0.1")
    return ap.parse_args()


def workload_from_args(args):
    import dataclasses

    from exact_io_aware_76_b200.workloads import WORKLOADS

    w = WORKLOADS[args.workload]
    if args.batch is not None or args.heads is not None:
        B = args.batch or w.B
        H = args.heads or w.H
        w = dataclasses.replace(w, B=B, H=H, name="%s_b%dh%d" % (w.name, B, H))
    return w


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("bf16_tflops", "bf16_tflops_sustained", "hbm_gbs")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def source_sha(kernel):
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)["%s/%s" % (kernel, workload)]
    except Exception:
        return None
    if rec.get("source_sha") != source_sha(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


# ------------------------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples (every 100 ms) of the SM clock, power and throttle reasons of one GPU."""

    FIELDS = ["timestamp", "uuid", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, uuid):
        self.uuid = (uuid or "").lower().replace("gpu-", "")
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == len(self.FIELDS):
                self.rows.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        def num(x):
            try:
                return float(x.split()[0])
            except Exception:
                return None

        mine = []
        for (ts, p) in self.rows:
            uid = p[1].lower().replace("gpu-", "")
            if self.uuid and uid and uid != self.uuid:
                continue
            mine.append((ts, p))
        sel = [p for (ts, p) in mine if t0 <= ts <= t1 + 0.15]
        window = "timed region"
        if not sel and mine:
            # A timed region shorter than the sampling period: the samples just before and just after it.
            before = [(ts, p) for (ts, p) in mine if ts < t0]
            after = [(ts, p) for (ts, p) in mine if ts > t1]
            sel = ([before[-1][1]] if before else []) + ([after[0][1]] if after else [])
            window = "nearest samples before and after the timed region (shorter than the 100 ms sampling period)"
        if not sel:
            return None
        sm = [num(p[2]) for p in sel if num(p[2]) is not None]
        mx = [num(p[3]) for p in sel if num(p[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in sel for i in range(4) if p[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sel), "window": window,
                "power_w_max": max((num(p[4]) for p in sel if num(p[4]) is not None), default=None)}


# ------------------------------------------------------------------------------------------------ oracle leg
CPU_SAMPLE_SEED = 0
CPU_SAMPLE_FLOPS = 1.6e10  # under a second of the oracle on a 16-core host


def oracle_rows(w):
    """The oracle's sample, identical in both legs: a fixed number of query rows of head (b=0, h=0), chosen by
    the workload alone (about CPU_SAMPLE_FLOPS of executed work, 16 to 1024 rows) and drawn with a fixed seed."""
    import numpy as np

    per_row = (4 if not w.backward else 14) * w.D * w.Sk
    n = int(max(16, min(1024, w.Sq, CPU_SAMPLE_FLOPS // per_row)))
    return np.sort(np.random.default_rng(CPU_SAMPLE_SEED).choice(w.Sq, n, replace=False)).astype(np.int64)


def oracle_sample(w, q, k, v, do, reps=1):
    """Time the fp64 oracle (forward, and backward for a training workload) ``reps`` times on the fixed row
    sample of ``oracle_rows``. Returns (TFLOP/s under the benchmark's FLOP convention, TFLOP/s of the work the
    oracle executes, description, threads, seconds). The oracle walks every key of a listed row (masked ones
    too) in each of its loops: forward 4*D*Sk and backward 10*D*Sk FLOPs per row, while the convention counts
    the visible keys only."""
    import numpy as np

    import oracle

    # The same OpenMP team size in every process that times the oracle: one thread per core this process may
    # run on (torch, loaded first, may have set its own default in the shared OpenMP runtime).
    threads = oracle.set_threads(len(os.sched_getaffinity(0)))
    to64 = lambda x: x[0, :, 0, :].detach().to("cpu").double().numpy()[None]  # noqa: E731
    qh, kh, vh, doh = to64(q), to64(k), to64(v), to64(do)
    fwd_only = not w.backward
    rows = oracle_rows(w)
    keys = np.minimum(w.Sk, rows + (w.Sk - w.Sq) + 1) if w.causal else np.full(rows.shape, w.Sk)
    per = 4 if fwd_only else 14
    algorithmic = float(per * w.D * keys.sum()) * reps
    executed = float(per * w.D * w.Sk * len(rows)) * reps
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.attn_fwd(qh, kh, vh, causal=w.causal, rows=rows[None])
        if not fwd_only:
            oracle.attn_bwd(qh, kh, vh, doh, causal=w.causal, rows=rows[None])
    dt = time.perf_counter() - t0
    desc = ("%d query rows of head (b=0,h=0) of the %s workload drawn with seed %d, %s, fp64 oracle, %d run(s); the "
            "oracle walks all %d keys of each row (executed %.3g TFLOP/s)" % (
                len(rows), w.name, CPU_SAMPLE_SEED, "forward only" if fwd_only else "forward + backward", reps,
                w.Sk, executed / dt / 1e12))
    return algorithmic / dt / 1e12, executed / dt / 1e12, desc, threads, dt


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline_record(w, value, executed, threads, desc):
    """The oracle's sampled rate, the host it ran on, and the time the whole problem would take at that rate
    (an extrapolation, labelled as one)."""
    full = w.fwd_flops() + (w.bwd_flops() if w.backward else 0)
    return {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
            "executed_tflops": executed, "cpu_model": cpu_model(),
            "extrapolated_full_problem_s": full / (value * 1e12) if value > 0 else None}


# ------------------------------------------------------------------------------------------------ arms
def run_reference(args):
    from exact_io_aware_76_b200.inputs import make_inputs
    from exact_io_aware_76_b200.replicas import env_rank

    rank, world, _ = env_rank()
    if rank != 0:
        return 0
    w = workload_from_args(args)
    # One head of the workload's distribution is all the oracle sample reads (same recipe, generated on the CPU).
    q, k, v, do = make_inputs(1, w.Sq, w.Sk, 1, w.D, w.dtype, w.seed, w.sigma, "cpu", with_dout=True)
    # Every step is one run of the same fixed sample the other arm's cpu_baseline leg times (oracle_rows).
    for _ in range(args.warmup):
        oracle_sample(w, q, k, v, do)
    vals, execs, secs = [], [], 0.0
    desc, threads = "", 0
    for _ in range(args.steps):
        val, ex, desc, threads, dt = oracle_sample(w, q, k, v, do)
        vals.append(val)
        execs.append(ex)
        secs += dt
    value = statistics.mean(vals)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1000.0 * secs / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": workload_config(w, 1),
            "cpu_baseline": cpu_baseline_record(w, value, statistics.mean(execs), threads, desc),
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


METRIC = "attention fwd/bwd TFLOP/s (bf16, causal) and % of B200 dense tensor peak"


L2_BYTES = 126 << 20


def input_bytes(w):
    """Bytes one step reads as its inputs (q, k, v, and dO for a training step)."""
    return (4 if w.backward else 3) * w.B * w.Sq * w.H * w.D * 2


def variant_config(cfg, variant):
    """The workload description of a --variant run (the plain run keeps the workload's own)."""
    cfg = dict(cfg, variant=variant)
    if variant == "fp8":
        cfg["workload"] = cfg["workload"].replace("training step (forward + recomputation backward)",
                                                  "forward on e4m3 inputs (descale 1), bf16 output")
    elif variant == "dropout":
        cfg["workload"] += ", attention dropout_p 0.1 (Philox seed 1234, offset 0)"
    return cfg


def workload_config(w, n):
    kind = "training step (forward + recomputation backward)" if w.backward else "forward"
    return {"workload": "%s %s: B=%d H=%d Sq=%d Sk=%d D=%d %s %s" % (
                w.name, kind, w.B, w.H, w.Sq, w.Sk, w.D, w.dtype, "causal" if w.causal else "non-causal"),
            "global_batch": w.B * n, "seq_len": w.Sq,
            "parallelism": "replicas x%d (weak scaling; no collective on the data path)" % n,
            "l2": ("inputs larger than L2 (%.2f GB per step)" % (input_bytes(w) / 1e9)) if input_bytes(w) >= L2_BYTES
            else ("L2 flushed before every timed step by a 256 MB write outside the step's events (inputs %.3f GB)"
                  % (input_bytes(w) / 1e9))}


def run_ours(args):
    import torch

    import exact_io_aware_76_b200 as fa
    from exact_io_aware_76_b200 import replicas
    from exact_io_aware_76_b200.inputs import make_inputs

    rank, world, local_rank = replicas.env_rank()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    replicas.init("nccl" if world > 1 else "gloo")
    w = workload_from_args(args)
    variant = args.variant
    fwd_only = not w.backward or variant == "fp8"
    seed = replicas.replica_seed(w.seed, rank)
    q, k, v, do = make_inputs(w.B, w.Sq, w.Sk, w.H, w.D, w.dtype, seed, w.sigma, "cuda", with_dout=True)
    out = torch.empty_like(q)
    if variant == "fp8":  # the same draws rounded to e4m3 (descale 1); the output stays bf16
        q, k, v = (t.to(torch.float8_e4m3fn) for t in (q, k, v))
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    drop = dict(dropout_p=0.1, seed=1234, offset=0) if variant == "dropout" else {}

    def fwd_call(q_, k_, v_, out_, lse_):
        if variant == "fp8":
            return fa.fwd_fp8(q_, k_, v_, causal=w.causal, out=out_, lse=lse_)
        return fa.fwd(q_, k_, v_, causal=w.causal, out=out_, lse=lse_, **drop)

    lse = torch.empty((w.B, w.H, w.Sq), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.workspace_size(w.B, w.Sq, w.H, w.D), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    if fwd_only:
        names = ["fa_fwd"]
    elif variant == "dropout":  # the backward's launches are not separable with dropout: timed as one interval
        names = ["fa_fwd", "fa_bwd"]
    else:
        names = ["fa_fwd", "fa_bwd_pre", "fa_bwd_main", "fa_bwd_dq"]

    def step(evs=None):
        def mark(i):
            if evs is not None:
                evs[i].record(stream)
        mark(0)
        fwd_call(q, k, v, out, lse)
        mark(1)
        if fwd_only:
            return
        if variant == "dropout":
            fa.bwd(q, k, v, out, lse, do, causal=w.causal, dq=dq, dk=dk, dv=dv, workspace=ws, **drop)
            mark(2)
            return
        for st in range(3):
            fa.bwd(q, k, v, out, lse, do, causal=w.causal, dq=dq, dk=dk, dv=dv, workspace=ws, stage=st)
            mark(2 + st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert fa.device_status() == 0, "a kernel reported a timeout during warm-up"

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(K)]
    # Inputs that fit in L2 would be re-read from it by the next step: then a 256 MB write (twice the 126 MB
    # L2) runs before every timed step, outside the step's own events, and `value` comes from those events.
    flush_l2 = input_bytes(w) < L2_BYTES
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush_l2 else None
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(str(getattr(props, "uuid", "")))
    if rank == 0:
        sampler.start()
        time.sleep(0.5)
    replicas.barrier(dev)
    torch.cuda.synchronize()
    t_host0 = time.time()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(K):
        if flush_l2:
            flush_buf.zero_()
        step(evs[i])
    stop.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.time()
    replicas.barrier(dev)
    local_ms = start.elapsed_time(stop)
    if flush_l2:
        local_ms = sum(evs[i][0].elapsed_time(evs[i][-1]) for i in range(K))
    # O(N) memory: everything the step holds on the device (inputs, outputs, workspace) against what one S x S
    # bf16 score matrix per (batch, head) would take.
    peak_bytes = torch.cuda.max_memory_allocated(dev)
    max_ms = replicas.max_over_ranks(local_ms, dev)
    if rank == 0:
        sampler.stop()
    status = fa.device_status()
    assert status == 0, "a kernel reported status %d" % status

    per_kernel = {n: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K))
                  for j, n in enumerate(names)}
    flops_fwd = w.fwd_flops()
    flops_bwd = 0 if fwd_only else w.bwd_flops()
    flops_step = flops_fwd + flops_bwd
    value = flops_step * world * K / (max_ms / 1e3) / 1e12

    # ---- e2e through the public API with pinned host buffers. Every step uploads its inputs from pinned host
    # memory and downloads its gradients (or, forward-only, its output) inside the timed region. Steps are
    # pipelined the way a training loop prefetches: two device buffer sets, an upload stream, the compute
    # stream and a download stream, so step i+1's upload and step i-1's download overlap step i's kernels;
    # events keep a buffer set from being overwritten before the kernels or the download that use it finish.
    e2e = None
    if args.e2e_steps > 0:
        hq, hk, hv, hdo = (t.to("cpu").pin_memory() for t in (q, k, v, do))
        host_in = (hq, hk, hv) if fwd_only else (hq, hk, hv, hdo)
        outs_h = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in ((out,) if fwd_only else (dq, dk, dv))]
        h2d = sum(t.numel() * t.element_size() for t in host_in)
        d2h = sum(t.numel() * t.element_size() for t in outs_h)
        dev_in = [tuple(q_ if i == 0 else torch.empty_like(q_) for q_ in ((q, k, v) if fwd_only else (q, k, v, do)))
                  for i in range(2)]
        dev_out = [tuple(t if i == 0 else torch.empty_like(t) for t in ((out,) if fwd_only else (dq, dk, dv)))
                   for i in range(2)]
        dev_lse = [lse, torch.empty_like(lse)]
        dev_o = [out, torch.empty_like(out)]
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        n_steps = args.e2e_steps

        def run_pipeline(n, a_ev=None, b_ev=None):
            uploaded = [torch.cuda.Event() for _ in range(n)]
            computed = [torch.cuda.Event() for _ in range(n)]
            downloaded = [torch.cuda.Event() for _ in range(n)]
            if a_ev is not None:
                a_ev.record(up)
            for i in range(n):
                x = i % 2
                with torch.cuda.stream(up):
                    if i >= 2:
                        up.wait_event(computed[i - 2])  # the kernels of step i-2 are done with this input set
                    for d_, h_ in zip(dev_in[x], host_in):
                        d_.copy_(h_, non_blocking=True)
                    uploaded[i].record(up)
                stream.wait_event(uploaded[i])
                if i >= 2:
                    stream.wait_event(downloaded[i - 2])  # step i-2's gradients have left this output set
                ins = dev_in[x]
                if fwd_only:
                    fwd_call(ins[0], ins[1], ins[2], dev_out[x][0], dev_lse[x])
                else:
                    o_, l_ = fwd_call(ins[0], ins[1], ins[2], dev_o[x], dev_lse[x])
                    fa.bwd(ins[0], ins[1], ins[2], o_, l_, ins[3], causal=w.causal, dq=dev_out[x][0],
                           dk=dev_out[x][1], dv=dev_out[x][2], workspace=ws, **drop)
                computed[i].record(stream)
                with torch.cuda.stream(down):
                    down.wait_event(computed[i])
                    for hbuf, t in zip(outs_h, dev_out[x]):
                        hbuf.copy_(t, non_blocking=True)
                    downloaded[i].record(down)
            if b_ev is not None:
                b_ev.record(down)

        run_pipeline(2)
        torch.cuda.synchronize()
        replicas.barrier(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        run_pipeline(n_steps, a, b)
        torch.cuda.synchronize()
        e2e_ms = replicas.max_over_ranks(a.elapsed_time(b), dev)
        e2e = {"value": flops_step * world * n_steps / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / n_steps,
               "pipelining": "two device buffer sets; step i+1's upload and step i-1's download overlap step i"}

    if rank != 0:
        replicas.shutdown()
        return 0

    peaks, peak_src = load_peaks()
    dom = max(per_kernel, key=per_kernel.get)
    dom_flops = flops_fwd if dom == "fa_fwd" else flops_bwd  # the backward's products all run in its main kernel
    achieved = dom_flops / (per_kernel[dom] / 1e3) / 1e12
    traffic = recorded_traffic(dom, w.name) if variant == "plain" else None
    # e4m3 products: the measured bf16 peak times the nominal e4m3/bf16 ratio (4.5 / 2.25 PFLOP/s dense)
    peak = peaks["bf16_tflops"] * (2.0 if variant == "fp8" else 1.0)
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                "peak_source": ("burst bf16 of %s x 2 (nominal e4m3/bf16 ratio)" if variant == "fp8"
                                else "burst bf16 of %s") % peak_src,
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "frac_of_nominal_2250": achieved / NOMINAL_BF16_TFLOPS,
                "algorithmic_flops_per_launch": dom_flops}
    kernels = {n: {"ms": per_kernel[n]} for n in names}
    kernels["fa_fwd"]["tflops"] = flops_fwd / (per_kernel["fa_fwd"] / 1e3) / 1e12
    if variant == "dropout":
        kernels["fa_bwd"]["tflops"] = flops_bwd / (per_kernel["fa_bwd"] / 1e3) / 1e12
        bwd_ms = per_kernel["fa_bwd"]
    elif not fwd_only:
        kernels["fa_bwd_main"]["tflops"] = flops_bwd / (per_kernel["fa_bwd_main"] / 1e3) / 1e12
        bwd_ms = per_kernel["fa_bwd_pre"] + per_kernel["fa_bwd_main"] + per_kernel["fa_bwd_dq"]
    cpu = None
    if world == 1 and not args.no_cpu_baseline and variant == "plain":
        _, _, _, _, t1 = oracle_sample(w, q, k, v, do)  # one untimed run (warm-up and calibration)
        reps = int(max(1, min(30, round(args.cpu_seconds / max(t1, 1e-3)))))
        val, ex, desc, threads, _ = oracle_sample(w, q, k, v, do, reps)
        cpu = cpu_baseline_record(w, val, ex, threads, desc)
    clocks = sampler.summary(t_host0, t_host1)
    # The softmax's exponentials, one per visible (query, key) pair in either kernel, against the MUFU bound; in
    # tensor-FLOP units that bound is exp/s times the kernel's FLOP per pair (4*D forward, 10*D backward), which
    # says which of the two units limits the kernel (the forward at head dim 64: MUFU).
    n_exp = w.B * w.H * w.pairs()
    mhz = (clocks or {}).get("sm_max_mhz") or NOMINAL_SM_MHZ
    exp_peak = MUFU_EXP_PER_CYCLE_SM * N_SMS * mhz * 1e6 / 1e9
    exp_achieved = n_exp / (per_kernel[dom] / 1e3) / 1e9
    equiv_peak = exp_peak * (dom_flops / n_exp) / 1e3
    roofline["mufu"] = {"achieved": exp_achieved, "peak": exp_peak, "unit": "Gexp/s", "frac": exp_achieved / exp_peak,
                        "tflops_equivalent_peak": equiv_peak, "binding": "mufu" if equiv_peak < peak else "tensor",
                        "peak_source": "%d exp per cycle per SM x %d SMs x %.0f MHz" % (MUFU_EXP_PER_CYCLE_SM, N_SMS,
                                                                                        mhz)}
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": max_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3" if variant == "fp8" else "bf16", "data": "synthetic",
            "config": variant_config(workload_config(w, world), variant), "roofline": roofline,
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": len(names) * K, "clocks": clocks,
            "fwd_tflops": kernels["fa_fwd"]["tflops"],
            "fwd_frac_of_measured_peak": kernels["fa_fwd"]["tflops"] / peaks["bf16_tflops"],
            "kernels": kernels,
            # model FLOPs: the backward without its recomputed Q K^T (8*B*H*D*pairs), alongside the
            # algorithmic 10*B*H*D*pairs that `value` uses
            "step_model_tflops": (flops_fwd + 0.8 * flops_bwd) * world * K / (max_ms / 1e3) / 1e12,
            "memory": {"peak_device_bytes": peak_bytes,
                       "score_matrix_bf16_bytes": 2 * w.B * w.H * w.Sq * w.Sk}}
    if not fwd_only:
        line["bwd_tflops"] = flops_bwd / (bwd_ms / 1e3) / 1e12
        line["bwd_frac_of_measured_peak"] = line["bwd_tflops"] / peaks["bf16_tflops"]
        line["step_frac_of_measured_peak"] = (flops_step / ((per_kernel["fa_fwd"] + bwd_ms) / 1e3) / 1e12) / peaks["bf16_tflops"]
    print(json.dumps(line), flush=True)
    replicas.shutdown()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
