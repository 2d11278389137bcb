#!/usr/bin/env python
"""Benchmark of one exact-attention training step on B200: forward + backward.

A step is one pass of the whole hot path over one batch of the training
workload (B=4, N=4096, H=8, d=64, bf16, seeded N(0,1) inputs): fa_fwd
(Q tiles x K/V tiles with online softmax, O and LSE out) then fa_bwd
(rowsum preprocess, recompute of P from the LSE, dQ/dK/dV).  Throughput counts
4 B H N^2 d for the forward and 2.5x that for the backward.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c5]
  python bench.py --impl reference ...   (the fp64 CPU oracle, timed on a sample)

Under torchrun every rank runs its own replica of the workload (weak scaling,
no collective on the data path); the step time is the max over ranks.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
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
import torch  # noqa: E402

import attn_inputs  # noqa: E402

METRIC = "fused attention fwd/bwd TFLOP/s on 1 B200 and % of bf16 tensor-core peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 512 << 20
L2_NOTE = "512 MiB written between timed GPU steps"
# The pages' five configurations and the N sweep, each timed on its own in the
# same run (forward; forward + backward for the training workload), and the
# backward at the detector-neck (d = 256) and long-sequence (d = 128) shapes.
PER_CONFIG = ("c1", "c2", "c3", "c4", "sweep1024", "sweep2048", "sweep4096", "sweep8192", "c5",
              "c3train", "c4train")
PER_CONFIG_RUNS = 20
# The oracle runs a whole configuration when it costs at most this much work,
# otherwise the first rows of every head, sized to about this much.
ORACLE_BUDGET_GFLOP = 40.0

# DRAM traffic of the dominant kernel per launch, from an ncu capture of the
# same workload (dram__bytes_read.sum + dram__bytes_write.sum), valid only
# while the kernel sources' code (comments excluded) hashes to the recorded
# value.
TRAFFIC = {
    ("fa_bwd_kernel", "c5_train_b4_n4096_h8_d64"): {"bytes": 101.761536e6 + 23.452672e6,
                                                    "src": "83d013b47bf940ef"},
    ("fa_fwd_pp_kernel", "c5_train_b4_n4096_h8_d64"): {"bytes": 50.483200e6 + 2.427392e6,
                                                       "src": "83d013b47bf940ef"},
    ("fa_fwd_pp_kernel", "c4_long_n8192_h8_d128"): {"bytes": 51.347456e6 + 4.947456e6,
                                                    "src": "83d013b47bf940ef"},
    ("fa_bwd_tq_kernel", "c4_train_n8192_h8_d128"): {"bytes": 102.718976e6 + 117.569280e6,
                                                     "src": "83d013b47bf940ef"},
    ("fa_fwd_pp_kernel", "c4_long_fp8_n8192_h8_d128"): {"bytes": 25.291776e6 + 0.559360e6,
                                                        "src": "83d013b47bf940ef"},
    ("fa_fwd_pp_kernel", "c2_detector_deep_b32_n400_h4_d64"): {"bytes": 19.760128e6,
                                                               "src": "83d013b47bf940ef"},
    ("fa_fwd_kernel", "c3_detector_neck_n6400_h1_d256"): {"bytes": 9.939200e6,
                                                          "src": "83d013b47bf940ef"},
    ("fa_bwd_tq_kernel", "c3_train_n6400_h1_d256"): {"bytes": 20.036864e6 + 6.463488e6,
                                                     "src": "83d013b47bf940ef"},
}


def workload_config(w: attn_inputs.Workload, world: int = 1) -> dict:
    """The `config` object of the JSON line: the workload, identical for both arms."""
    return {"workload": w.name, "global_batch": w.B * world, "seq_len": w.N, "heads": w.H,
            "head_dim": w.d, "causal": False,
            "parallelism": f"replicas x{world} (batch per rank, no collective)",
            "l2": L2_NOTE,
            "inputs": "seeded N(0,1) draws rounded to the "
                      + ("E4M3 type (descale factors 1), bf16 O" if w.dtype == "fp8"
                         else "16-bit type")}


def io_bytes(w: attn_inputs.Workload, backward: bool) -> float:
    """Algorithmic HBM bytes of one call: forward reads Q, K, V and writes O
    and the LSE; backward reads Q, K, V, O, dO and the LSE and writes dQ, dK,
    dV."""
    eb = 1 if w.dtype == "fp8" else 2
    elems = float(w.B) * w.N * w.H * w.d
    lse = 4.0 * w.B * w.H * w.N
    if backward:
        return 8 * elems * eb + lse
    return 3 * elems * eb + elems * (2 if w.dtype == "fp8" else eb) + lse


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _code_tokens(src: str) -> str:
    """The source with C/C++ comments removed and whitespace collapsed, so
    that editing a comment leaves the hash of the kernel code unchanged."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash() -> str:
    """Hash of the kernel sources' code (comments and layout excluded)."""
    h = hashlib.sha256()
    for name in ("fa_common.cuh", "fa_fwd.cu", "fa_bwd.cu"):
        with open(os.path.join(ROOT, "exact_attention_144_b200", "csrc", name)) as f:
            h.update(_code_tokens(f.read()).encode())
    return h.hexdigest()[:16]


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.001):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self.period, self.stop_ev, self.thread = period_s, threading.Event(), None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report nothing rather than guess
            self.nvml = None

    def _run(self):
        nv = self.nvml
        while not self.stop_ev.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml is not None:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def __exit__(self, *exc):
        self.stop_ev.set()
        if self.thread:
            self.thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def replica_seed(w: attn_inputs.Workload, rank: int) -> int:
    """Each rank owns one replica of the workload with its own seeded batch."""
    return w.seed + 7919 * rank


def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """The slowest rank's value (timing is reported as the max over ranks)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flop_per_step: float, ms_per_step: float, world: int) -> float:
    """Whole-job throughput: every rank processes flop_per_step in ms_per_step."""
    return world * flop_per_step / (ms_per_step * 1e-3) / 1e12


def entry_points(fa, w: attn_inputs.Workload):
    """(forward, backward, output dtype) of the library for the workload's
    element type; the 8-bit workloads are forward only, with bf16 O."""
    if w.dtype == "fp8":
        def fwd(q, k, v, o=None, lse=None, scale=None, stream=None):
            return fa.fa_fwd_fp8(q, k, v, o=o, lse=lse, scale=scale, stream=stream)
        return fwd, None, torch.bfloat16
    if w.dtype == "bf16":
        return fa.fa_fwd, fa.fa_bwd, torch.bfloat16
    return fa.fa_fwd_f16, fa.fa_bwd_f16, torch.float16


def tensor_peak(pk: dict, w: attn_inputs.Workload) -> tuple:
    """Dense tensor-core peak for the workload's operand type: the measured
    bf16 figure, doubled for 8-bit operands (the nominal fp8:bf16 ratio,
    4.5 : 2.25 PFLOP/s dense)."""
    if w.dtype == "fp8":
        return 2.0 * pk["bf16_tflops"], 2.0 * pk["bf16_tflops_sustained"], "2 x bf16_tflops"
    return pk["bf16_tflops"], pk["bf16_tflops_sustained"], "bf16_tflops"


def e2e_pipelined(fa, w, args, dev, q, k, v, do, train, mk):
    """Per-step time (ms) of steps that each upload their inputs from pinned
    host memory, compute, and download their results, overlapped across
    steps with two device buffer sets.  Every input uploads on a stream of
    its own and every result downloads on a stream of its own: a host-to-
    device copy carries a fixed start-up cost (about 0.1 ms on B200 hosts,
    against ~60 GB/s once running) that copies queued on one stream pay one
    after another and copies on separate streams overlap.  Returns (ms per
    step, bytes uploaded per step, bytes downloaded per step, the copies'
    own times)."""
    fwd, bwd, out_dtype = entry_points(fa, w)
    host_in = [t.cpu().pin_memory() for t in ((q, k, v, do) if train else (q, k, v))]
    sets = []
    for _ in range(2):
        ins = [torch.empty_like(t, device=dev) for t in host_in]
        outs = [torch.empty(q.shape, dtype=out_dtype, device=dev),
                torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)]
        if train:
            outs += [torch.empty_like(q) for _ in range(3)]
        hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
        sets.append((ins, outs, hout))
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in sets[0][2])
    s_up = [torch.cuda.Stream(dev) for _ in host_in]
    s_down = [torch.cuda.Stream(dev) for _ in sets[0][1]]
    s_comp = torch.cuda.Stream(dev)
    total = args.warmup + args.steps
    ev_in = [[torch.cuda.Event() for _ in s_up] for _ in range(total)]
    ev_comp = [torch.cuda.Event() for _ in range(total)]
    ev_out = [[torch.cuda.Event() for _ in s_down] for _ in range(total)]
    t0, t1 = mk(), mk()
    torch.cuda.synchronize()
    for i in range(total):
        ins, outs, hout = sets[i % 2]
        if i == args.warmup:
            t0.record(s_up[0])
        for j, (hsrc, dst, s) in enumerate(zip(host_in, ins, s_up)):
            with torch.cuda.stream(s):
                if i == args.warmup and j > 0:
                    s.wait_event(t0)  # no timed upload starts before the timed region
                if i >= 2:
                    s.wait_event(ev_comp[i - 2])  # compute of step i-2 is done with these inputs
                dst.copy_(hsrc, non_blocking=True)
                ev_in[i][j].record(s)
        with torch.cuda.stream(s_comp):
            for e in ev_in[i]:
                s_comp.wait_event(e)
            if i >= 2:
                for e in ev_out[i - 2]:
                    s_comp.wait_event(e)  # results of step i-2 have been read
            fwd(ins[0], ins[1], ins[2], o=outs[0], lse=outs[1], scale=w.scale, stream=s_comp)
            if train:
                bwd(ins[0], ins[1], ins[2], outs[0], ins[3], outs[1], dq=outs[2], dk=outs[3],
                    dv=outs[4], scale=w.scale, stream=s_comp)
            ev_comp[i].record(s_comp)
        for j, (dsrc, hdst, s) in enumerate(zip(outs, hout, s_down)):
            with torch.cuda.stream(s):
                s.wait_event(ev_comp[i])
                hdst.copy_(dsrc, non_blocking=True)
                ev_out[i][j].record(s)
    for e in ev_out[total - 1]:
        s_down[0].wait_event(e)
    t1.record(s_down[0])
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / args.steps

    # The same copies without kernels: uploads alone, downloads alone, and
    # both at once (the PCIe floor of the pipelined steps).
    ins, outs, hout = sets[0]
    main = s_comp

    def timed(up: bool, down: bool) -> float:
        a, b = mk(), mk()
        torch.cuda.synchronize()
        a.record(main)
        for s in s_up + s_down:
            s.wait_event(a)
        for _ in range(args.steps):
            if up:
                for hsrc, dst, s in zip(host_in, ins, s_up):
                    with torch.cuda.stream(s):
                        dst.copy_(hsrc, non_blocking=True)
            if down:
                for dsrc, hdst, s in zip(outs, hout, s_down):
                    with torch.cuda.stream(s):
                        hdst.copy_(dsrc, non_blocking=True)
        for s in s_up + s_down:
            main.wait_stream(s)
        b.record(main)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / args.steps

    copies = {"h2d_ms": timed(True, False), "d2h_ms": timed(False, True),
              "both_ms": timed(True, True)}
    copies["h2d_gbs"] = h2d / (copies["h2d_ms"] * 1e-3) / 1e9
    copies["d2h_gbs"] = d2h / (copies["d2h_ms"] * 1e-3) / 1e9
    return ms, h2d, d2h, copies


def main_kernel_names(fa, w: attn_inputs.Workload, props) -> tuple:
    """Names of the forward and backward main kernels the library launches for
    this workload (the ones the kernel events bracket)."""
    plan = fa.fa_fwd_plan(w.B, w.H, w.N, w.d, props.multi_processor_count)
    fwd = "fa_fwd_pp_kernel" if plan["kernel"] == 1 else "fa_fwd_kernel"
    bwd = "fa_bwd_kernel" if w.d == 64 else "fa_bwd_tq_kernel"
    return fwd, bwd


def _stats(xs):
    return statistics.mean(xs), statistics.median(xs)


def time_config(fa, w: attn_inputs.Workload, dev, flush, runs: int, local: int, pk: dict):
    """Times one configuration on its own: `runs` forward calls (and backward
    calls for the training workload), each after a 512 MiB write that evicts
    L2.  CUDA events bracket the whole call and, through
    fa_set_kernel_events, the main kernel alone.  Returns the configuration's
    entry of the JSON line's per_config object (plus the forward output and
    LSE, for the C1 report on the unrounded draws)."""
    q, k, v, do = attn_inputs.draw(w.B, w.N, w.H, w.d, w.dtype, w.seed, 4, std=w.std,
                                   device=dev)
    fwd, bwd, out_dtype = entry_points(fa, w)
    train = w.backward and bwd is not None
    o = torch.empty(q.shape, dtype=out_dtype, device=dev)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))

    def call_fwd():
        fwd(q, k, v, o=o, lse=lse, scale=w.scale)

    def call_bwd():
        bwd(q, k, v, o, do, lse, dq=dq, dk=dk, dv=dv, scale=w.scale)

    for _ in range(3):
        call_fwd()
        if train:
            call_bwd()
    torch.cuda.synchronize()
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev = [[mk() for _ in range(8)] for _ in range(runs)]
    with ClockSampler(local) as clk:
        for e in ev:
            flush.zero_()
            fa.fa_set_kernel_events(e[2], e[3], e[6] if train else None, e[7] if train else None)
            e[0].record()
            call_fwd()
            e[1].record()
            if train:
                e[4].record()
                call_bwd()
                e[5].record()
        torch.cuda.synchronize()
    clocks = clk.summary()
    mhz = clocks["sm_mhz"]
    props = torch.cuda.get_device_properties(dev)
    plan = fa.fa_fwd_plan(w.B, w.H, w.N, w.d, props.multi_processor_count)
    fwd_name, bwd_name = main_kernel_names(fa, w, props)
    peak, peak_sus, _ = tensor_peak(pk, w)

    src_hash = kernel_source_hash()

    def part(kern_ms, call_ms, flop, nbytes, name):
        k_mean, k_med = _stats(kern_ms)
        c_mean, c_med = _stats(call_ms)
        tf = flop / (k_mean * 1e-3) / 1e12
        gbs = nbytes / (k_mean * 1e-3) / 1e9
        tr = TRAFFIC.get((name.split(" ")[0], w.name))
        return {"kernel": name, "kernel_us": 1e3 * k_mean, "kernel_us_median": 1e3 * k_med,
                "traffic": tr["bytes"] if tr and tr["src"] == src_hash else None,
                "call_us": 1e3 * c_mean, "call_us_median": 1e3 * c_med,
                "kernel_cycles": (1e3 * k_mean * mhz) if mhz else None,
                "tflops": tf, "pct_peak": 100.0 * tf / peak,
                "pct_peak_sustained": 100.0 * tf / peak_sus,
                "call_tflops": flop / (c_mean * 1e-3) / 1e12,
                "gbs": gbs, "pct_hbm": 100.0 * gbs / pk["hbm_gbs"],
                "algorithmic_bytes": nbytes}

    extra = " + fa_combine_kernel" if plan["n_split"] > 1 else ""
    entry = {"workload": w.name, "shape_bnhd": [w.B, w.N, w.H, w.d], "dtype": w.dtype,
             "seed": w.seed, "runs": runs, "plan": plan,
             "fwd": part([e[2].elapsed_time(e[3]) for e in ev],
                         [e[0].elapsed_time(e[1]) for e in ev], w.fwd_flop, io_bytes(w, False),
                         fwd_name + extra),
             "clocks": clocks}
    if train:
        entry["bwd"] = part([e[6].elapsed_time(e[7]) for e in ev],
                            [e[4].elapsed_time(e[5]) for e in ev], w.bwd_flop, io_bytes(w, True),
                            bwd_name)
    return entry, o, lse


def oracle_time_config(w: attn_inputs.Workload, budget_gflop: float, single_core: bool) -> dict:
    """Times the fp64 oracle, as it stands, on one configuration's inputs on
    the host cores: the whole configuration when its work is within
    budget_gflop, else the first rows of every head sized to about that much
    (the FLOP rate is then that of the sample).  With single_core, also on
    one thread."""
    import oracle  # the CPU-baseline leg is one of the oracle's permitted users
    q, k, v, do = attn_inputs.draw_workload(w, count=4)
    f64 = attn_inputs.to_f64
    Q, K, V, DO = f64(q), f64(k), f64(v), f64(do)
    flop = w.fwd_flop + (w.bwd_flop if w.backward else 0.0)
    whole = flop <= budget_gflop * 1e9

    def run():
        t0 = time.perf_counter()
        if whole:
            oracle.attn_fwd(Q, K, V, w.scale)
            if w.backward:
                oracle.attn_bwd(Q, K, V, DO, w.scale)
            done = flop
        else:
            rows = max(1, min(w.N, int(w.N * budget_gflop * 1e9 / flop)))
            sel = [(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(rows)]
            oracle.attn_fwd_rows(Q, K, V, w.scale, sel)
            if w.backward:
                oracle.attn_bwd_rows(Q, K, V, DO, w.scale, 0, rows)
            done = (14.0 if w.backward else 4.0) * rows * w.N * w.d * w.B * w.H
        return time.perf_counter() - t0, done

    threads = oracle.num_threads()
    dt, done = run()
    rows = w.N if whole else max(1, min(w.N, int(w.N * budget_gflop * 1e9 / flop)))
    out = {"tflops": done / dt / 1e12, "seconds": dt, "gflop": done / 1e9, "threads": threads,
           "sample": ("whole configuration" if whole else
                      f"query rows [0,{rows}) of all {w.B * w.H} heads"
                      + (" (forward rows and their backward)" if w.backward else "")),
           "extrapolated_seconds": dt * flop / done}
    if single_core:
        oracle.set_num_threads(1)
        try:
            dt1, done1 = run()
        finally:
            oracle.set_num_threads(threads)
        out["single_core"] = {"tflops": done1 / dt1 / 1e12, "seconds": dt1}
    return out


def c1_fp32_report(w: attn_inputs.Workload, o_gpu, lse_gpu) -> dict:
    """C1 draws fp32 inputs, which the GPU receives rounded to bf16.  Reports
    the oracle on the unrounded fp32 draws beside the oracle on the rounded
    inputs (the parity reference) and the GPU result: informational, not a
    gate."""
    import oracle
    raw = attn_inputs.draw_fp32(w.B, w.N, w.H, w.d, w.seed, count=3, std=w.std)
    q, k, v = attn_inputs.draw_workload(w, count=3)
    f64 = attn_inputs.to_f64
    o_raw, lse_raw = oracle.attn_fwd(*(x.astype(np.float64) for x in raw), w.scale)
    o_rnd, lse_rnd = oracle.attn_fwd(f64(q), f64(k), f64(v), w.scale)
    o_g = f64(o_gpu)
    l_g = lse_gpu.detach().cpu().double().numpy()
    return {"o_max_abs_rounded_vs_fp32_oracle": float(np.abs(o_rnd - o_raw).max()),
            "lse_max_abs_rounded_vs_fp32_oracle": float(np.abs(lse_rnd - lse_raw).max()),
            "o_max_abs_gpu_vs_rounded_oracle": float(np.abs(o_g - o_rnd).max()),
            "o_max_abs_gpu_vs_fp32_oracle": float(np.abs(o_g - o_raw).max()),
            "lse_max_abs_gpu_vs_fp32_oracle": float(np.abs(l_g - lse_raw).max())}


def cpu_oracle_sample(w: attn_inputs.Workload, rows: int, heads: int):
    """Times the fp64 oracle on a bounded sample of the workload: the first
    `rows` query rows of `heads` heads (forward rows and, for the training
    workload, their backward contributions).  Returns (TFLOP/s at the
    workload's FLOP-per-row rate, seconds, threads, description)."""
    import oracle  # the CPU baseline leg is one of the oracle's permitted users
    rows = max(1, min(rows, w.N))
    q, k, v, do = attn_inputs.draw_workload(w, count=4)
    f64 = attn_inputs.to_f64
    hs = [(b, h) for b in range(w.B) for h in range(w.H)][:heads]
    qs = np.stack([f64(q[b, :, h]) for b, h in hs], axis=1)[None]  # [1, N, S, d]
    ks = np.stack([f64(k[b, :, h]) for b, h in hs], axis=1)[None]
    vs = np.stack([f64(v[b, :, h]) for b, h in hs], axis=1)[None]
    ds = np.stack([f64(do[b, :, h]) for b, h in hs], axis=1)[None]
    sel = [(0, s, i) for s in range(len(hs)) for i in range(rows)]
    t0 = time.perf_counter()
    oracle.attn_fwd_rows(qs, ks, vs, w.scale, sel)
    if w.backward:
        oracle.attn_bwd_rows(qs, ks, vs, ds, w.scale, 0, rows)
    dt = time.perf_counter() - t0
    per_row = 14.0 if w.backward else 4.0  # 4 (fwd) + 10 (bwd) per row, N keys, d
    flop = per_row * rows * w.N * w.d * len(hs)
    step = (w.fwd_flop + w.bwd_flop) if w.backward else w.fwd_flop
    desc = (f"fp64 oracle {'fwd+bwd' if w.backward else 'fwd'} of query rows [0,{rows}) of "
            f"{len(hs)} of {w.B * w.H} heads (N={w.N}, d={w.d}); {flop / 1e9:.2f} GFLOP of the "
            f"step's {step / 1e9:.1f}")
    return flop / dt / 1e12, dt, oracle.num_threads(), desc


def run_reference(args, w, rank):
    """The reference arm: the fp64 CPU oracle, timed as it stands on the host cores."""
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    heads = max(1, min(oracle.num_threads(), w.B * w.H))
    # a few minutes in total: rows per step shrink as the step count grows
    rows = int(max(8, min(512, 512 * 40 / max(1, args.steps + args.warmup))))
    for _ in range(args.warmup):
        cpu_oracle_sample(w, rows, heads)
    vals, secs = [], []
    for _ in range(args.steps):
        v, dt, threads, desc = cpu_oracle_sample(w, rows, heads)
        vals.append(v)
        secs.append(dt)
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(secs),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(w, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc, "cpu_model": cpu_model(), "host_cores": host_cores()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="c5", choices=sorted(attn_inputs.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip timing each configuration on its own")
    ap.add_argument("--oracle-budget-gflop", type=float, default=ORACLE_BUDGET_GFLOP,
                    help="per-configuration oracle work above which a row sample is timed")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = attn_inputs.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w, rank)

    import exact_attention_144_b200 as fa
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    # Each rank owns one replica of the workload (its own seeded batch).
    q, k, v, do = attn_inputs.draw(w.B, w.N, w.H, w.d, w.dtype, replica_seed(w, rank), 4,
                                   std=w.std, device=dev)
    fwd, bwd, out_dtype = entry_points(fa, w)
    o = torch.empty(q.shape, dtype=out_dtype, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    train = w.backward and bwd is not None

    def step():
        fwd(q, k, v, o=o, lse=lse, scale=w.scale)
        if train:
            bwd(q, k, v, o, do, lse, dq=dq, dk=dk, dv=dv, scale=w.scale)

    flop_step = w.fwd_flop + (w.bwd_flop if train else 0.0)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---------------------------------------------- device-timed steps
    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev = [(mk(), mk(), mk(), mk(), mk(), mk()) for _ in range(args.steps)]
    launches0 = fa.fa_kernel_launches()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for s0, s1, f0, f1, b0, b1 in ev:
            flush.zero_()  # write 512 MiB between steps: no input stays in L2
            fa.fa_set_kernel_events(f0, f1, b0 if train else None, b1 if train else None)
            s0.record()
            step()
            s1.record()
        torch.cuda.synchronize()
    barrier()
    launches = fa.fa_kernel_launches() - launches0
    step_ms = [s0.elapsed_time(s1) for s0, s1, *_ in ev]
    fwd_ms = [f0.elapsed_time(f1) for _, _, f0, f1, _, _ in ev]
    bwd_ms = [b0.elapsed_time(b1) for *_, b0, b1 in ev] if train else []
    ms = max_over_ranks(statistics.mean(step_ms), dist, dev)
    value = job_tflops(flop_step, ms, world)
    status = fa.fa_get_device_status()
    if status != 0:
        raise RuntimeError(f"a kernel gave up a bounded wait (status {status:#x})")

    # ------------------------------ end to end, host buffers, pipelined steps
    # Every step copies its inputs from pinned host memory to the device, runs
    # forward (+ backward), and copies its results back to pinned host memory.
    # Three streams and two device buffer sets let step i+1's upload and step
    # i-1's download run while step i computes; events order each buffer's
    # reuse.  The timed region spans the first upload to the last download.
    e2e_ms, h2d, d2h, copies = e2e_pipelined(fa, w, args, dev, q, k, v, do, train, mk)
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    pk, pk_src = peaks()

    # ------------------------------ every configuration on its own (one GPU)
    per_config = {}
    c1_out = None
    if world == 1 and not args.no_per_config:
        for name in PER_CONFIG:
            entry, o_c, lse_c = time_config(fa, attn_inputs.WORKLOADS[name], dev, flush,
                                            PER_CONFIG_RUNS, local, pk)
            per_config[name] = entry
            if name == "c1":
                c1_out = (o_c.cpu(), lse_c.cpu())
        if fa.fa_get_device_status() != 0:
            raise RuntimeError("a kernel gave up a bounded wait during the per-config timing")

    # ----------------------------------------- roofline of the dominant kernel
    fwd_name, bwd_name = main_kernel_names(fa, w, torch.cuda.get_device_properties(dev))
    if train:
        dom, dom_ms, dom_flop = bwd_name, statistics.mean(bwd_ms), w.bwd_flop
    else:
        dom, dom_ms, dom_flop = fwd_name, statistics.mean(fwd_ms), w.fwd_flop
    achieved = dom_flop / (dom_ms * 1e-3) / 1e12
    tr = TRAFFIC.get((dom, w.name))
    traffic = tr["bytes"] if tr and tr["src"] == kernel_source_hash() else None
    peak, peak_sus, peak_name = tensor_peak(pk, w)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                "kernel": dom, "kernel_ms": dom_ms,
                "peak_source": f"{peak_name} (burst) of {pk_src} MEASURED_PEAKS.json",
                "frac_of_sustained": achieved / peak_sus}
    kernels = {fwd_name: {"ms": statistics.mean(fwd_ms),
                          "tflops": w.fwd_flop / (statistics.mean(fwd_ms) * 1e-3) / 1e12}}
    if train:
        kernels[bwd_name] = {"ms": statistics.mean(bwd_ms), "tflops": achieved}
    for kv in kernels.values():
        kv["frac"] = kv["tflops"] / peak

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = None
        try:
            import oracle
            oracle.build()
            threads = oracle.num_threads()
        except Exception as exc:  # the baseline is reported, never the target
            cpu = {"error": str(exc)}
        if threads:
            val, dt, threads, desc = cpu_oracle_sample(w, 1024 if train else 256,
                                                       max(1, min(threads, w.B * w.H)))
            cpu = {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle",
                   "sample": desc, "seconds": dt, "cpu_model": cpu_model(),
                   "host_cores": host_cores()}
            # the oracle on each configuration (after all GPU work)
            for name, entry in per_config.items():
                cw = attn_inputs.WORKLOADS[name]
                entry["oracle"] = oracle_time_config(cw, args.oracle_budget_gflop,
                                                     single_core=name in ("c1", "c2"))
                if name == "c1" and c1_out is not None:
                    entry["c1_fp32_draws"] = c1_fp32_report(cw, *c1_out)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": {"bf16": "bf16", "fp16": "fp16", "fp8": "fp8e4m3"}[w.dtype],
            "data": "synthetic",
            "config": workload_config(w, world),
            "e2e": {"value": job_tflops(flop_step, e2e_ms, world), "unit": UNIT,
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "how": "pinned host -> device inputs, step, device -> pinned host results "
                           "every step; uploads, kernels and downloads of neighbouring steps "
                           "overlap (two device buffer sets); each input uploads and each "
                           "result downloads on a stream of its own",
                    "copies_alone": copies},
            "gpu_launches": launches,
            "roofline": roofline,
            "kernels": kernels,
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
            "pct_of_bf16_peak": 100.0 * value / world / pk["bf16_tflops"],
            "pct_of_dtype_peak": 100.0 * value / world / peak,
        }
        if per_config:
            line["per_config"] = per_config
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
