#!/usr/bin/env python
"""Benchmark of the W4A16 weight-only matmul on B200.

Metric: W4A16 GEMM achieved HBM GB/s (and fraction of roofline) at decode and
speculative-verify row counts, one B200.

One step = the four decode linears of the 5120-hidden, 64-layer dense model at
M = 1 (int4 GPTQ g128): QKV 5120->8192, O 6144->5120, gate/up 5120->34816,
down 17408->5120, run back to back on one stream.  ``value`` is algorithmic
bytes (packed weights + scales + activations + outputs) per second over the
timed steps, aggregated over all GPUs.  The other configurations (every row
count, NVFP4, the 64-layer sweep) and the widened rows (M up to 2048, FP8
weights, the fused gate/up layer) are reported in ``sweep``, ``gate_up_silu``
and ``whole_stack``.  ``--case fmt,M,N,K[,path][;...]`` launches GEMMs a few
times for a profiler; ``--traffic-csv`` turns an ncu capture of the decode
shapes into profiles/traffic.json.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
Multi-GPU: launched by torchrun, one process per GPU; each GPU runs its own
replica of the workload (the path needs no exchange between GPUs).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DECODE_SHAPES = [("qkv", 5120, 8192, 1), ("o", 6144, 5120, 2), ("gate_up", 5120, 34816, 3),
                 ("down", 17408, 5120, 4)]
METRIC = "W4A16 GEMM achieved HBM GB/s & % of roofline at M=1/4/9/16/64 (1 B200)"
UNIT = "GB/s"
WORKLOAD = ("decode-shape int4 g128 W4A16, M=1: QKV 5120->8192, O 6144->5120, "
            "gate/up 5120->34816, down 17408->5120 (seeds 1-4)")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def alg_bytes(fmt, M, N, K):
    if fmt == "fp8":                                  # a byte per weight, one fp32 scale
        w = N * K + 4
    else:
        w = N * K * (0.5 + (2 / 128 if fmt == "int4" else 1 / 16)) + (4 if fmt == "nvfp4" else 0)
    return w + 2 * M * K + 2 * M * N


def flops(M, N, K):
    return 2.0 * M * N * K


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def load_traffic():
    """Per-launch DRAM bytes of the dominant kernel from the committed ncu summary,
    valid only while the kernel sources hash the same as when it was captured."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("source_hash") != kernel_source_hash():
        return None
    return d


def kernel_source_hash():
    """Hash of the sources that define the GEMV kernel (the kernel whose DRAM
    traffic profiles/traffic.json records): its file and the headers it uses."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_weight_only_dequant_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name in ("gemv.cu", "common.cuh", "layout.h", "kernels.h"):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode())
                h.update(f.read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, out_path=None):
        self.samples = []
        self.proc = None
        self.gpu_id = gpu_id
        self.out_path = out_path

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.gpu_id],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)
        if self.out_path:
            with open(self.out_path, "w") as f:
                for ts, line in self.samples:
                    f.write(f"{ts:.3f},{line}\n")

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.samples:
            if t0 <= ts <= t1:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ---------------------------------------------------------------- the CPU oracle baseline


def cpu_oracle_sample(seconds: float):
    """Run the fp64 oracle on blocks of output columns of the decode shapes until
    ``seconds`` of oracle time have passed (input generation not counted);
    returns (GB/s of weight+scale bytes processed, description, seconds)."""
    import oracle
    import synth
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except Exception:  # pragma: no cover
        pass
    block = 256
    done_bytes = 0.0
    done_rows = {name: 0 for name, *_ in DECODE_SHAPES}
    xs = {K: synth.activations(seed, 1, K) for _, K, _, seed in DECODE_SHAPES}
    busy = 0.0
    wall0 = time.perf_counter()
    i = 0
    while busy < seconds and time.perf_counter() - wall0 < 4 * seconds:
        name, K, N, seed = DECODE_SHAPES[i % len(DECODE_SHAPES)]
        r0 = done_rows[name] % N
        rows = np.arange(r0, min(N, r0 + block))
        p = synth.problem("int4", seed, 1, N, K, rows=rows)
        t0 = time.perf_counter()
        wd = oracle.dequant_int4_g128(p["codes"], p["scales"])
        oracle.gemm_ref(xs[K], wd)
        busy += time.perf_counter() - t0
        done_rows[name] += len(rows)
        done_bytes += len(rows) * K * (0.5 + 2 / 128)
        i += 1
    desc = (f"fp64 oracle (dequantise then matmul), 1 thread, on blocks of {block} output columns "
            f"of the four decode shapes at M=1, round robin, {busy:.1f} s of oracle time: "
            + ", ".join(f"{k} {v} rows" for k, v in done_rows.items())
            + "; GB/s of packed weight+scale bytes; input generation not counted")
    return done_bytes / busy / 1e9, desc, busy


def _oracle_worker_init():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except Exception:  # pragma: no cover
        pass


def _oracle_blocks(task):
    """One worker's share of an all-cores oracle run: ``blocks`` blocks of
    ``rows`` output columns of one shape (inputs generated first, not timed).
    Returns (weight+scale bytes processed, seconds of oracle work)."""
    import oracle
    import synth
    fmt, M, N, K, seed, first_row, rows, blocks = task
    x = synth.activations(seed, M, K)
    probs = []
    for b in range(blocks):
        r0 = (first_row + b * rows) % N
        probs.append(synth.problem(fmt, seed, M, N, K, rows=np.arange(r0, min(N, r0 + rows))))
    t0 = time.perf_counter()
    done = 0.0
    for p in probs:
        wd = (oracle.dequant_int4_g128(p["codes"], p["scales"]) if fmt == "int4"
              else oracle.dequant_nvfp4(p["codes"], p["scales"], p["g"]))
        oracle.gemm_ref(x, wd)
        done += p["codes"].shape[0] * K * (0.5 + (2 / 128 if fmt == "int4" else 1 / 16))
    return done, time.perf_counter() - t0


def weight_bytes(fmt, N, K):
    return N * K * (0.5 + (2 / 128 if fmt == "int4" else 1 / 16))


def cpu_oracle_all_cores(rows=256, blocks=2):
    """The oracle on every host core at once (one process per core, started
    with spawn, one BLAS thread each), per configuration: every core takes
    ``blocks`` blocks of ``rows`` output columns of each shape of the
    configuration; the configuration's oracle time is extrapolated from the
    bytes the cores processed per second (the slowest core's time).  The
    whole-stack configuration is extrapolated from the int4 rates at
    M = 1 / 16 / 64."""
    import concurrent.futures as cf
    import multiprocessing as mp
    cores = os.cpu_count() or 1
    configs = [("decode int4 M=1", "int4", [1], [(K, N, s) for _, K, N, s in DECODE_SHAPES])]
    configs += [(f"verify int4 M={M}", "int4", [M], [(K, N, 5) for _, K, N, _ in DECODE_SHAPES])
                for M in (2, 4, 9, 16, 64)]
    configs += [(f"nvfp4 M={M}", "nvfp4", [M], [(K, N, 6) for _, K, N, _ in DECODE_SHAPES])
                for M in (1, 9, 64)]
    out = {"cores": cores, "threads_per_core": 1, "rows_per_block": rows, "blocks_per_core": blocks,
           "by_config": {}}
    with cf.ProcessPoolExecutor(max_workers=cores, mp_context=mp.get_context("spawn"),
                                initializer=_oracle_worker_init) as ex:
        list(ex.map(_oracle_blocks, [("int4", 1, 256, 128, 0, 0, 16, 1)] * cores))   # warm the pool
        for label, fmt, (M,), shapes in configs:
            done = busy = 0.0
            full = 0.0
            for K, N, seed in shapes:
                tasks = [(fmt, M, N, K, seed, c * rows * blocks, rows, blocks) for c in range(cores)]
                res = list(ex.map(_oracle_blocks, tasks))
                done += sum(r[0] for r in res)
                busy += max(r[1] for r in res)
                full += weight_bytes(fmt, N, K)
            gbps = done / busy / 1e9
            out["by_config"][label] = {"GBps": round(gbps, 4),
                                       "s_per_step_extrapolated": round(full / (gbps * 1e9), 4)}
    stack = sum(weight_bytes("int4", N, K) for _, K, N, _ in DECODE_SHAPES) * 64 + \
        weight_bytes("int4", 248320, 5120)
    for M, key in ((1, "decode int4 M=1"), (16, "verify int4 M=16"), (64, "verify int4 M=64")):
        r = out["by_config"][key]["GBps"]
        out["by_config"][f"whole stack int4 M={M} (extrapolated)"] = {
            "GBps": r, "s_per_step_extrapolated": round(stack / (r * 1e9), 2)}
    return out


def cpu_oracle_step(rows_per_shape: int):
    """One reference step: the oracle on the first rows of every decode shape."""
    import oracle
    import synth
    total = 0.0
    t_work = 0.0
    for name, K, N, seed in DECODE_SHAPES:
        rows = np.arange(min(N, rows_per_shape))
        p = synth.problem("int4", seed, 1, N, K, rows=rows)
        t0 = time.perf_counter()
        wd = oracle.dequant_int4_g128(p["codes"], p["scales"])
        oracle.gemm_ref(p["x"], wd)
        t_work += time.perf_counter() - t0
        total += len(rows) * K * (0.5 + 2 / 128)
    return total, t_work


def max_over_ranks(values, world, device):
    """Element-wise maximum of a list of floats over all ranks; every rank gets it.

    Multi-GPU runs are replicas: each rank times its own copy of the workload
    and the job's time is the slowest rank's."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_gbps(world, bytes_per_step, steps, seconds):
    """Aggregate throughput of `world` replicas that each moved `bytes_per_step`
    for `steps` steps within `seconds` (the slowest rank's time)."""
    return world * bytes_per_step * steps / seconds / 1e9


def run_reference(args, rank, world):
    if rank != 0:
        return
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except Exception:
        pass
    rows = 256
    for _ in range(args.warmup):
        cpu_oracle_step(rows)
    tot_b = tot_t = 0.0
    for _ in range(args.steps):
        b, t = cpu_oracle_step(rows)
        tot_b += b
        tot_t += t
    value = tot_b / tot_t / 1e9
    sample = (f"fp64 oracle on the first {rows} output columns of each decode shape per step "
              f"(weights + scales of {tot_b / args.steps / 1e6:.1f} MB per step), 1 thread")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded SplitMix64)",
            "config": {"workload": WORKLOAD, "M": 1, "fmt": "int4_g128"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU side


def make_weights(fmt, seed, N, K, copies):
    import torch
    import synth
    from bit_weight_only_dequant_b200 import w4a16 as W
    p = synth.device_problem("nvfp4" if fmt == "nvfp4_bs" else fmt, seed, 1, N, K)
    pw, ps = W.pack_on_device(fmt, N, K, p["codes"], p["scales"])
    del p
    ws = [(pw, ps)]
    for _ in range(copies - 1):
        ws.append((pw.clone(), ps.clone()))
    torch.cuda.synchronize()
    return ws


def make_x(fmt, seed, M, K):
    import torch
    import synth
    x = torch.empty((M, K), dtype=torch.int16, device="cuda")
    synth.device_fill(synth.KIND_X, seed, synth.T_X, x)
    return x.view(torch.bfloat16)


def copies_for(weight_bytes):
    """Weight copies to rotate so one cycle is at least 3x the L2 size."""
    return max(2, min(16, int(np.ceil(3 * L2_BYTES / max(1, weight_bytes)))))


REPEATS = 5


def spread(values):
    """Median and range of repeated timings (ms)."""
    v = sorted(values)
    return {"median": statistics.median(v), "min": v[0], "max": v[-1], "n": len(v)}


def time_back_to_back(launch, reps, stream, repeats=REPEATS):
    """Capture ``reps`` calls of ``launch(r)`` back to back in one CUDA graph
    (no event between launches, so a launch may start its weight prologue
    while the previous one finishes, as in a decode step), replay it once to
    warm up, then time ``repeats`` replays, each with its own CUDA events on
    the launching stream and a synchronize on both sides.  Returns the
    milliseconds per call of every replay."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for r in range(reps):
            launch(r)
    with torch.cuda.stream(stream):
        g.replay()  # warm replay
    torch.cuda.synchronize()
    out = []
    for _ in range(repeats):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            start.record()
            g.replay()
            end.record()
        torch.cuda.synchronize()
        out.append(start.elapsed_time(end) / reps)
    del g
    return out


def sweep_entry(fmt, name, K, N, M, seed, peaks, stream, reps=24):
    import torch
    from bit_weight_only_dequant_b200 import w4a16 as W
    f = W.FMTS[fmt]
    wbytes = W.w4a16_packed_weight_bytes(f, N, K) + W.w4a16_packed_scale_bytes(f, N, K)
    copies = copies_for(wbytes)
    ws = make_weights(fmt, seed, N, K, copies)
    x = make_x(fmt, seed, M, K)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    g = torch.tensor([1.0 / 448.0], dtype=torch.float32, device="cuda") if fmt != "int4" else None
    path = W.w4a16_gemm_path(f, M, N, K)

    def launch(r, ws=ws):
        pw, ps = ws[r % len(ws)]
        W.check(W.w4a16_gemm(f, M, N, K, x, pw, ps, g, y, stream.cuda_stream), "gemm")

    with torch.cuda.stream(stream):
        for r in range(3):
            launch(r)
    torch.cuda.synchronize()
    rep = spread([v * 1e3 for v in time_back_to_back(launch, reps, stream)])
    us = rep["median"]
    b = alg_bytes(fmt, M, N, K)
    fl = flops(M, N, K)
    t_mem = b / (peaks["hbm_gbs"] * 1e9)
    t_tc = fl / (peaks["bf16_tflops"] * 1e12)
    t_roof = max(t_mem, t_tc)
    del ws
    torch.cuda.empty_cache()
    return {"fmt": fmt, "shape": name, "K": K, "N": N, "M": M, "path": int(path),
            "us": round(us, 3), "us_min": round(rep["min"], 3), "us_max": round(rep["max"], 3),
            "GBps": round(b / us / 1e3, 1), "TFLOPs": round(fl / us / 1e6, 2),
            "bound": "hbm" if t_mem >= t_tc else "tensor",
            "frac_roofline": round(t_roof * 1e6 / us, 4),
            "frac_of_8TBps": round(b / us / 1e3 / 8000.0, 4)}


def w4a4_entry(name, K, N, M, seed, peaks, stream, reps=24, block_scaled=False):
    """W4A4 NVFP4 (activations quantised inside the call) at one decode shape:
    the quantiser and the matmul, back to back like the sweep.  Algorithmic
    bytes: the NVFP4 weights and scales, x and y.  block_scaled: the
    tcgen05 kind::mxf4nvf4 path (weights in its own layout, same bytes);
    its tensor roofline is the FP4 peak (the measured BF16 peak times the
    nominal 4x ratio)."""
    import torch
    from bit_weight_only_dequant_b200 import w4a16 as W
    wfmt = "nvfp4_bs" if block_scaled else "nvfp4"
    f = W.FMTS[wfmt]
    wbytes = W.w4a16_packed_weight_bytes(f, N, K) + W.w4a16_packed_scale_bytes(f, N, K)
    ws = make_weights(wfmt, seed, N, K, copies_for(wbytes))
    x = make_x("nvfp4", seed, M, K)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    g = torch.tensor([1.0 / 448.0], dtype=torch.float32, device="cuda")

    def launch(r, ws=ws):
        pw, ps = ws[r % len(ws)]
        if block_scaled:
            W.check(W.w4a16_gemm_w4a4_bs(M, N, K, x, pw, ps, g, y, stream.cuda_stream), "gemm_w4a4_bs")
        else:
            W.check(W.w4a16_gemm_w4a4(M, N, K, x, pw, ps, g, y, stream.cuda_stream), "gemm_w4a4")

    with torch.cuda.stream(stream):
        for r in range(3):
            launch(r)
    torch.cuda.synchronize()
    rep = spread([v * 1e3 for v in time_back_to_back(launch, reps, stream)])
    us = rep["median"]
    b = alg_bytes("nvfp4", M, N, K)
    fl = flops(M, N, K)
    tpeak = peaks["bf16_tflops"] * (4.0 if block_scaled else 1.0)
    t_roof = max(b / (peaks["hbm_gbs"] * 1e9), fl / (tpeak * 1e12))
    del ws
    torch.cuda.empty_cache()
    path = W.PATH_BS if block_scaled else int(W.w4a16_gemm_path(W.FMTS["nvfp4"], M, N, K))
    return {"fmt": "w4a4_nvfp4_bs" if block_scaled else "w4a4_nvfp4", "shape": name, "K": K, "N": N,
            "M": M, "path": path, "us": round(us, 3),
            "us_min": round(rep["min"], 3), "us_max": round(rep["max"], 3),
            "GBps": round(b / us / 1e3, 1), "frac_roofline": round(t_roof * 1e6 / us, 4)}


def gate_up_entry(fmt, M, seed, peaks, stream, reps=24):
    """The fused gate/up layer h = SiLU(gate) * up at the decode gate/up shape
    (K = 5120, I = 17408: the 34816-row weight), back to back like the sweep.
    Algorithmic bytes: the weight and scales, x, and h (M x I BF16)."""
    import torch
    from bit_weight_only_dequant_b200 import w4a16 as W
    f = W.FMTS[fmt]
    K, N = 5120, 34816
    I = N // 2
    wbytes = W.w4a16_packed_weight_bytes(f, N, K) + W.w4a16_packed_scale_bytes(f, N, K)
    ws = make_weights(fmt, seed, N, K, copies_for(wbytes))
    x = make_x(fmt, seed, M, K)
    h = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    g = torch.tensor([1.0 / 448.0], dtype=torch.float32, device="cuda") if fmt != "int4" else None
    path = W.w4a16_gemm_path(f, M, N, K)

    def launch(r, ws=ws):
        pw, ps = ws[r % len(ws)]
        W.check(W.w4a16_gemm_gate_up_silu(f, M, I, K, x, pw, ps, g, h, stream.cuda_stream),
                "gate_up_silu")

    with torch.cuda.stream(stream):
        for r in range(3):
            launch(r)
    torch.cuda.synchronize()
    rep = spread([v * 1e3 for v in time_back_to_back(launch, reps, stream)])
    us = rep["median"]
    b = alg_bytes(fmt, M, N, K) - 2 * M * N + 2 * M * I
    fl = flops(M, N, K)
    t_roof = max(b / (peaks["hbm_gbs"] * 1e9), fl / (peaks["bf16_tflops"] * 1e12))
    del ws
    torch.cuda.empty_cache()
    return {"fmt": fmt, "M": M, "K": K, "I": I, "path": int(path), "us": round(us, 3),
            "us_min": round(rep["min"], 3), "us_max": round(rep["max"], 3),
            "GBps": round(b / us / 1e3, 1), "frac_roofline": round(t_roof * 1e6 / us, 4)}


def whole_stack(Ms, peaks, stream, reps=3):
    """64 layers x (QKV, O, gate/up, down) + the 5120->248320 output projection,
    int4 g128, weights of layer l drawn with seed 7+l and the output projection
    with seed 71; the linears do not feed each other (one x per distinct K)."""
    import torch
    from bit_weight_only_dequant_b200 import w4a16 as W
    layers = []
    for l in range(64):
        for name, K, N, _ in DECODE_SHAPES:
            (pw, ps), = make_weights("int4", 7 + l, N, K, 1)
            layers.append((K, N, pw, ps))
    (pw, ps), = make_weights("int4", 71, 248320, 5120, 1)
    layers.append((5120, 248320, pw, ps))
    wbytes = sum(W.w4a16_packed_weight_bytes(0, N, K) + W.w4a16_packed_scale_bytes(0, N, K)
                 for K, N, _, _ in layers)
    out = {"layers": 64, "gemms_per_step": len(layers), "weight_and_scale_bytes_per_step": int(wbytes),
           "weights_per_step": int(sum(N * K for K, N, _, _ in layers)), "by_M": {}}
    for M in Ms:
        xs = {K: make_x("int4", 7, M, K) for K in (5120, 6144, 17408)}
        ys = {N: torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
              for N in (8192, 5120, 34816, 248320)}

        def step(r, M=M, xs=xs, ys=ys):
            for K, N, pw, ps in layers:
                W.check(W.w4a16_gemm(0, M, N, K, xs[K], pw, ps, None, ys[N], stream.cuda_stream),
                        "gemm")

        with torch.cuda.stream(stream):
            step(0)
        torch.cuda.synchronize()
        rep = spread(time_back_to_back(step, reps, stream))
        ms = rep["median"]
        b = sum(alg_bytes("int4", M, N, K) for K, N, _, _ in layers)
        fl = sum(flops(M, N, K) for K, N, _, _ in layers)
        out["by_M"][str(M)] = {"ms_per_step": round(ms, 4), "ms_min": round(rep["min"], 4),
                               "ms_max": round(rep["max"], 4), "steps_per_s": round(1e3 / ms, 2),
                               "GBps": round(b / ms / 1e6, 1), "TFLOPs": round(fl / ms / 1e9, 2),
                               "weight_bound_steps_per_s_at_peak": round(
                                   peaks["hbm_gbs"] * 1e9 / wbytes, 1)}
    del layers
    torch.cuda.empty_cache()
    return out


def run_native(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from bit_weight_only_dequant_b200 import w4a16 as W

    torch.cuda.set_device(local_rank)
    W.lib()
    peaks = load_peaks()
    stream = torch.cuda.Stream()
    M = 1

    # ---- the workload: four decode linears, weights rotated over enough copies
    wsets = []
    for name, K, N, seed in DECODE_SHAPES:
        wsets.append((name, K, N, seed))
    step_wbytes = sum(W.w4a16_packed_weight_bytes(0, N, K) + W.w4a16_packed_scale_bytes(0, N, K)
                      for _, K, N, _ in wsets)
    copies = copies_for(step_wbytes)
    weights = {name: make_weights("int4", seed, N, K, copies) for name, K, N, seed in wsets}
    # the step's activations and outputs live in one device buffer each (views
    # per linear), so the end-to-end leg moves them with one copy each way
    x_all = torch.empty(sum(M * K for _, K, _, _ in wsets), dtype=torch.bfloat16, device="cuda")
    y_all = torch.empty(sum(M * N for _, _, N, _ in wsets), dtype=torch.bfloat16, device="cuda")
    xs, ys, xo, yo = {}, {}, 0, 0
    for name, K, N, seed in wsets:
        xs[name] = x_all[xo:xo + M * K].view(M, K)
        xs[name].copy_(make_x("int4", seed, M, K))
        ys[name] = y_all[yo:yo + M * N].view(M, N)
        xo += M * K
        yo += M * N
    step_bytes = sum(alg_bytes("int4", M, N, K) for _, K, N, _ in wsets)

    def gemm_fn(name, K, N):
        def fn(r):
            pw, ps = weights[name][r % copies]
            W.check(W.w4a16_gemm(0, M, N, K, xs[name], pw, ps, None, ys[name],
                                 stream.cuda_stream), "gemm")
        return fn

    launches = [gemm_fn(name, K, N) for name, K, N, _ in wsets]
    with torch.cuda.stream(stream):
        for w in range(max(3, args.warmup)):
            for fn in launches:
                fn(w)
    torch.cuda.synchronize()
    W.check(W.w4a16_device_status(stream.cuda_stream), "device status")

    # ---- capture the K timed steps back to back (a launch may start its
    # weight prologue while the previous one finishes), soak, time one replay
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(args.steps):
            for fn in launches:
                fn(i)
    props = torch.cuda.get_device_properties(local_rank)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local_rank)
    # the raw clock samples go to a CSV only when W4A16_CLOCKS_DIR names a folder;
    # their summary is always part of the JSON line
    clocks_dir = os.environ.get("W4A16_CLOCKS_DIR")
    clocks_csv = None
    if clocks_dir:
        os.makedirs(clocks_dir, exist_ok=True)
        clocks_csv = os.path.join(clocks_dir, f"clocks_rank{rank}.csv")
    sampler = ClockSampler(gpu_id, clocks_csv)
    sampler.start()
    time.sleep(0.3)
    t_soak = time.time()
    soak_until = t_soak + args.soak
    while time.time() < soak_until:
        graph.replay()
        torch.cuda.synchronize()
    # REPEATS timed replays of the K steps, each bracketed by a barrier and a
    # synchronize; the line reports the median replay (max over ranks)
    replay_ms = []
    for _ in range(REPEATS):
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            start.record()
            graph.replay()
            end.record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        replay_ms.append(start.elapsed_time(end))
    t_end = time.time()
    time.sleep(0.25)
    sampler.stop()
    W.check(W.w4a16_device_status(stream.cuda_stream), "device status")
    replay_ms = max_over_ranks(replay_ms, world, "cuda")
    rep = spread(replay_ms)
    ms_total = rep["median"]
    ms_per_step = ms_total / args.steps
    value = whole_job_gbps(world, step_bytes, args.steps, ms_total * 1e-3)
    clocks = sampler.summary(t_soak, t_end)
    del graph

    # ---- dominant kernel: the GEMV (every launch of the step).  Its average
    # launch duration is the timed replay over the launches it holds; per-shape
    # durations come from each shape alone, back to back, on the same stream.
    launch_bytes = np.array([alg_bytes("int4", M, N, K) for _, K, N, _ in wsets])
    n_launch = len(launches) * args.steps
    avg_ms = ms_total / n_launch
    achieved = float(launch_bytes.mean() / (avg_ms * 1e-3) / 1e9)
    per_shape_rep = [spread(time_back_to_back(fn, max(24, 2 * copies), stream)) for fn in launches]
    per_shape_ms = [r["median"] for r in per_shape_rep]
    traffic = load_traffic()
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": (traffic or {}).get("dram_bytes_per_launch"),
                "peak_source": peaks["source"] + " (STREAM-style copy)",
                "kernel": "gemv_kernel<int4, 1 m-tile> (all four launches of the step)",
                "avg_launch_us": round(avg_ms * 1e3, 3),
                "per_shape_us": {name: round(per_shape_ms[j] * 1e3, 3)
                                 for j, (name, *_) in enumerate(wsets)},
                "per_shape_us_range": {name: [round(per_shape_rep[j]["min"] * 1e3, 3),
                                              round(per_shape_rep[j]["max"] * 1e3, 3)]
                                       for j, (name, *_) in enumerate(wsets)},
                "per_shape_frac": {name: round(float(launch_bytes[j] / (per_shape_ms[j] * 1e-3)
                                                     / 1e9 / peaks["hbm_gbs"]), 4)
                                   for j, (name, *_) in enumerate(wsets)}}

    # ---- end to end through the C ABI with host buffers
    xh = torch.empty(x_all.numel(), dtype=torch.bfloat16).pin_memory()
    yh = torch.empty(y_all.numel(), dtype=torch.bfloat16).pin_memory()
    xh.copy_(x_all.cpu())
    h2d = x_all.numel() * 2
    d2h = y_all.numel() * 2

    def e2e_step(i):
        with torch.cuda.stream(stream):
            x_all.copy_(xh, non_blocking=True)
            for fn in launches:
                fn(i)
            yh.copy_(y_all, non_blocking=True)
        stream.synchronize()

    for i in range(3):
        e2e_step(i)
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for i in range(args.steps):
        e2e_step(i)
    e2e_s = time.perf_counter() - t0
    e2e_s = max_over_ranks([e2e_s], world, "cuda")[0]
    e2e = {"value": round(whole_job_gbps(world, step_bytes, args.steps, e2e_s), 1), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": round(e2e_s / args.steps * 1e3, 4),
           "how": "pinned host x of the step -> device (one copy), the four w4a16_gemm calls via "
                  "the C ABI, device -> pinned host y (one copy), stream synchronize, per step, "
                  "wall clock"}
    del weights
    torch.cuda.empty_cache()

    extra = {}
    if world == 1 and not args.no_sweep:
        entries = []
        target = [("int4", "target", 5120, 17408, 1, 3)]
        cfg2 = [("int4", n, K, N, 1, s) for n, K, N, s in DECODE_SHAPES]
        cfg3 = [("int4", n, K, N, Mv, 5) for Mv in (2, 4, 9, 16, 64) for n, K, N, _ in DECODE_SHAPES]
        cfg4 = [("nvfp4", n, K, N, Mv, 6) for Mv in (1, 9, 64) for n, K, N, _ in DECODE_SHAPES]
        cfg5 = [(fmt, n, K, N, Mv, 7) for fmt in ("int4", "nvfp4") for Mv in (128, 256)
                for n, K, N, _ in DECODE_SHAPES]
        cfg5 += [("int4", n, K, N, 2048, 8) for n, K, N, _ in DECODE_SHAPES]
        # FP8-E4M3 weights (W8A16) on the attention linears
        cfg5 += [("fp8", n, K, N, Mv, 9) for Mv in (1, 9, 64) for n, K, N, _ in DECODE_SHAPES[:2]]
        for fmt, n, K, N, Mv, s in target + cfg2 + cfg3 + cfg4 + cfg5:
            entries.append(sweep_entry(fmt, n, K, N, Mv, s, peaks, stream))
        extra["sweep"] = entries
        extra["w4a4_block_scaled"] = [w4a4_entry(n, K, N, Mv, 6, peaks, stream, block_scaled=True)
                                      for Mv in (1, 9, 64) for n, K, N, _ in DECODE_SHAPES]
        extra["w4a4"] = [w4a4_entry(n, K, N, Mv, 6, peaks, stream) for Mv in (1, 9, 64)
                         for n, K, N, _ in DECODE_SHAPES]
        extra["gate_up_silu"] = [gate_up_entry(fmt, Mv, 3, peaks, stream)
                                 for fmt, Mv in (("int4", 1), ("int4", 4), ("int4", 9),
                                                 ("int4", 16), ("int4", 64), ("int4", 256),
                                                 ("nvfp4", 1), ("nvfp4", 64))]
    if world == 1 and not args.no_stack:
        extra["whole_stack"] = whole_stack((1, 16, 64), peaks, stream)

    cpu = None
    if rank == 0 and world == 1:
        v, desc, secs = cpu_oracle_sample(args.cpu_seconds)
        cpu = {"value": round(v, 4), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc}
        if not args.no_cpu_all:
            cpu["all_cores"] = cpu_oracle_all_cores()

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded SplitMix64 draws with the checkpoint geometry)",
                "config": {"workload": WORKLOAD, "M": 1, "fmt": "int4_g128",
                           "bytes_per_step": int(step_bytes),
                           "l2": f"inputs larger than L2: {copies} weight copies rotated "
                                 f"({copies * step_wbytes / 1e6:.0f} MB per cycle, L2 126 MB)",
                           "timing": "CUDA graph of the K steps back to back, CUDA events on "
                                     "the launching stream around the replay, max over ranks; "
                                     "the roofline's launch duration is that replay over the "
                                     "launches it holds; per-shape durations from each shape "
                                     "alone, back to back in its own graph, one event pair",
                           "replicas": world},
                "timing_repeats": {"ms_per_step": [round(v / args.steps, 5) for v in replay_ms],
                                   "median": round(rep["median"] / args.steps, 5),
                                   "min": round(rep["min"] / args.steps, 5),
                                   "max": round(rep["max"] / args.steps, 5)},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
                "gpu_launches": len(launches) * args.steps,
                "peaks": peaks}
        line.update(extra)
        print(json.dumps(line), flush=True)


def run_case(specs: str, launches: int):
    """Launch GEMMs a few times each (for profilers).  specs = one or more
    fmt,M,N,K[,path] separated by ';', run in that order; fmt is int4, nvfp4,
    fp8, w4a4 (NVFP4 weights, activations quantised by the library) or w4a4bs
    (the same on the block-scaled tensor cores)."""
    import torch
    from bit_weight_only_dequant_b200 import w4a16 as W
    torch.cuda.set_device(0)
    out = []
    for spec in specs.split(";"):
        parts = spec.split(",")
        fmt, M, N, K = parts[0], int(parts[1]), int(parts[2]), int(parts[3])
        path = int(parts[4]) if len(parts) > 4 else W.PATH_AUTO
        wfmt = {"w4a4": "nvfp4", "w4a4bs": "nvfp4_bs"}.get(fmt, fmt)
        f = W.FMTS[wfmt]
        (pw, ps), = make_weights(wfmt, 3, N, K, 1)
        x = make_x("nvfp4" if wfmt == "nvfp4_bs" else wfmt, 3, M, K)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        g = torch.tensor([1.0 / 448.0], dtype=torch.float32, device="cuda") if wfmt != "int4" else None
        for _ in range(launches):
            if fmt == "w4a4":
                W.check(W.w4a16_gemm_w4a4_ex(path, M, N, K, x, pw, ps, g, y), "gemm_w4a4")
            elif fmt == "w4a4bs":
                W.check(W.w4a16_gemm_w4a4_bs(M, N, K, x, pw, ps, g, y), "gemm_w4a4_bs")
            else:
                W.check(W.w4a16_gemm_ex(path, f, M, N, K, x, pw, ps, g, y), "gemm")
        torch.cuda.synchronize()
        W.check(W.w4a16_device_status(), "device status")
        out.append({"case": spec, "launches": launches,
                    "path": W.PATH_BS if fmt == "w4a4bs" else
                    W.w4a16_gemm_path(f, M, N, K) if path == W.PATH_AUTO else path})
        del pw, ps, x, y
        torch.cuda.empty_cache()
    print(json.dumps(out))


TRAFFIC_SPECS = ";".join(f"int4,1,{N},{K},1" for _, K, N, _ in DECODE_SHAPES)


def _ncu_value(value: str, unit: str) -> float:
    v = float(value.replace(",", ""))
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "nsecond": 1, "ns": 1,
             "usecond": 1e3, "us": 1e3, "msecond": 1e6, "ms": 1e6}
    if unit not in scale:
        raise ValueError(f"unexpected ncu unit {unit!r}")
    return v * scale[unit]


def write_traffic(csv_path: str, launches: int, out_path=None):
    """profiles/traffic.json from one ncu CSV of the GEMV over the four decode
    shapes at M = 1 (``--case`` with TRAFFIC_SPECS, ``launches`` per shape, all
    captured): per shape the last launch's DRAM bytes, stamped with the hash of
    the GEMV's sources as they are now."""
    import csv
    rows = {}
    with open(csv_path) as f:
        lines = [ln for ln in f if ln.startswith('"')]
    for r in csv.DictReader(lines):
        if "gemv" not in r["Kernel Name"]:
            continue
        rows.setdefault(int(r["ID"]), {})[r["Metric Name"]] = _ncu_value(r["Metric Value"],
                                                                          r["Metric Unit"])
    ids = sorted(rows)
    if len(ids) != launches * len(DECODE_SHAPES):
        raise SystemExit(f"expected {launches * len(DECODE_SHAPES)} GEMV launches, found {len(ids)}")
    per_shape, total, alg = {}, 0.0, 0
    for i, (name, K, N, _) in enumerate(DECODE_SHAPES):
        m = rows[ids[(i + 1) * launches - 1]]
        rd, wr = m["dram__bytes_read.sum"], m["dram__bytes_write.sum"]
        a = int(alg_bytes("int4", 1, N, K))
        per_shape[f"{name} {K}->{N}"] = {"dram_read": int(rd), "dram_write": int(wr), "algorithmic": a,
                                         "ncu_duration_ns": int(m["gpu__time_duration.sum"])}
        total += rd + wr
        alg += a
    n = len(DECODE_SHAPES)
    d = {"kernel": "gemv_kernel<int4, 1 m-tile> (the four launches of the decode step at M=1)",
         "dram_bytes_per_launch": int(round(total / n)), "algorithmic_bytes_per_launch": alg // n,
         "per_shape": per_shape,
         "metrics": "dram__bytes_read.sum + dram__bytes_write.sum of the last captured launch per shape",
         "command": ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum "
                     "--clock-control none --print-units base -k regex:gemv --csv --log-file CSV "
                     f"python bench.py --case '{TRAFFIC_SPECS}' --launches {launches}; then "
                     f"python bench.py --traffic-csv CSV --launches {launches}"),
         "source_hash": kernel_source_hash()}
    with open(out_path or os.path.join(ROOT, "profiles", "traffic.json"), "w") as f:
        json.dump(d, f, indent=1)
        f.write("\n")
    print(json.dumps({"dram_bytes_per_launch": d["dram_bytes_per_launch"],
                      "algorithmic_bytes_per_launch": d["algorithmic_bytes_per_launch"]}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--soak", type=float, default=1.5, help="seconds of untimed replays first")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-stack", action="store_true")
    ap.add_argument("--no-cpu-all", action="store_true", help="skip the all-cores oracle timing")
    ap.add_argument("--case", default=None,
                    help="profiling mode: launch GEMMs fmt,M,N,K[,path][;...] --launches times each")
    ap.add_argument("--launches", type=int, default=5)
    ap.add_argument("--traffic-csv", default=None,
                    help="write profiles/traffic.json from an ncu CSV of --case over the decode shapes")
    args = ap.parse_args()
    if args.traffic_csv:
        write_traffic(args.traffic_csv, args.launches)
        return
    if args.case:
        run_case(args.case, args.launches)
        return
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_native(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
