"""Benchmark: Q4_K GEMV (m = 1) over the decode N x K sweep on B200.

One step = one q4k_gemv call for each of the 8 decode projections of the
1.5B / 7B / 8B classes (N x K: 8960x1536, 1536x8960, 1536x1536, 11008x4096,
4096x11008, 4096x4096, 4096x14336, 128256x4096), inputs already in HBM.
value = bytes counted per step / device time per step, in GB/s, with
bytes = N*K/256*144 + 4*m*(K+N) per call.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs the same sweep on its own GPU (replicas:
the GEMV needs no exchange); value sums the bytes of all ranks over the slowest
rank's time. `--impl reference` times the CPU oracle instead (rank 0 only).
Prints one JSON line on rank 0. Besides the contract keys it carries
`per_shape` (µs per call of each projection: 200 back-to-back calls over
rotating weight copies replayed from a CUDA graph, median of 5 repeats, and the
same with one copy, `l2_hot_us_per_call`, where W fits in L2) and `extra` (multi-vector,
32-layer, fused SwiGLU and embedding figures).
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import q4k_synth  # noqa: E402

METRIC = ("Q4_K GEMV µs/call & achieved HBM GB/s (% of B200 peak), m=1, "
          "N×K sweep")
FULL_SWEEP = q4k_synth.SHAPES_1P5B + q4k_synth.SHAPES_7B + q4k_synth.SHAPES_8B
SWEEP = FULL_SWEEP
WORKLOAD = ("Q4_K GEMV m=1 decode sweep, one call per projection: "
            + ", ".join(f"{n}x{k}" for n, k in SWEEP))
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
GRAPH_STEPS = 10


def bytes_counted(n: int, k: int, m: int = 1) -> int:
    return n * k // 256 * 144 + 4 * m * (k + n)


BYTES_PER_STEP = sum(bytes_counted(n, k) for n, k in SWEEP)
VECTORS = 1   # vectors per call of the timed sweep (--vectors, profiling runs only)


def workload_config(world: int) -> dict:
    """The `config` of the JSON line: the same for the GPU arm and the oracle arm."""
    return {
        "workload": WORKLOAD, "m": VECTORS, "bytes_per_step": BYTES_PER_STEP,
        "bytes_rule": "N*K/256*144 + 4*m*(K+N) per call",
        "l2": (f"inputs larger than L2: {BYTES_PER_STEP / 1e6:.0f} MB of Q4_K per step and two "
               f"rotating copies of every W, so a copy is re-read only after "
               f"~{2 * BYTES_PER_STEP / 1e6:.0f} MB of other traffic"),
        "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
    }


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


GEMV_SOURCES = ("q4k_gemv_stream.cu", "q4k_stream.h", "q4k_gemv.cu", "q4k_sm100.cuh",
                "q4k_superblock.cuh", "q4k_swiglu.cuh", "q4k_gemv_i8.cu", "q4k_gemv_i8.h",
                "q4k_tcgen05.cuh")


def _code_only(text: str) -> str:
    """C/C++ source without its comments and blank-line / trailing-space
    differences (string literals in these files hold no comment markers)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def source_digest() -> str:
    """Hash of the code of the GEMV kernel sources (the files the sweep's
    launches are built from; comments ignored), to tell whether committed ncu
    counters still apply."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gguf_quant_dequant_q4k_b200", "csrc")
    for name in GEMV_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + b"\0" + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def committed_traffic():
    """DRAM bytes per step from the committed ncu summary, if it matches the sources."""
    path = os.path.join(ROOT, "profiles", "q4k_gemv_sweep_traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("source_digest") != source_digest():
        return None
    return t.get("dram_bytes_per_step")


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid: str | None):
        self.proc = None
        self.out = None
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "50"]
            if gpu_uuid:
                cmd += ["-i", gpu_uuid]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [v.strip() for v in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- reference arm

def oracle_sample_rows(frac: float):
    return [(n, k, max(1, int(round(n * frac)))) for n, k in SWEEP]


def run_reference(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    cores = len(os.sched_getaffinity(0))
    threads = max(1, min(cores, 64))
    problems = []
    for n, k in SWEEP:
        # the same bytes the GPU arm streams, first rows only (a bounded sample)
        w, x = q4k_synth.q4k_problem(n, k, 1, q4k_synth.SEEDS[(n, k)])
        problems.append((n, k, w, x))

    def step(frac):
        nbytes = 0
        for n, k, w, x in problems:
            rows = max(1, int(round(n * frac)))
            wrows = w[: rows * (k // 256) * 144]
            oracle.gemv(wrows, x, rows, k, nthreads=threads)
            nbytes += bytes_counted(rows, k)
        return nbytes

    # size the sample so the whole run stays within about two minutes
    t0 = time.perf_counter()
    probe = 0.002
    step(probe)
    per_frac = (time.perf_counter() - t0) / probe
    budget = min(2.0, 120.0 / max(1, args.steps + args.warmup))
    frac = min(1.0, max(1e-4, budget / per_frac))
    for _ in range(args.warmup):
        step(frac)
    t0 = time.perf_counter()
    nbytes = 0
    for _ in range(args.steps):
        nbytes += step(frac)
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    sample = (f"first {frac:.2%} of the rows of each of the 8 sweep projections per step "
              f"(CPU oracle, {threads} threads, double accumulation)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


CPU_BASELINE_SECONDS = 10.0


def cpu_baseline() -> dict:
    """The oracle as it stands on this host's cores: full passes of the sweep
    (all rows of the 8 projections), repeated until about CPU_BASELINE_SECONDS
    of oracle time have been spent."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    threads = max(1, min(cores, 64))
    problems = [(n, k, *q4k_synth.q4k_problem(n, k, 1, q4k_synth.SEEDS[(n, k)])) for n, k in SWEEP]
    nbytes, dt, passes = 0, 0.0, 0
    while dt < CPU_BASELINE_SECONDS:
        for n, k, w, x in problems:
            t0 = time.perf_counter()
            oracle.gemv(w, x, n, k, nthreads=threads)
            dt += time.perf_counter() - t0
            nbytes += bytes_counted(n, k)
        passes += 1
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{passes} full passes of the 8-projection sweep (all rows), row-parallel "
                      f"over {threads} threads, {dt:.1f} s of oracle time"}


# --------------------------------------------------------------------------- extra workloads

def device_us_per_call(torch, dev, stream, call, reps: int = 100, warm: int = 10) -> float:
    """Device time per call of call(0), ..., call(reps - 1) back to back,
    captured in one CUDA graph and replayed (after a warm-up replay), timed with
    CUDA events on `stream`: the host's launch rate never enters."""
    with torch.cuda.stream(stream):
        for i in range(warm):
            call(i)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(reps):
            call(i)
    with torch.cuda.stream(stream):
        g.replay()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    with torch.cuda.stream(stream):
        g.replay()
    a1.record(stream)
    torch.cuda.synchronize(dev)
    del g
    return a0.elapsed_time(a1) * 1e3 / reps


def extra_workloads(q4k, torch, dev, stream, l2: int) -> dict:
    """The other decode workloads of the sweep's configuration list, on this GPU:
    multi-vector shapes (m = 1, 2, 4, 8, and the batches 16 and 32), the
    32-layer 8B-class decode sweep and embedding lookups.
    Each figure is bytes counted / device time (CUDA events)."""
    out = {"multivector": [], "layer_sweep_32": None}
    for n, k in q4k_synth.SHAPES_MULTIVEC:
        w, _ = q4k_synth.q4k_problem(n, k, 1, q4k_synth.SEED_MULTIVEC[(n, k)])
        wd = torch.from_numpy(w).to(dev)
        ws = [wd] + [wd.clone() for _ in range(max(2, -(-2 * l2 // w.nbytes) + 1) - 1)]
        for m in (1, 2, 4, 8, 16, 32):
            x = torch.from_numpy(q4k_synth.x_vectors(k, m, 77 + m)).to(dev)
            y = torch.empty((m, n), dtype=torch.float32, device=dev)
            us = device_us_per_call(
                torch, dev, stream,
                lambda i: q4k.q4k_gemv(ws[i % len(ws)], x, y, m, n, k, stream=stream))
            b = bytes_counted(n, k, m)
            out["multivector"].append({"n": n, "k": k, "m": m, "us_per_call": round(us, 3),
                                       "gbs": round(b / us / 1e3, 1)})
        del ws, wd
    # 32 layers x (q, k, v, o, gate, up, down), each layer's weights seeded
    # independently; one pass = 224 launches captured in one CUDA graph.
    layers = []
    total = 0
    for layer in range(32):
        for proj, (n, k) in enumerate(q4k_synth.LAYER_8B):
            w, x = q4k_synth.q4k_problem(n, k, 1, q4k_synth.layer_seed(layer, proj))
            layers.append((torch.from_numpy(w).to(dev), torch.from_numpy(x).to(dev),
                           torch.empty((1, n), dtype=torch.float32, device=dev), n, k))
            total += bytes_counted(n, k)
    def one_pass():
        for w, x, y, n, k in layers:
            q4k.q4k_gemv(w, x, y, 1, n, k, stream=stream)
    with torch.cuda.stream(stream):
        one_pass()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        one_pass()
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    reps = 20
    a0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            g.replay()
    a1.record(stream)
    torch.cuda.synchronize(dev)
    us = a0.elapsed_time(a1) * 1e3 / reps
    out["layer_sweep_32"] = {"launches": len(layers), "bytes": total, "us_per_pass": round(us, 1),
                             "gbs": round(total / us / 1e3, 1),
                             "how": "one CUDA graph of the 224 projection GEMVs, replayed"}
    del g
    # The same weights as a decode step reads them: k and v take q's input and
    # up takes gate's, and those three calls pass Q4K_GEMV_X_READY (their x
    # is final before the preceding call starts), so their x loads overlap
    # the preceding kernel's tail.
    shared_from = {1: 0, 2: 0, 5: 4}   # projection -> projection whose x it reads
    per_layer = len(q4k_synth.LAYER_8B)
    def one_pass_x_ready():
        for idx, (w, x, y, n, k) in enumerate(layers):
            proj = idx % per_layer
            if proj in shared_from:
                x = layers[idx - proj + shared_from[proj]][1]
            q4k.q4k_gemv(w, x, y, 1, n, k, stream=stream, x_ready=proj in shared_from)
    with torch.cuda.stream(stream):
        one_pass_x_ready()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        one_pass_x_ready()
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            g.replay()
    a1.record(stream)
    torch.cuda.synchronize(dev)
    us = a0.elapsed_time(a1) * 1e3 / reps
    out["layer_sweep_32_x_ready"] = {
        "launches": len(layers), "bytes": total, "us_per_pass": round(us, 1), "gbs": round(total / us / 1e3, 1),
        "how": "the same 224 GEMVs, k / v reading q's input and up reading gate's, those calls with "
               "Q4K_GEMV_X_READY"}
    del g
    # Per call with Q4K_GEMV_X_READY (back-to-back calls of one projection on a
    # constant x, rotating weight copies as in per_shape).
    out["x_ready_per_call"] = []
    for n, k in SWEEP:
        w, x = q4k_synth.q4k_problem(n, k, 1, q4k_synth.SEEDS[(n, k)])
        wd = torch.from_numpy(w).to(dev)
        ws = [wd] + [wd.clone() for _ in range(max(2, -(-2 * l2 // w.nbytes) + 1) - 1)]
        xd = torch.from_numpy(x).to(dev)
        y = torch.empty((1, n), dtype=torch.float32, device=dev)
        us = device_us_per_call(
            torch, dev, stream,
            lambda i: q4k.q4k_gemv(ws[i % len(ws)], xd, y, 1, n, k, stream=stream, x_ready=True))
        out["x_ready_per_call"].append({"n": n, "k": k, "us_per_call": round(us, 3)})
        del ws, wd
    # The same weights with each layer's gate and up projections as one fused
    # SwiGLU call (q4k_gemv_swiglu): 6 launches per layer, same bytes.
    gate_i, up_i = 4, 5
    assert q4k_synth.LAYER_8B[gate_i] == q4k_synth.LAYER_8B[up_i]
    def fused_pass():
        for layer in range(32):
            base = layer * len(q4k_synth.LAYER_8B)
            for proj in range(len(q4k_synth.LAYER_8B)):
                w, x, y, n, k = layers[base + proj]
                if proj == gate_i:
                    q4k.q4k_gemv_swiglu(w, layers[base + up_i][0], x, y, 1, n, k, stream=stream)
                elif proj != up_i:
                    q4k.q4k_gemv(w, x, y, 1, n, k, stream=stream)
    with torch.cuda.stream(stream):
        fused_pass()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fused_pass()
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    a0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            g.replay()
    a1.record(stream)
    torch.cuda.synchronize(dev)
    us = a0.elapsed_time(a1) * 1e3 / reps
    out["layer_sweep_32_fused_gate_up"] = {
        "launches": 32 * (len(q4k_synth.LAYER_8B) - 1), "bytes": total,
        "us_per_pass": round(us, 1), "gbs": round(total / us / 1e3, 1),
        "how": "the same 32 layers, gate and up of each layer as one q4k_gemv_swiglu call"}
    del g, layers
    torch.cuda.empty_cache()
    out["embedding"] = embedding_workloads(q4k, torch, dev, stream)
    out["prefill_f16"] = prefill_workloads(q4k, torch, dev, stream)
    out["swiglu"] = swiglu_workloads(q4k, torch, dev, stream, l2)
    return out


def swiglu_workloads(q4k, torch, dev, stream, l2: int) -> list:
    """Fused gate/up SwiGLU (q4k_gemv_swiglu) on the 7B and 8B FFN shapes, m = 1
    and 2, against the same work as two q4k_gemv calls (the fused call also does
    the SwiGLU, which the separate pair leaves undone). Bytes counted per call =
    both matrices + x once + y once."""
    res = []
    for n, k in ((11008, 4096), (14336, 4096)):
        wg, _ = q4k_synth.q4k_problem(n, k, 1, 400 + n)
        wu, _ = q4k_synth.q4k_problem(n, k, 1, 401 + n)
        copies = max(2, -(-2 * l2 // (2 * wg.nbytes)) + 1)
        gs = [torch.from_numpy(wg).to(dev) for _ in range(copies)]
        us = [torch.from_numpy(wu).to(dev) for _ in range(copies)]
        for m in (1, 2):
            x = torch.from_numpy(q4k_synth.x_vectors(k, m, 90 + m)).to(dev)
            y = torch.empty((m, n), dtype=torch.float32, device=dev)
            y2 = torch.empty((m, n), dtype=torch.float32, device=dev)

            def timed(fn):
                return device_us_per_call(torch, dev, stream, fn)

            fused = timed(lambda i: q4k.q4k_gemv_swiglu(gs[i % copies], us[i % copies], x, y, m,
                                                        n, k, stream=stream))

            def pair(i):
                q4k.q4k_gemv(gs[i % copies], x, y, m, n, k, stream=stream)
                q4k.q4k_gemv(us[i % copies], x, y2, m, n, k, stream=stream)
            separate = timed(pair)
            b = 2 * n * (k // 256) * 144 + 4 * m * (k + n)
            res.append({"n": n, "k": k, "m": m, "us_per_call": round(fused, 3),
                        "gbs": round(b / fused / 1e3, 1),
                        "two_gemv_calls_us": round(separate, 3)})
        del gs, us
    torch.cuda.empty_cache()
    return res


PREFILL_TOKENS = 512
FALLBACK_BF16_TFLOPS = 1590.0


def measured_tensor_peak():
    """Dense fp16/bf16 tensor peak in TFLOP/s: the measured cuBLAS bf16 burst
    figure (fp16 has the same nominal rate), else the recipe's fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured bf16 burst"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, "fallback bf16 burst"


def prefill_workloads(q4k, torch, dev, stream) -> dict:
    """The prefill route on the 8B-class projections at m = 512 tokens: the
    fp16 mirror (q4k_dequant_f16, GB/s of Q4_K read + fp16 written), the GEMM on
    pre-converted activations (q4k_gemm_f16) and the one-call route with the
    convert into the caller's scratch (q4k_prefill_f16), in TFLOP/s (2 m n k per
    call) against the dense tensor peak. Device time of 20 calls from a CUDA
    graph after 5 eager ones."""
    peak, peak_kind = measured_tensor_peak()
    m = PREFILL_TOKENS
    res = []

    def timed(fn, reps=20):
        return device_us_per_call(torch, dev, stream, lambda _i: fn(), reps=reps, warm=5)

    for n, k in [(4096, 4096), (1024, 4096), (14336, 4096), (4096, 14336)]:
        w, _ = q4k_synth.q4k_problem(n, k, 1, 530 + n + k)
        wd = torch.from_numpy(w).to(dev)
        w16 = torch.empty((n, k), dtype=torch.float16, device=dev)
        x = torch.from_numpy(q4k_synth.x_vectors(k, m, 531)).to(dev)
        x16 = torch.empty((m, k), dtype=torch.float16, device=dev)
        scratch = torch.empty(m * k * 2, dtype=torch.uint8, device=dev)
        y = torch.empty((m, n), dtype=torch.float32, device=dev)
        mirror_us = timed(lambda: q4k.q4k_dequant_f16(wd, w16, n, k, stream=stream))
        q4k.q4k_f32_to_f16(x, x16, m * k, stream=stream)
        gemm_us = timed(lambda: q4k.q4k_gemm_f16(w16, x16, y, m, n, k, stream=stream))
        one_us = timed(lambda: q4k.q4k_prefill_f16(w16, x, scratch, y, m, n, k, stream=stream))
        flops = 2.0 * m * n * k
        res.append({"m": m, "n": n, "k": k,
                    "gemm_us": round(gemm_us, 2), "gemm_tflops": round(flops / gemm_us / 1e6, 1),
                    "gemm_frac_of_peak": round(flops / gemm_us / 1e6 / peak, 3),
                    "prefill_call_us": round(one_us, 2),
                    "prefill_call_tflops": round(flops / one_us / 1e6, 1),
                    "mirror_us": round(mirror_us, 2),
                    "mirror_gbs": round((n * k // 256 * 144 + 2 * n * k) / mirror_us / 1e3, 1)})
        del wd, w16, x, x16, scratch, y
    torch.cuda.empty_cache()
    assert q4k.q4k_device_fault_flags() == 0
    return {"tokens": m, "peak_tflops": peak, "peak_kind": peak_kind, "shapes": res}


def embedding_workloads(q4k, torch, dev, stream) -> list:
    """Q4_K embedding lookups from a 128256 x 4096 table (an 8B model's token
    embedding): one token (q4k_embed_lookup_f32) and gathers of 8 and 512
    device-resident tokens (q4k_embed_gather_f32). Bytes counted per call =
    rows read (hidden/256*144 each) + f32 rows written (4*hidden each)."""
    rows, hidden = 128256, 4096
    w, _ = q4k_synth.q4k_problem(rows, hidden, 1, q4k_synth.SEEDS[(rows, hidden)])
    table = torch.from_numpy(w).to(dev)
    rng = np.random.default_rng(3)
    res = []
    for n_tok in (1, 8, 512):
        toks = torch.from_numpy(rng.integers(0, rows, n_tok).astype(np.int32)).to(dev)
        out = torch.empty((n_tok, hidden), dtype=torch.float32, device=dev)

        def call(_i):
            if n_tok == 1:
                q4k.q4k_embed_lookup_f32(table, rows, hidden, hidden, 12345, 1.0, out,
                                         stream=stream)
            else:
                q4k.q4k_embed_gather_f32(table, rows, hidden, toks, n_tok, 1.0, out,
                                         stream=stream)
        us = device_us_per_call(torch, dev, stream, call, reps=200)
        b = n_tok * (hidden // 256 * 144 + 4 * hidden)
        res.append({"rows": rows, "hidden": hidden, "tokens": n_tok,
                    "call": "q4k_embed_lookup_f32" if n_tok == 1 else "q4k_embed_gather_f32",
                    "us_per_call": round(us, 3), "gbs": round(b / us / 1e3, 1)})
    assert q4k.q4k_device_fault_flags() == 0
    del table
    torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------------------- our arm

def max_over_ranks(value: float, world: int, device) -> float:
    """The slowest rank's figure (max over ranks): a multi-GPU time is the job's
    time, set by its slowest rank. `device` holds the reduction tensor (the
    process group's device: a GPU under NCCL, the CPU under gloo)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_step: int, steps: int, ms: float) -> float:
    """Bytes all ranks processed / the slowest rank's time, in GB/s (replicas:
    every rank streams the same step)."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


def run_ours(args) -> None:
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    import gguf_quant_dequant_q4k_b200 as q4k

    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 << 20))
    stream = torch.cuda.Stream(device=dev)

    # inputs: per projection, enough copies of W that each copy is re-read only
    # after more than 2 x L2 of other traffic
    shapes = []
    for n, k in SWEEP:
        seed = q4k_synth.SEEDS.get((n, k), q4k_synth.SEED_MULTIVEC.get((n, k)))
        w, x = q4k_synth.q4k_problem(n, k, VECTORS, seed)
        wdev = torch.from_numpy(w).to(dev)
        copies = max(2, -(-2 * l2 // w.nbytes) + 1)
        ws = [wdev] + [wdev.clone() for _ in range(copies - 1)]
        xdev = torch.from_numpy(x).to(dev)
        ydev = torch.empty((VECTORS, n), dtype=torch.float32, device=dev)
        shapes.append({"n": n, "k": k, "ws": ws, "x": xdev, "y": ydev, "x_host": x})
    torch.cuda.synchronize(dev)
    plans = [q4k.q4k_gemv_plan_for(VECTORS, s["n"], s["k"], props.multi_processor_count)
             for s in shapes]
    launches_per_step = sum(p["launches"] for p in plans)

    def sweep(step_index: int):
        for s in shapes:
            w = s["ws"][step_index % 2]
            q4k.q4k_gemv(w, s["x"], s["y"], VECTORS, s["n"], s["k"], stream=stream)

    # CUDA graphs of GRAPH_STEPS steps and of one step (copies alternate step
    # to step; an even GRAPH_STEPS keeps the alternation across replays)
    use_graph = not args.no_graph
    graph = graph1 = None
    if use_graph:
        with torch.cuda.stream(stream):
            sweep(0)  # make sure per-device set-up happened outside capture
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(GRAPH_STEPS):
                sweep(i)
        graph1 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph1, stream=stream):
            sweep(0)

    def run_steps(count: int):
        if use_graph:
            reps = count // GRAPH_STEPS
            with torch.cuda.stream(stream):
                for _ in range(reps):
                    graph.replay()
                for _ in range(count - reps * GRAPH_STEPS):
                    graph1.replay()
        else:
            for i in range(count):
                sweep(i)

    # warm-up: the requested steps (at least 3), and with graphs at least two
    # replays of the GRAPH_STEPS-step graph and one of the one-step graph, so
    # that no graph is replayed for the first time inside the timed region
    warm_steps = max(args.warmup, 3)
    warm_replays = max(2, -(-warm_steps // GRAPH_STEPS)) if use_graph else 0
    if use_graph:
        with torch.cuda.stream(stream):
            for _ in range(warm_replays):
                graph.replay()
            graph1.replay()
    else:
        run_steps(warm_steps)
    torch.cuda.synchronize(dev)

    uuid = str(getattr(props, "uuid", "") or "")
    if uuid and not uuid.startswith("GPU-"):
        uuid = "GPU-" + uuid
    sampler = ClockSampler(uuid or None) if rank == 0 else None
    if sampler is not None:
        time.sleep(0.15)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run_steps(args.steps)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler is not None else None
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ms_per_step = ms / args.steps
    value = whole_job_gbs(world, BYTES_PER_STEP, args.steps, ms)

    # per-projection us/call: R = 200 back-to-back calls over rotating copies
    # (each copy re-read only after more than 2 x L2 of other traffic), median
    # of 5 repeats; and the same with one copy (L2-hot where W fits in L2)
    per_shape = []
    peak, peak_kind = measured_peak()

    def timed_calls(s, copies, reps=200):
        return device_us_per_call(
            torch, dev, stream,
            lambda i: q4k.q4k_gemv(s["ws"][i % copies], s["x"], s["y"], 1, s["n"], s["k"],
                                   stream=stream), reps=reps)

    for s, p in zip([] if args.skip_extras else shapes, plans):
        us = statistics.median(timed_calls(s, len(s["ws"])) for _ in range(5))
        hot = statistics.median(timed_calls(s, 1) for _ in range(5))
        b = bytes_counted(s["n"], s["k"])
        per_shape.append({"n": s["n"], "k": s["k"], "us_per_call": round(us, 3),
                          "gbs": round(b / us / 1e3, 1), "frac_of_measured": round(b / us / 1e3 / peak, 4),
                          "frac_of_nominal": round(b / us / 1e3 / NOMINAL_HBM_GBS, 4),
                          "l2_hot_us_per_call": round(hot, 3),
                          "w_copies": len(s["ws"]), "kernel": p["kernel"], "grid": p["grid"],
                          "teams": p["teams"], "depth": p["depth"], "slices": p["slices"]})

    # end to end through the public API: pinned x -> device, gemv, y -> pinned host
    e2e_steps = 0 if args.skip_extras else min(args.steps, 500)
    # The step's inputs (the 8 x vectors) sit in one pinned host buffer and go
    # to the device in one copy; the 8 results come back in one copy.
    x_off = np.cumsum([0] + [s["k"] for s in shapes])
    y_off = np.cumsum([0] + [s["n"] for s in shapes])
    x_host = torch.from_numpy(np.concatenate([s["x_host"].reshape(-1) for s in shapes])).pin_memory()
    y_host = torch.empty(int(y_off[-1]), dtype=torch.float32).pin_memory()
    x_dev = torch.empty(int(x_off[-1]), dtype=torch.float32, device=dev)
    y_dev = torch.empty(int(y_off[-1]), dtype=torch.float32, device=dev)
    x_views = [x_dev[int(x_off[j]):int(x_off[j + 1])] for j in range(len(shapes))]
    y_views = [y_dev[int(y_off[j]):int(y_off[j + 1])] for j in range(len(shapes))]
    h2d = x_host.numel() * 4
    d2h = y_host.numel() * 4

    def e2e_step(i):
        with torch.cuda.stream(stream):
            x_dev.copy_(x_host, non_blocking=True)
            for s, xv, yv in zip(shapes, x_views, y_views):
                q4k.q4k_gemv(s["ws"][i % 2], xv, yv, 1, s["n"], s["k"], stream=stream)
            y_host.copy_(y_dev, non_blocking=True)

    for i in range(3 if e2e_steps else 0):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    b0 = torch.cuda.Event(enable_timing=True)
    b1 = torch.cuda.Event(enable_timing=True)
    b0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    b1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(b0.elapsed_time(b1), world, dev)
    e2e_value = whole_job_gbs(world, BYTES_PER_STEP, e2e_steps, e2e_ms) if e2e_steps else None

    if world > 1:
        dist.barrier()
        graph = graph1 = None
        dist.destroy_process_group()
    if rank != 0:
        return

    achieved = BYTES_PER_STEP / (ms_per_step * 1e-3) / 1e9   # per GPU, all launches of a step
    full_sweep = VECTORS == 1 and SWEEP == FULL_SWEEP
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": (warm_replays * GRAPH_STEPS + 1) if use_graph else warm_steps,
        "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic: seeded Q4_K superblocks (d, dmin fp16 of U[1e-3,2e-2], random "
                "scale and quant bytes), x ~ N(0,1) f32",
        "config": workload_config(world),
        "launch": (f"CUDA graphs of {GRAPH_STEPS} steps and of 1 step, replayed; "
                   f"{warm_replays} warm-up replays of the {GRAPH_STEPS}-step graph first"
                   if use_graph else "eager launches"),
        "per_shape": per_shape,
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_kind": f"{peak_kind} copy bandwidth",
            "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
            "traffic": committed_traffic() if full_sweep else None,
            "algorithmic_bytes": BYTES_PER_STEP,
            "per": (f"one step = the {len(shapes)} q4k_gemv calls ({launches_per_step} "
                    f"launches) of the {'sweep' if full_sweep else 'subset'}"),
            "kernel": "q4k_gemv",
        },
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "how": "per step: the 8 x vectors from one pinned host buffer in one copy, "
                       "8 q4k_gemv calls, the 8 results to one pinned host buffer in one "
                       "copy; eager through the ctypes API"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_extras and not args.skip_extras:
        line["extra"] = extra_workloads(q4k, torch, dev, stream, l2)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-graph", action="store_true", help="eager launches (for profilers)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the multi-vector and 32-layer sweep measurements")
    ap.add_argument("--shapes", default=None,
                    help="comma-separated NxK subset of the sweep (profiling runs only)")
    ap.add_argument("--skip-extras", action="store_true",
                    help="skip the per-shape and end-to-end passes (profiling runs only)")
    ap.add_argument("--vectors", type=int, default=1,
                    help="vectors per call of the timed sweep (profiling runs only: needs "
                         "--shapes and --skip-extras; the multi-vector shapes are allowed)")
    ap.add_argument("--prefill-only", action="store_true",
                    help="print only the prefill (fp16 mirror + tensor-core GEMM) figures")
    args = ap.parse_args()
    if args.steps < 1 or args.warmup < 0:
        raise SystemExit("--steps must be >= 1 and --warmup >= 0")
    if args.vectors != 1 and not (args.shapes and args.skip_extras):
        raise SystemExit("--vectors needs --shapes and --skip-extras")
    if args.shapes:
        global SWEEP, BYTES_PER_STEP, WORKLOAD, VECTORS
        VECTORS = args.vectors
        SWEEP = [tuple(int(v) for v in s.lower().split("x")) for s in args.shapes.split(",")]
        for sh in SWEEP:
            if sh not in q4k_synth.SEEDS and not (VECTORS > 1 and sh in q4k_synth.SEED_MULTIVEC):
                raise SystemExit(f"shape {sh} is not one of the sweep's")
        BYTES_PER_STEP = sum(bytes_counted(n, k, VECTORS) for n, k in SWEEP)
        WORKLOAD = "subset of the sweep: " + ", ".join(f"{n}x{k}" for n, k in SWEEP)
        if VECTORS > 1:
            WORKLOAD += f", {VECTORS} vectors per call"
    if args.prefill_only:
        import torch
        import gguf_quant_dequant_q4k_b200 as q4k
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps(prefill_workloads(q4k, torch, dev, torch.cuda.Stream(device=dev))),
              flush=True)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
