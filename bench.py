"""Benchmark of the block-scaled projection GEMM path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--no-extra] [--no-e2e]

A step is one pass of the hot path -- activation quantisation to e4m3 with
1 x 32 E8M0 scales, then the block-scaled GEMM -- over the decode-shaped MXFP8
workload of the fused q_a + kv projection: M in {1, 8, 32, 64} tokens,
N = 2048, K = 7168, e4m3 weights with 32 x 32 E8M0 scales, no bias, bf16 out.
The step makes one mx_gemm call per M on the bf16 activations
(MX_A_BF16_E8M0_1X32): the library quantises them (bit for bit as mx_quant_act
would) into its workspace and runs the decode GEMM.  The same step as separate
mx_quant_act + mx_gemm calls is timed too (step_unfused_ms).  Each step runs all four M values; the weights
rotate through enough copies (> 2x L2) that every GEMM streams them from HBM.
Each step is one CUDA graph replay.

Printed (rank 0, one JSON line): the weight-stream throughput of the whole job
in GB/s, the GEMM kernel's roofline against the measured HBM copy bandwidth,
the fp64 CPU oracle's throughput on a bounded sample (cpu_baseline), the SM
clocks seen during the timed region, an end-to-end number through the public
API with host buffers, and the other workloads (DiT/ViT MLP GEMM, W4A8
gate_up SwiGLU, fp8 lm_head, small case) measured the same way.

Multi-GPU (torchrun, one rank per GPU): every rank runs the same workload on
its own replica (the GEMM shards with no exchange); the time is the max over
ranks and the value sums all ranks' work ("scaling": "weak").

`--impl reference` times the fp64 CPU oracle (the only reference this path
has) on a bounded sample per step, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "MX GEMM TFLOP/s (M≥2048) & weight GB/s (M≤64), % of B200 roofline"
L2_BYTES = 126 * 1024 * 1024

# decode workload: fused q_a + kv projection shape
DEC_MS = (1, 8, 32, 64)
DEC_N, DEC_K = 2048, 7168


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------- dist

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (SM clock, throttle reasons) during a timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.t_start = self.t_stop = None

    def start(self):
        sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "50"] + sel, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_start(self):
        self.t_start = time.time()

    def mark_stop(self):
        self.t_stop = time.time()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.reader.join(timeout=2)

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((ts, parts))
        inside = [r for r in rows if self.t_start and self.t_stop and self.t_start <= r[0] <= self.t_stop]
        use = inside if inside else rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[1]) for _, p in use if num(p[1]) is not None]
        mx = [num(p[2]) for _, p in use if num(p[2]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, p in use:
            for name, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(use), "in_timed_region": bool(inside)}


# ---------------------------------------------------------------------------- workloads

class Workload:
    """Device buffers and the launch list of one GEMM workload."""

    def __init__(self, mx, name, Ms, N, K, a_fmt, b_fmt, epi, seed, with_bias, desc):
        import synth
        self.mx = mx
        # 1x32 E8M0 activations can also be handed over as bf16 (quantised by the GEMM)
        self.can_fuse = a_fmt == mx.MX_A_E4M3_E8M0_1X32
        self.name, self.Ms, self.N, self.K = name, tuple(Ms), N, K
        self.a_fmt, self.b_fmt, self.epi = a_fmt, b_fmt, epi
        self.desc = desc
        dev = "cuda"
        # weights: seeded bf16 on the device, quantised by the library
        w = synth.bf16_matrix(seed + 1, N, K, synth.W_SIGMA, device=dev)
        wc, ws = mx.weight_buffers(N, K, b_fmt)
        mx.mx_quant_weight(w, wc, ws, b_fmt)
        del w
        torch.cuda.synchronize()
        self.w_bytes = wc.numel() + ws.numel() * ws.element_size()
        # enough copies that the rotation exceeds 2x L2
        copies = min(64, max(1, math.ceil(2 * L2_BYTES / self.w_bytes)))
        self.weights = [(wc, ws)] + [(wc.clone(), ws.clone()) for _ in range(copies - 1)]
        self.bias = synth.f32_vector(seed + 2, N, synth.BIAS_SIGMA, device=dev) if with_bias else None
        self.nout = N // 2 if epi in (mx.MX_EPI_SWIGLU, mx.MX_EPI_SWIGLU_MXQ) else N
        # bytes of one output row: bf16, or e4m3 codes + E8M0 scales when the
        # SwiGLU output is handed on as the next GEMM's MX operand
        self.out_row_bytes = (N // 2 + N // 64) if epi == mx.MX_EPI_SWIGLU_MXQ else 2 * self.nout
        self.x, self.acodes, self.ascales, self.out = {}, {}, {}, {}
        for M in self.Ms:
            self.x[M] = synth.bf16_matrix(seed, M, K, synth.X_SIGMA, device=dev)
            self.acodes[M], self.ascales[M] = mx.act_buffers(M, K, a_fmt)
            self.out[M] = mx.out_buffer(M, N, epi)
        # one workspace for all of this workload's launches (they share a stream)
        probs = [(M, N, K, a_fmt, b_fmt, epi) for M in self.Ms]
        if self.can_fuse:
            probs += [(M, N, K, mx.MX_A_BF16_E8M0_1X32, b_fmt, epi) for M in self.Ms]
        self.ws = mx.workspace(problems=probs)
        self.rot = 0
        # everything above ran on the default stream; the launches go to another
        torch.cuda.synchronize()

    def flops(self, M):
        return 2.0 * M * self.N * self.K

    def act_bytes(self, M):
        """Activation codes + scales of M rows."""
        if self.a_fmt == 3:  # packed e2m1 + 1x32 E8M0
            return M * self.K // 2 + M * (self.K // 32)
        return M * self.K + (M * (self.K // 32) if self.a_fmt == 0 else 4 * M)

    def gemm_bytes(self, M):
        """Algorithmic bytes of one GEMM launch: weights + their scales, activation
        codes + scales, and the output."""
        return self.w_bytes + self.act_bytes(M) + M * self.out_row_bytes

    def fused_bytes(self, M):
        """Algorithmic bytes of one fused launch: weights + their scales, the bf16
        activations, and the output."""
        return self.w_bytes + 2 * M * self.K + M * self.out_row_bytes

    def quant_bytes(self, M):
        return 2 * M * self.K + self.act_bytes(M)

    def next_weights(self):
        wc, ws = self.weights[self.rot % len(self.weights)]
        self.rot += 1
        return wc, ws

    def enqueue_quant(self, M, stream):
        self.mx.mx_quant_act(self.x[M], self.acodes[M], self.ascales[M], self.a_fmt, stream=stream)

    def enqueue_gemm(self, M, stream, weights=None):
        wc, ws = weights if weights is not None else self.next_weights()
        self.mx.mx_gemm(self.acodes[M], self.ascales[M], self.a_fmt, wc, ws, self.b_fmt, self.bias, self.epi,
                        self.out[M], M, self.N, self.K, self.ws, stream=stream)

    def enqueue_fused(self, M, stream, weights=None, x=None):
        """The GEMM on the bf16 activations (quantised inside the GEMM)."""
        wc, ws = weights if weights is not None else self.next_weights()
        self.mx.mx_gemm(self.x[M] if x is None else x, None, self.mx.MX_A_BF16_E8M0_1X32, wc, ws, self.b_fmt,
                        self.bias, self.epi, self.out[M], M, self.N, self.K, self.ws, stream=stream)


def plan_info(mx, M, N, K, af, bf, epi):
    """The library's plan for one problem with the workspace the bench gives it."""
    p = mx.mx_gemm_plan_info(M, N, K, af, bf, epi)
    return {k: p[k] for k in ("kernel", "block_m", "block_n", "splits", "k_reduction", "grid", "acc_bufs",
                              "stages", "tiles")}


def capture(stream, fn):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


class StepGraphs:
    """The decode step as CUDA graphs.  A step is one GEMM on the bf16
    activations per M of the workload (or, with fused=False, quant + GEMM on
    the codes), each with the next weight copy of the rotation.  A graph
    holds a whole walk through the rotation (`phases` steps, so that every
    copy is used equally and consecutive launches stream different copies),
    one per starting phase; single-step graphs cover a remainder.  run(k)
    enqueues exactly k steps, continuing the rotation."""

    def __init__(self, wl: Workload, stream, fused=True):
        nper = len(wl.Ms)
        copies = len(wl.weights)
        self.phases = copies // math.gcd(copies, nper)
        self.stream = stream

        def one_step(p):
            for j, M in enumerate(wl.Ms):
                w = wl.weights[(p * nper + j) % copies]
                if fused:
                    wl.enqueue_fused(M, stream, w)
                else:
                    wl.enqueue_quant(M, stream)
                    wl.enqueue_gemm(M, stream, w)

        def walk(p0):
            for i in range(self.phases):
                one_step((p0 + i) % self.phases)
        # a full walk from every starting phase, so any run is whole walks
        # plus fewer than `phases` single steps
        self.full = [capture(stream, lambda p0=p0: walk(p0)) for p0 in range(self.phases)]
        self.single = [capture(stream, lambda p=p: one_step(p)) for p in range(self.phases)]
        self.pos = 0
        # a graph's first replay uploads it to the device: do that for every
        # graph now, outside any timed region
        with torch.cuda.stream(stream):
            for g in self.full + self.single:
                g.replay()
        stream.synchronize()

    def run(self, k):
        """Enqueue k steps on the stream (the caller is inside torch.cuda.stream)."""
        while k >= self.phases:
            self.full[self.pos].replay()
            k -= self.phases
        while k > 0:
            self.single[self.pos].replay()
            self.pos = (self.pos + 1) % self.phases
            k -= 1


def time_steps(sg: StepGraphs, stream, steps):
    """Seconds for `steps` steps, CUDA events on `stream`."""
    with torch.cuda.stream(stream):
        sg.run(3)
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        sg.run(steps)
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / 1e3


def gemm_only_graph(wl: Workload, M, stream, launches, fused=False):
    copies = len(wl.weights)

    def body():
        for i in range(launches):
            if fused:
                wl.enqueue_fused(M, stream, wl.weights[i % copies])
            else:
                wl.enqueue_gemm(M, stream, wl.weights[i % copies])
    return capture(stream, body)


def quant_only_graph(wl: Workload, M, stream, launches):
    def body():
        for _ in range(launches):
            wl.enqueue_quant(M, stream)
    return capture(stream, body)


def time_graph(g, stream, reps, warm=3):
    """Seconds for `reps` replays; replays go to `stream` (CUDAGraph.replay
    launches on the current stream), bracketed by events on that stream."""
    with torch.cuda.stream(stream):
        for _ in range(warm):
            g.replay()
        stream.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / 1e3  # seconds


def launch_time(g, launches, stream, seconds):
    t1 = time_graph(g, stream, 1)
    reps = min(20000, max(3, int(seconds / max(t1, 1e-6))))
    return time_graph(g, stream, reps) / (reps * launches)


def kernel_timing(wl: Workload, M, stream, seconds=0.3):
    """Average duration of one GEMM launch on codes, one quant launch and (for
    1x32 E8M0 activations) one GEMM launch on bf16 activations, measured with
    CUDA events around graphs of back-to-back launches on `stream`."""
    launches = max(len(wl.weights), 16)
    tg = launch_time(gemm_only_graph(wl, M, stream, launches), launches, stream, seconds)
    tq = launch_time(quant_only_graph(wl, M, stream, 32), 32, stream, 0.1)
    tf = launch_time(gemm_only_graph(wl, M, stream, launches, fused=True), launches, stream, seconds) \
        if wl.can_fuse else None
    return tg, tq, tf


# Sources each kernel family's code comes from: a traffic row in
# profiles/traffic.md counts only while its family's sources hash to the value
# recorded beside it.
_CSRC = "mxfp4_gemm_transformer_b200/csrc/"
KERNEL_FAMILIES = {
    "decode": tuple(_CSRC + f for f in ("mx_decode.cu", "mx_decode_common.cuh", "mx_kernel_common.cuh",
                                        "mx_quant_common.cuh", "mx_ptx.cuh", "mx_internal.h")),
    "tile": tuple(_CSRC + f for f in ("mx_gemm.cu", "mx_kernel_common.cuh", "mx_ptx.cuh", "mx_internal.h")),
}
# the family of the kernel that runs each workload's GEMM on codes
WORKLOAD_FAMILY = {"decode": "decode", "small": "decode", "gateup16": "decode", "gateup16_mxq": "decode",
                   "down16": "decode", "lmhead": "decode", "mlp": "tile", "gateup4096": "tile",
                   "down4096": "tile", "gateup4096_w4a4": "tile"}


def kernel_hash(family: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_FAMILIES[family]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic():
    """(workload, M) -> DRAM bytes per launch from profiles/traffic.md, for rows
    captured from the kernel sources as they are now (else nothing)."""
    out = {}
    try:
        cur = {fam: kernel_hash(fam) for fam in KERNEL_FAMILIES}
        with open(os.path.join(ROOT, "profiles", "traffic.md")) as f:
            for line in f:
                cells = [c.strip() for c in line.strip().strip("|").split("|")]
                if len(cells) == 4 and cells[1].isdigit() and cells[2].isdigit():
                    fam = WORKLOAD_FAMILY.get(cells[0])
                    if fam and cells[3] == cur[fam]:
                        out[(cells[0], int(cells[1]))] = int(cells[2])
    except OSError:
        pass
    return out


def roofline_entry(wl: Workload, M, t_gemm, pk, bound, fused=False):
    if bound == "hbm":
        ach = (wl.fused_bytes(M) if fused else wl.gemm_bytes(M)) / t_gemm / 1e9
        return {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / pk["hbm_gbs"], 4), "traffic": None,
                "peak_note": f"{pk['source']} HBM copy bandwidth"}
    ach = wl.flops(M) / t_gemm / 1e12
    if wl.a_fmt == 3:
        # W4A4 runs at the fp4 rate: 4x bf16 (nominal ratio 9 / 2.25)
        fp4_peak = 4.0 * pk["bf16_tflops"]
        return {"bound": "tensor", "achieved": round(ach, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                "frac": round(ach / fp4_peak, 4), "traffic": None,
                "peak_note": f"fp4 = 4 x {pk['source']} bf16 burst", "frac_of_spec_9000": round(ach / 9000.0, 4)}
    fp8_peak = 2.0 * pk["bf16_tflops"]  # dense fp8 = 2x bf16 (nominal ratio 4.5 / 2.25)
    return {"bound": "tensor", "achieved": round(ach, 1), "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
            "frac": round(ach / fp8_peak, 4), "traffic": None,
            "peak_note": f"fp8 = 2 x {pk['source']} bf16 burst", "frac_of_spec_4500": round(ach / 4500.0, 4)}


# ---------------------------------------------------------------------------- CPU oracle

def oracle_sample(rows_w: int, Ms=(1,), seed=0):
    """Prepare an oracle sample of the decode workload: the first `rows_w` weight
    rows (32-row blocks) and the activation rows; returns a callable timing
    one oracle GEMM pass and the weight bytes it covers."""
    import oracle
    import synth
    w = synth.bf16_matrix(seed + 1, DEC_N, DEC_K, synth.W_SIGMA, row0=0, nrows=rows_w)
    bc, bs = oracle.quant_w_e4m3_32x32(w)
    xs = {M: oracle.quant_act_e8m0(synth.bf16_matrix(seed, M, DEC_K, synth.X_SIGMA)) for M in Ms}

    def run():
        for M in Ms:
            a, sa = xs[M]
            oracle.gemm(a, sa, 0, bc, bs, 0, None, 0, M, rows_w, DEC_K)
    wbytes = len(Ms) * (rows_w * DEC_K + (rows_w // 32) * (DEC_K // 32))
    return run, wbytes


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(target_s=12.0):
    """The oracle as it stands, timed on the host cores on a bounded sample of
    the decode workload: all four M values against the first rows of W (all
    of them when one pass is shorter than the target, then whole passes are
    repeated until about `target_s` seconds of work)."""
    run, wb = oracle_sample(64, DEC_MS)
    t0 = time.perf_counter()
    run()
    t1 = time.perf_counter() - t0
    rows = int(min(DEC_N, max(32, 64 * target_s / max(t1, 1e-3))) // 32 * 32)
    run, wb = oracle_sample(rows, DEC_MS)
    t0 = time.perf_counter()
    run()
    one = time.perf_counter() - t0
    passes = max(1, int(round(target_s / max(one, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(passes):
        run()
    dt = time.perf_counter() - t0
    return {"value": round(wb * passes / dt / 1e9, 6), "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"decode workload, all M in {list(DEC_MS)}, first {rows} of {DEC_N} weight rows, K={DEC_K}, "
                      f"{passes} pass(es); {dt:.1f} s of fp64 oracle GEMM (OpenMP over output elements)"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    budget = 150.0  # seconds for the whole --steps + --warmup run
    run, wb = oracle_sample(32, (1,))
    t0 = time.perf_counter()
    run()
    t1 = time.perf_counter() - t0
    per_step = budget / max(1, args.steps + args.warmup)
    rows = int(max(32, min(DEC_N, 32 * per_step / max(t1, 1e-4))) // 32 * 32)
    run, wb = oracle_sample(rows, (1,))
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    value = wb * args.steps / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": f"decode MXFP8 GEMM M=1 N={DEC_N} K={DEC_K} (fused q_a+kv shape), "
                                   f"32x32 E8M0 e4m3 weights, sample of {rows} weight rows per step"},
            "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": f"M=1 token x first {rows} weight rows x K={DEC_K} per step"},
            "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- main arm

def e2e_measure(mx, wl: Workload, steps: int, stream, graph: bool):
    """Same metric through the public API with host buffers: every step copies
    the bf16 activations in from pinned memory, calls mx_gemm on them for
    every M (the library quantises them) and copies the bf16 outputs back to
    pinned memory.  graph=False: eager calls from Python, one by one, on one
    stream; graph=True: the steps (copies included) captured once and
    replayed, as a serving loop would issue them, with the copies on their own
    streams overlapping the GEMMs of the other problems -- a graph holds a
    whole walk through the weight rotation."""
    hx = {M: wl.x[M].cpu().pin_memory() for M in wl.Ms}
    hout = {M: torch.empty_like(wl.out[M], device="cpu").pin_memory() for M in wl.Ms}
    dx = {M: torch.empty_like(wl.x[M]) for M in wl.Ms}
    h2d = sum(hx[M].numel() * 2 for M in wl.Ms)
    d2h = sum(hout[M].numel() * 2 for M in wl.Ms)
    nper = len(wl.Ms)
    copies = len(wl.weights)
    phases = copies // math.gcd(copies, nper)

    def step(p):
        for j, M in enumerate(wl.Ms):
            dx[M].copy_(hx[M], non_blocking=True)
            wl.enqueue_fused(M, stream, wl.weights[(p * nper + j) % copies], x=dx[M])
            hout[M].copy_(wl.out[M], non_blocking=True)

    # graph form: the step's four problems are independent, so the input
    # copies go to one copy stream and the output copies to another; each GEMM
    # waits for its own input, each output copy for its own GEMM, and the next
    # step's input copies for the GEMMs that read the previous inputs
    cs_in, cs_out = torch.cuda.Stream(), torch.cuda.Stream()

    def step_overlapped(p):
        ev_in = {M: torch.cuda.Event() for M in wl.Ms}
        ev_gemm = {M: torch.cuda.Event() for M in wl.Ms}
        cs_in.wait_stream(stream)  # the previous step's GEMMs are done with dx
        with torch.cuda.stream(cs_in):
            for M in wl.Ms:
                dx[M].copy_(hx[M], non_blocking=True)
                ev_in[M].record(cs_in)
        for j, M in enumerate(wl.Ms):
            stream.wait_event(ev_in[M])
            wl.enqueue_fused(M, stream, wl.weights[(p * nper + j) % copies], x=dx[M])
            ev_gemm[M].record(stream)
        with torch.cuda.stream(cs_out):
            for M in wl.Ms:
                cs_out.wait_event(ev_gemm[M])
                hout[M].copy_(wl.out[M], non_blocking=True)
        stream.wait_stream(cs_out)  # outputs are back before the next step rewrites them

    with torch.cuda.stream(stream):
        if graph:
            g = capture(stream, lambda: [step_overlapped(p) for p in range(phases)])
            g.replay()
            stream.synchronize()
            reps = max(1, steps // phases)
            run = lambda: [g.replay() for _ in range(reps)]
            n = reps * phases
        else:
            for p in range(5):
                step(p % phases)
            stream.synchronize()
            run = lambda: [step(i % phases) for i in range(steps)]
            n = steps
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
    e1.synchronize()
    dt = e0.elapsed_time(e1) / 1e3
    return dt, n, h2d, d2h


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--profile-only", default=None, choices=sorted(PROFILE_SPECS),
                    help="run a few eager quant + GEMM launches of one workload and exit (for ncu)")
    ap.add_argument("--profile-m", type=int, default=None)
    ap.add_argument("--profile-iters", type=int, default=4)
    ap.add_argument("--kernel-hashes", action="store_true",
                    help="print the source hash of each kernel family (the key of profiles/traffic.md rows) and exit")
    args = ap.parse_args()
    if args.kernel_hashes:
        print(json.dumps({fam: kernel_hash(fam) for fam in KERNEL_FAMILIES}))
        return

    rank, world, local = dist_init()
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
            return
        if args.profile_only:
            run_profile_only(args)
            return
        run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


T0 = time.time()


def log(msg):
    sys.stderr.write(f"[bench {time.time() - T0:7.1f}s] {msg}\n")
    sys.stderr.flush()


def run_ours(args, rank, world, local):
    import mxfp4_gemm_transformer_b200 as mx
    mx.load()
    # weights are constant during the run, so the GEMM may start streaming them
    # before the preceding quantisation kernel has finished
    mx.mx_set_launch_flags(mx.MX_LAUNCH_PDL | mx.MX_LAUNCH_PREFETCH_WEIGHTS)
    pk = peaks()
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()

    dec = Workload(mx, "decode", DEC_MS, DEC_N, DEC_K, 0, 0, mx.MX_EPI_NONE, seed=1, with_bias=False,
                   desc=f"decode MXFP8 GEMM (fused q_a+kv shape) M in {list(DEC_MS)}, N={DEC_N}, K={DEC_K}, "
                        f"e4m3 W with 32x32 E8M0 scales, no bias, bf16 out")
    # eager warm-up on the capture stream sets kernel attributes before capture
    with torch.cuda.stream(stream):
        for M in dec.Ms:
            dec.enqueue_quant(M, stream)
            dec.enqueue_gemm(M, stream)
            dec.enqueue_fused(M, stream)
    stream.synchronize()
    assert mx.mx_workspace_status(dec.ws) == mx.MX_OK, "a GEMM gave up on a bounded wait"
    log("decode workload ready")
    steps_g = StepGraphs(dec, stream)
    log(f"captured the step graphs ({steps_g.phases} steps per rotation)")

    sampler = ClockSampler(torch.cuda.current_device())
    if rank == 0:
        sampler.start()
        time.sleep(0.3)
    # the warm-up steps run right before the timed region, so that it starts
    # on a busy GPU (not on clocks that dropped while the sampler started)
    with torch.cuda.stream(stream):
        steps_g.run(args.warmup)
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark_start()
    with torch.cuda.stream(stream):
        e0.record(stream)
        steps_g.run(args.steps)
        e1.record(stream)
    e1.synchronize()
    sampler.mark_stop()
    torch.cuda.synchronize()
    barrier(world)
    dt = e0.elapsed_time(e1) / 1e3
    dt = max_over_ranks(dt, world)
    log(f"timed region done: {dt * 1e3:.2f} ms for {args.steps} steps")
    if rank == 0:
        time.sleep(0.2)
        sampler.stop()
    clocks = sampler.summary() if rank == 0 else None
    assert mx.mx_workspace_status(dec.ws) == mx.MX_OK

    w_bytes_step = dec.w_bytes * len(dec.Ms)
    value = w_bytes_step * args.steps * world / dt / 1e9

    # the same step as separate quant + GEMM calls, for comparison
    unfused = StepGraphs(dec, stream, fused=False)
    n_unf = max(2 * unfused.phases, args.steps)
    unfused_ms = time_steps(unfused, stream, n_unf) / n_unf * 1e3
    del unfused

    # per-kernel timing of the dominant kernel (the decode GEMM on codes, the
    # kernel every call of the step runs), per M; "fused_us" is one mx_gemm
    # call on bf16 activations (quantisation + GEMM)
    per_m = {}
    for M in dec.Ms:
        tg, tq, tf = kernel_timing(dec, M, stream)
        plan = plan_info(mx, M, DEC_N, DEC_K, 0, 0, 0)
        pf = mx.mx_gemm_plan_info(M, DEC_N, DEC_K, mx.MX_A_BF16_E8M0_1X32, 0, 0, dec.ws.numel())
        per_m[M] = {"gemm_us": round(tg * 1e6, 3), "quant_us": round(tq * 1e6, 3), "fused_us": round(tf * 1e6, 3),
                    "act_quant": {1: "inside the decode kernel", 2: "quantisation kernel ahead"}.get(pf["act_quant"]),
                    "roofline": roofline_entry(dec, M, tg, pk, "hbm"), "plan": plan}
    log("per-kernel timing done")
    t_gemm_avg = sum(per_m[M]["gemm_us"] for M in dec.Ms) / len(dec.Ms) / 1e6
    bytes_avg = sum(dec.gemm_bytes(M) for M in dec.Ms) / len(dec.Ms)
    ach = bytes_avg / t_gemm_avg / 1e9
    traffic = ncu_traffic()
    for M in dec.Ms:
        per_m[M]["roofline"]["traffic"] = traffic.get(("decode", M))
    measured = [traffic[("decode", M)] for M in dec.Ms if ("decode", M) in traffic]
    roofline = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / pk["hbm_gbs"], 4),
                "traffic": round(sum(measured) / len(measured)) if measured else None,
                "traffic_note": "ncu dram read+write per launch, mean of the M values captured (profiles/traffic.md)",
                "kernel": "decode_kernel (the decode GEMM on e4m3 codes), mean over the four M values; algorithmic "
                          "bytes = weights + their scales + activation codes + scales + bf16 out",
                "peak_note": f"{pk['source']} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"}

    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 (E8M0 block scales, fp32 accumulate)",
            "data": "synthetic",
            "config": {"workload": dec.desc, "value_is": "weight bytes (codes + E8M0 scales) streamed per second",
                       "l2": f"{len(dec.weights)} rotating weight copies "
                             f"({len(dec.weights) * dec.w_bytes / 1e6:.0f} MB > 2x L2)",
                       "step": "4 x mx_gemm on bf16 activations (MX_A_BF16_E8M0_1X32: 1x32 E8M0 "
                               "quantisation by the quantisation kernel into the workspace, then the decode "
                               "GEMM); CUDA graphs of one walk through the weight "
                               f"rotation ({steps_g.phases} steps), single-step graphs for a remainder",
                       "launch": "programmatic dependent launch, weight prefetch allowed (constant weights)",
                       "parallelism": f"replica x{world}"},
            "step_unfused_ms": round(unfused_ms, 5),
            "roofline": roofline, "per_m": {str(k): v for k, v in per_m.items()},
            "clocks": clocks,
            # one launch per M when the decode kernel quantises, two when the
            # quantisation kernel runs ahead of it
            "gpu_launches": sum(2 if per_m[M]["act_quant"] == "quantisation kernel ahead" else 1
                                for M in dec.Ms) * args.steps}

    if not args.no_e2e:
        e_steps = max(50, min(2000, args.steps // 10))
        edt, en, h2d, d2h = e2e_measure(mx, dec, e_steps, stream, graph=False)
        edt = max_over_ranks(edt, world)
        eager = {"value": round(w_bytes_step * en * world / edt / 1e9, 2), "unit": "GB/s",
                 "note": "the same calls issued one by one from Python on one stream (copies and GEMMs in "
                         "sequence)"}
        try:
            gdt, gn, _, _ = e2e_measure(mx, dec, e_steps, stream, graph=True)
            gdt = max_over_ranks(gdt, world)
            line["e2e"] = {"value": round(w_bytes_step * gn * world / gdt / 1e9, 2), "unit": "GB/s",
                           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                           "note": "through the Python binding of the C ABI: per step and M, the bf16 activations "
                                   "copied in from pinned host memory, mx_gemm on them, the bf16 output copied "
                                   "back (copies on their own streams, overlapping the other problems' GEMMs); "
                                   "the steps captured in CUDA graphs and replayed",
                           "eager": eager}
        except Exception as e:  # capture refused: report the eager figure
            log(f"graph-captured e2e failed: {e!r}"[:300])
            line["e2e"] = dict(eager, h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h,
                               note="eager calls through the Python binding of the C ABI, pinned host buffers "
                                    "(graph capture failed: " + repr(e)[:120] + ")")

    log("e2e done")
    if not args.no_extra:
        line["other_workloads"] = extra_workloads(mx, stream, pk)

    if rank == 0 and world == 1 and not args.no_cpu:
        log("cpu baseline")
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)


# name -> (Ms, N, K, a_fmt, b_fmt, epi, seed, with_bias, bound, description)
PROFILE_SPECS = {
    "small": ((16,), 256, 512, 0, 0, 1, 0, True, "hbm", "small MXFP8 GEMM + bias (M16 N256 K512)"),
    "decode": (DEC_MS, DEC_N, DEC_K, 0, 0, 0, 1, False, "hbm",
               f"decode MXFP8 GEMM (fused q_a+kv shape) M in {list(DEC_MS)} N={DEC_N} K={DEC_K}"),
    "mlp": ((4096,), 4096, 4096, 0, 0, 2, 2, True, "tensor",
            "DiT/ViT MLP MXFP8 GEMM + bias + GELU-tanh (M4096 N4096 K4096)"),
    "gateup16": ((16,), 34816, 5120, 0, 1, 3, 3, False, "hbm", "W4A8 gate_up + SwiGLU, decode (M16 N34816 K5120)"),
    "gateup4096": ((4096,), 34816, 5120, 0, 1, 3, 3, False, "tensor",
                   "W4A8 gate_up + SwiGLU, prefill (M4096 N34816 K5120)"),
    "lmhead": ((16,), 248320, 5120, 1, 2, 0, 4, False, "hbm", "fp8 per-channel lm_head (M16 N248320 K5120)"),
    # the same FFN's neighbours: the gate_up handing its SwiGLU output on as MX
    # codes, the down projection that takes them, and the gate_up as W4A4
    "gateup16_mxq": ((16,), 34816, 5120, 0, 1, 5, 3, False, "hbm",
                     "W4A8 gate_up + SwiGLU -> e4m3 + 1x32 E8M0 codes, decode (M16 N34816 K5120)"),
    "down16": ((16,), 5120, 17408, 0, 1, 0, 5, False, "hbm", "W4A8 down projection, decode (M16 N5120 K17408)"),
    "down4096": ((4096,), 5120, 17408, 0, 1, 0, 5, False, "tensor",
                 "W4A8 down projection, prefill (M4096 N5120 K17408)"),
    "gateup4096_w4a4": ((4096,), 34816, 5120, 3, 1, 3, 3, False, "tensor",
                        "W4A4 gate_up + SwiGLU, prefill (M4096 N34816 K5120), kind::mxf4"),
}


def run_profile_only(args):
    """A few eager launches of one workload (for ncu captures): quant, GEMM on
    the codes and, for 1x32 E8M0 activations, the GEMM on bf16 activations."""
    import mxfp4_gemm_transformer_b200 as mx
    mx.load()
    Ms, N, K, af, bf, epi, seed, bias, _, desc = PROFILE_SPECS[args.profile_only]
    if args.profile_m is not None:
        Ms = (args.profile_m,)
    wl = Workload(mx, args.profile_only, Ms, N, K, af, bf, epi, seed=seed, with_bias=bias, desc=desc)
    stream = torch.cuda.current_stream()
    for _ in range(args.profile_iters):
        for M in wl.Ms:
            wl.enqueue_quant(M, stream)
            wl.enqueue_gemm(M, stream)
            if wl.can_fuse:
                wl.enqueue_fused(M, stream)
    torch.cuda.synchronize()
    st = mx.mx_workspace_status(wl.ws)
    print(json.dumps({"profile_only": args.profile_only, "Ms": list(wl.Ms), "status": st,
                      "plan": {M: plan_info(mx, M, N, K, af, bf, epi) for M in wl.Ms}}))
    if st != mx.MX_OK:
        sys.exit(3)


# routed-expert gate_up of a mixture-of-experts layer, W4A8 (the DeepSeek-V4
# mono runner page's w13 layout: [experts, 2 inter, hidden / 2] e2m1 with 1x32
# E8M0 scales), hidden 7168, 2 x inter = 1024, SwiGLU; the tokens routed to
# 8 local experts, unevenly, one expert empty
MOE_COUNTS = (448, 384, 320, 288, 256, 192, 160, 0)
MOE_N, MOE_K = 1024, 7168


def moe_grouped_workload(mx, stream, pk, seed=6):
    """One mx_gemm_grouped launch over every expert against one mx_gemm launch
    per non-empty expert, graphs of back-to-back launches over rotating
    weight copies (> 2x L2)."""
    import synth
    E, N, K = len(MOE_COUNTS), MOE_N, MOE_K
    offsets = [0]
    for c in MOE_COUNTS:
        offsets.append(offsets[-1] + c)
    M = offsets[-1]
    x = synth.bf16_matrix(seed, M, K, synth.X_SIGMA, device="cuda")
    ac, asc = mx.act_buffers(M, K)
    mx.mx_quant_act(x, ac, asc)
    wc = torch.empty(E * N, K // 2, dtype=torch.uint8, device="cuda")
    wsc = torch.empty(E * N, K // 32, dtype=torch.uint8, device="cuda")
    for e in range(E):
        w = synth.bf16_matrix(seed + 10 + e, N, K, synth.W_SIGMA, device="cuda")
        mx.mx_quant_weight(w, wc[e * N:(e + 1) * N], wsc[e * N:(e + 1) * N], mx.MX_B_E2M1_E8M0_1X32)
    torch.cuda.synchronize()
    w_bytes = wc.numel() + wsc.numel()
    copies = min(32, max(1, math.ceil(2 * L2_BYTES / w_bytes)))
    weights = [(wc, wsc)] + [(wc.clone(), wsc.clone()) for _ in range(copies - 1)]
    out = mx.out_buffer(M, N, mx.MX_EPI_SWIGLU)
    ws = mx.workspace()
    launches = max(copies, 8)

    def grouped_body():
        for i in range(launches):
            b, sb = weights[i % copies]
            mx.mx_gemm_grouped(ac, asc, 0, b, sb, 1, None, mx.MX_EPI_SWIGLU, out, offsets, N, K, ws, stream=stream)

    def per_expert_body():
        for i in range(launches):
            b, sb = weights[i % copies]
            for e in range(E):
                r0, r1 = offsets[e], offsets[e + 1]
                if r1 == r0:
                    continue
                mx.mx_gemm(ac[r0:r1], asc[r0:r1], 0, b[e * N:(e + 1) * N], sb[e * N:(e + 1) * N], 1, None,
                           mx.MX_EPI_SWIGLU, out[r0:r1], r1 - r0, N, K, ws, stream=stream)
    with torch.cuda.stream(stream):
        grouped_body()
        per_expert_body()
    stream.synchronize()
    assert mx.mx_workspace_status(ws) == mx.MX_OK
    tg = launch_time(capture(stream, grouped_body), launches, stream, 0.3)
    tp = launch_time(capture(stream, per_expert_body), launches, stream, 0.3)
    flops = 2.0 * M * N * K
    fp8_peak = 2.0 * pk["bf16_tflops"]
    ach = flops / tg / 1e12
    return {"workload": f"grouped MoE gate_up W4A8 + SwiGLU: {E} experts, rows {list(MOE_COUNTS)}, "
                        f"N={N} (2 x inter), K={K}",
            "gemm_us": round(tg * 1e6, 3), "per_expert_launches_us": round(tp * 1e6, 3),
            "tflops": round(ach, 2),
            "roofline": {"bound": "tensor", "achieved": round(ach, 1), "peak": round(fp8_peak, 1),
                         "unit": "TFLOP/s", "frac": round(ach / fp8_peak, 4), "traffic": None,
                         "peak_note": f"fp8 = 2 x {pk['source']} bf16 burst"},
            "rotating_copies": copies}


def extra_workloads(mx, stream, pk):
    """The other workloads, each GEMM timed alone (graph of back-to-back
    launches over rotating weights) against its roofline."""
    res = []
    for key in ("small", "mlp", "gateup16", "gateup4096", "lmhead", "gateup16_mxq", "down16", "down4096",
                "gateup4096_w4a4"):
        Ms, N, K, af, bf, epi, seed, bias, bound, name = PROFILE_SPECS[key]
        log(f"workload: {name}")
        try:
            wl = Workload(mx, name, Ms, N, K, af, bf, epi, seed=seed, with_bias=bias, desc=name)
            M = Ms[0]
            with torch.cuda.stream(stream):
                wl.enqueue_quant(M, stream)
                wl.enqueue_gemm(M, stream)
                if wl.can_fuse:
                    wl.enqueue_fused(M, stream)
            stream.synchronize()
            if mx.mx_workspace_status(wl.ws) != mx.MX_OK:
                raise RuntimeError("a GEMM gave up on a bounded wait")
            log("  warm-up ok")
            tg, tq, tf = kernel_timing(wl, M, stream)
            rl = roofline_entry(wl, M, tg, pk, bound)
            rl["traffic"] = ncu_traffic().get((key, M))
            entry = {"workload": name, "gemm_us": round(tg * 1e6, 3), "quant_us": round(tq * 1e6, 3),
                     "fused_us": None if tf is None else round(tf * 1e6, 3),
                     "plan": plan_info(mx, M, N, K, af, bf, epi),
                     "roofline": rl,
                     "tflops": round(wl.flops(M) / tg / 1e12, 2),
                     "weight_gbs": round(wl.w_bytes / tg / 1e9, 1),
                     "rotating_copies": len(wl.weights)}
            assert mx.mx_workspace_status(wl.ws) == mx.MX_OK
            res.append(entry)
            del wl
            torch.cuda.empty_cache()
        except Exception as e:  # report, keep going
            res.append({"workload": name, "error": repr(e)[:300]})
    log("workload: grouped MoE gate_up")
    try:
        res.append(moe_grouped_workload(mx, stream, pk))
    except Exception as e:
        res.append({"workload": "grouped MoE gate_up", "error": repr(e)[:300]})
    torch.cuda.empty_cache()
    return res


if __name__ == "__main__":
    main()
