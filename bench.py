#!/usr/bin/env python
"""Benchmark of the W2A8 BitLinear hot path on B200.

Headline workload: the W2A8 GEMV shape sweep at M = 1 (eight (N, K) shapes,
uniform int8 activations in [-127, 127], ternary weights with P = 1/3 each,
int32 output).  One step = one pass over the eight shapes, each through
bitnet_w2a8_gemm.  Metric: achieved HBM GB/s with algorithmic bytes
N*K/4 + M*K + 4*M*N per call; per-shape us/call are in "details".
Extra lines of "details": the large GEMV shapes, the BitLinear decode
(M = 1, bf16 in/out) and the prefill GEMM int8 TOPS (M >= 128).

Timing: inputs resident in HBM; the weights rotate over enough copies that
each step's set was last read more than 2x L2 capacity ago (no L2 reuse
between steps); each step is one CUDA-graph replay; CUDA events on the
launching stream; max over ranks.  `--impl reference` times the CPU oracle
instead (rank 0 only).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--quick]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from ternary_weight_bit_w2a8_b200 import synth  # noqa: E402

METRIC = "W2A8 GEMV us/call & HBM GB/s (% of peak) at M=1; int8 TOPS at M=128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES_DEFAULT = 126 * 2**20


def gemv_bytes(M, N, K):
    """Algorithmic bytes of one call: packed weights + int8 activations + int32 outputs."""
    return N * K / 4 + M * K + 4 * M * N


def bitlinear_bytes(M, N, K):
    return N * K / 4 + 2 * M * K + 2 * M * N


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while it runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, period_ms: int = 50):
        self.gpu_id = gpu_id
        self.period_ms = period_ms
        self.proc = None
        self.file = None

    def start(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms)], stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(2 * self.period_ms / 1000)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id_for(torch, dev):
    p = torch.cuda.get_device_properties(dev)
    try:
        return "GPU-" + str(p.uuid)
    except Exception:
        return f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"


# ----------------------------------------------------------------------------- helpers
def to_dev(torch, a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_dev(torch, bits):
    return to_dev(torch, bits.view(np.int16)).view(torch.bfloat16)


def max_over_ranks(torch, x, dist, device):
    """The largest value of x over all ranks (x itself without a process group)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbps(bytes_per_step_per_rank, steps, ms_max, world):
    """Whole-job throughput: the bytes all ranks processed over the slowest rank's time."""
    return world * bytes_per_step_per_rank * steps / (ms_max * 1e-3) / 1e9


def step_plan(steps, chunk):
    """How `timed_steps` covers exactly `steps` steps: [(first step, steps in
    the graph, replays)], a graph of `chunk` steps replayed while whole chunks
    remain, then one graph of the remainder."""
    n_big, rem = divmod(steps, chunk)
    plan = []
    if n_big:
        plan.append((0, chunk, n_big))
    if rem:
        plan.append((n_big * chunk, rem, 1))
    return plan


def timed_steps(torch, step_fn, steps, warmup, dist=None, chunk=448):
    """Times exactly `steps` steps: `step_fn(i0, n)` enqueues steps i0 .. i0 +
    n - 1 (step i decides its own rotation copy, so `chunk` is a multiple of
    the copy count).  The timed sequence is captured as at most two CUDA graphs
    (see step_plan), each replayed once beforehand, so that graph boundaries
    (a few us each) do not depend on the run length; `warmup` steps run
    untimed first.  Returns the elapsed ms (max over ranks)."""
    graphs = [(capture(torch, lambda i0=i0, n=n: step_fn(i0, n)), r) for (i0, n, r) in step_plan(steps, chunk)]
    for g, _ in graphs:
        g.replay()
    if warmup:
        step_fn(0, warmup)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for g, r in graphs:
        for _ in range(r):
            g.replay()
    end.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(torch, start.elapsed_time(end), dist, "cuda")
    if dist is not None:
        dist.barrier()
    del graphs
    return ms


def capture(torch, fn):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm the library (device info, function attributes) outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=s):
        fn()
    torch.cuda.synchronize()
    return g


def rotation_copies(total_bytes, l2_bytes):
    return max(3, int(math.ceil(2 * l2_bytes / max(total_bytes, 1))) + 1)


# ----------------------------------------------------------------------------- our arm
class GemvSet:
    """Device buffers for a list of M=1 GEMV shapes with rotating weight copies.
    The shapes' activations are views of one buffer, and so are their outputs,
    so that a step's inputs and results each cross the host link in one copy."""

    def __init__(self, torch, bn, shapes, gen, seed, l2_bytes, max_copies=None):
        self.torch, self.bn, self.shapes = torch, bn, shapes
        self.q, self.y, self.ws, self.packed0 = [], [], [], []
        # every K and N of these shapes keeps the views 16-byte aligned
        self.q_all = torch.empty(sum(K for _, K in shapes), dtype=torch.int8, device="cuda")
        self.y_all = torch.empty(sum(N for N, _ in shapes), dtype=torch.int32, device="cuda")
        total, qo, yo = 0, 0, 0
        for (N, K) in shapes:
            q, w = gen(N, K, seed=seed)
            qv = self.q_all[qo:qo + K].view(1, K)
            qv.copy_(to_dev(torch, q))
            self.q.append(qv)
            self.packed0.append(bn.bitnet_pack_weights(to_dev(torch, w)))
            del w
            self.y.append(self.y_all[yo:yo + N].view(1, N))
            self.ws.append(bn.workspace(1, N, K))
            total += bn.bitnet_packed_bytes(N, K)
            qo += K
            yo += N
        c = rotation_copies(total, l2_bytes)
        if max_copies:
            c = min(c, max_copies)
        self.copies = [self.packed0] + [[p.clone() for p in self.packed0] for _ in range(c - 1)]
        self.packed_total = total
        self.bytes_per_step = sum(gemv_bytes(1, N, K) for N, K in shapes)
        torch.cuda.synchronize()

    def run(self, c, events=None):
        for j, (N, K) in enumerate(self.shapes):
            if events is not None:
                events[j][0].record()
            self.bn.bitnet_w2a8_gemm(self.q[j], self.copies[c][j], N, y=self.y[j], ws=self.ws[j])
            if events is not None:
                events[j][1].record()


def measure_gemv_set(torch, bn, gs, steps, warmup, dist=None, clocks=None):
    """Headline: a step is the calls of all shapes back to back (linked by
    programmatic dependent launch) over one rotation copy, step i on copy i mod
    C.  Exactly `steps` steps are timed, captured in graphs of 64 rounds of the
    copies (see timed_steps)."""
    C = len(gs.copies)
    n_before = bn.bitnet_launch_count()
    gs.run(0)
    torch.cuda.synchronize()
    launches_per_step = bn.bitnet_launch_count() - n_before

    def step_fn(i0, n):
        for i in range(i0, i0 + n):
            gs.run(i % C)
    if clocks is not None:
        clocks.start()
    ms = timed_steps(torch, step_fn, steps, warmup, dist, chunk=64 * C)
    clk = clocks.stop() if clocks is not None else None
    return ms, launches_per_step, clk


def per_launch_us(torch, bn, gs, warmup, reps=30):
    """Average duration of one call of each shape: a graph of back-to-back calls
    of that shape over the rotating weight copies (each copy last read more than
    2x L2 capacity earlier), timed with CUDA events on the capturing stream."""
    out = []
    C = len(gs.copies)
    for j, (N, K) in enumerate(gs.shapes):
        L = 4 * C

        def step_fn(i0, n, j=j, N=N, L=L):  # a step: L back-to-back calls
            for _ in range(n):
                for i in range(L):
                    bn.bitnet_w2a8_gemm(gs.q[j], gs.copies[i % C][j], N, y=gs.y[j], ws=gs.ws[j])
        ms = timed_steps(torch, step_fn, reps, max(3, warmup // 10), chunk=reps)
        out.append(ms * 1e3 / (reps * L))
    return out


def e2e_sweep(torch, bn, gs, steps):
    """Through the public API with host buffers: each step copies the eight
    shapes' activations from pinned host memory to the device (one copy),
    makes the eight calls and copies their int32 results back to pinned host
    memory (one copy), then synchronises."""
    hq = gs.q_all.cpu().pin_memory()
    hy = torch.empty(gs.y_all.shape, dtype=torch.int32).pin_memory()
    h2d = hq.numel()
    d2h = hy.numel() * 4

    def step(i):
        gs.q_all.copy_(hq, non_blocking=True)
        for j, (N, K) in enumerate(gs.shapes):
            bn.bitnet_w2a8_gemm(gs.q[j], gs.copies[i % len(gs.copies)][j], N, y=gs.y[j], ws=gs.ws[j])
        hy.copy_(gs.y_all, non_blocking=True)
        torch.cuda.current_stream().synchronize()
    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        step(i)
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    return ms, h2d, d2h


E2E_SRC = os.path.join(ROOT, "bench_e2e.cu")
E2E_LIB = os.path.join(ROOT, "bench_e2e.so")


def build_e2e():
    """Compiles bench_e2e.cu (the C loop of the end-to-end leg) if needed."""
    if not os.path.exists(E2E_LIB) or os.path.getmtime(E2E_LIB) < os.path.getmtime(E2E_SRC):
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17", "-shared",
                        "-Xcompiler", "-fPIC", "--cudart", "static",
                        "-o", E2E_LIB + ".tmp", E2E_SRC, "-ldl"], check=True)
        os.replace(E2E_LIB + ".tmp", E2E_LIB)
    return E2E_LIB


def e2e_sweep_c(torch, bn, gs, steps):
    """The end-to-end sweep of e2e_sweep driven from C (bench_e2e.cu): the same
    copies and bitnet_w2a8_gemm calls with no interpreter between them."""
    import ctypes
    lib = ctypes.CDLL(build_e2e())
    fn = lib.e2e_sweep_loop
    fn.restype = ctypes.c_double
    P = ctypes.c_void_p
    fn.argtypes = [ctypes.c_char_p, ctypes.c_int, P, P, P, P, ctypes.c_int64, P, ctypes.c_int, P, P, P,
                   ctypes.c_int64, P, P, P, ctypes.c_int, P, ctypes.POINTER(ctypes.c_int)]
    S = len(gs.shapes)
    hq = gs.q_all.cpu().pin_memory()
    hy = torch.empty(gs.y_all.shape, dtype=torch.int32).pin_memory()
    arr = lambda ts: (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])  # noqa: E731
    Ns = (ctypes.c_int64 * S)(*[N for N, _ in gs.shapes])
    Ks = (ctypes.c_int64 * S)(*[K for _, K in gs.shapes])
    packed = arr([p for cp in gs.copies for p in cp])
    wsb = (ctypes.c_int64 * S)(*[w.numel() for w in gs.ws])
    status = ctypes.c_int(0)
    args = [bn.LIB_PATH.encode(), S, Ns, Ks, hq.data_ptr(), gs.q_all.data_ptr(), hq.numel(), arr(gs.q),
            len(gs.copies), packed, arr(gs.y), hy.data_ptr(), hy.numel() * 4, gs.y_all.data_ptr(), arr(gs.ws), wsb]
    stream = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    if fn(*args, 3, stream, ctypes.byref(status)) < 0:
        raise RuntimeError(f"e2e C loop failed (library status {status.value})")
    ms = fn(*args, steps, stream, ctypes.byref(status))
    if ms < 0:
        raise RuntimeError(f"e2e C loop failed (library status {status.value})")
    return ms


def measure_bitlinear_decode(torch, bn, shapes, warmup, l2_bytes, reps=30):
    """Fused BitLinear decode (bf16 in, bf16 out, weights ternarised and packed
    on the GPU): mean per-call time in a graph of back-to-back calls over
    rotating weight copies."""
    out = []
    for (N, K) in shapes:
        x, W = synth.bitlinear_inputs(1, N, K, seed=0)
        Wd = bf16_dev(torch, W)
        gamma = bn.bitnet_absmean(Wd)
        packed = bn.bitnet_pack_weights(bn.bitnet_ternarize(Wd, gamma))
        del Wd
        C = rotation_copies(packed.numel(), l2_bytes)
        copies = [packed] + [packed.clone() for _ in range(C - 1)]
        xd = bf16_dev(torch, x)
        y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
        ws = bn.workspace(1, N, K)
        L = 4 * C

        def run():
            for i in range(L):
                bn.bitnet_bitlinear(xd, copies[i % C], gamma, N, y=y, ws=ws)
        ms = timed_steps(torch, lambda i0, n, f=run: [f() for _ in range(n)], reps,
                         max(3, warmup // 10), chunk=reps)
        us = ms * 1e3 / (reps * L)
        out.append({"N": N, "K": K, "us_per_call": round(us, 3),
                    "GBps": round(bitlinear_bytes(1, N, K) / (us * 1e-6) / 1e9, 1)})
        del copies
    return out


def measure_small_batch(torch, bn, shapes, ms_list, warmup, l2_bytes, reps=30):
    """Small-batch decode (M tokens, one pass over the weights): int32 GEMM and
    BitLinear, mean per-call time in a graph of back-to-back calls over
    rotating weight copies (each copy last read more than 2x L2 earlier)."""
    out = []
    for (N, K) in shapes:
        q1, w = synth.uniform_int8_ternary(N, K, seed=0, M=max(ms_list))
        packed = bn.bitnet_pack_weights(to_dev(torch, w))
        del w
        C = rotation_copies(packed.numel(), l2_bytes)
        copies = [packed] + [packed.clone() for _ in range(C - 1)]
        gamma = torch.tensor([0.02], dtype=torch.float32, device="cuda")
        L = 4 * C
        for M in ms_list:
            q = to_dev(torch, q1[:M].copy())
            x = bf16_dev(torch, synth.bf16_activations(M, K, seed=M, outlier_p=0.01))
            y = torch.empty((M, N), dtype=torch.int32, device="cuda")
            yb = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            ws = bn.workspace(M, N, K)
            # the library's plan: one weight pass of the TMA GEMV (m16n8k32 MMA
            # product) up to 16 tokens, the tcgen05 GEMM beyond
            row = {"M": M, "N": N, "K": K, "path": "gemv_tma_mma" if M <= 16 else "gemm_tcgen05"}
            for name, fn in (("int32", lambda i: bn.bitnet_w2a8_gemm(q, copies[i % C], N, y=y, ws=ws)),
                             ("bitlinear", lambda i: bn.bitnet_bitlinear(x, copies[i % C], gamma, N, y=yb, ws=ws))):
                def run(fn=fn):
                    for i in range(L):
                        fn(i)
                ms = timed_steps(torch, lambda i0, n, f=run: [f() for _ in range(n)], reps,
                                 max(3, warmup // 10), chunk=reps)
                us = ms * 1e3 / (reps * L)
                nbytes = gemv_bytes(M, N, K) if name == "int32" else bitlinear_bytes(M, N, K)
                row[f"{name}_us_per_call"] = round(us, 3)
                row[f"{name}_GBps"] = round(nbytes / (us * 1e-6) / 1e9, 1)
            out.append(row)
        del copies
    return out


def measure_prefill(torch, bn, ms_list, shapes, warmup, int8_peak_tops, reps=20, L=10):
    """Prefill GEMM (tcgen05): mean per-call time in a graph of L back-to-back
    calls, int32 out (int8 TOPS = 2*M*N*K / time) and the whole BitLinear (bf16
    in: quantisation pass + GEMM with the bf16 epilogue)."""
    out = []
    for (N, K) in shapes:
        W = synth.bf16_weights(N, K, seed=1)
        Wd = bf16_dev(torch, W)
        gamma = bn.bitnet_absmean(Wd)
        packed = bn.bitnet_pack_weights(bn.bitnet_ternarize(Wd, gamma))
        del Wd
        for M in ms_list:
            x = synth.bf16_activations(M, K, seed=0, outlier_p=0.0)
            xd = bf16_dev(torch, x)
            q, s, _ = bn.bitnet_quant_act(xd)
            y = torch.empty((M, N), dtype=torch.int32, device="cuda")
            ws = bn.workspace(M, N, K)

            def run():
                for _ in range(L):
                    bn.bitnet_w2a8_gemm(q, packed, N, y=y, ws=ws)
            ms = timed_steps(torch, lambda i0, n, f=run: [f() for _ in range(n)], reps,
                             max(3, warmup // 10), chunk=reps)
            us = ms * 1e3 / (reps * L)
            tops = 2.0 * M * N * K / (us * 1e-6) / 1e12
            yb = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            wsb = bn.workspace(M, N, K)

            def run_bl():
                for _ in range(L):
                    bn.bitnet_bitlinear(xd, packed, gamma, N, y=yb, ws=wsb)
            ms_bl = timed_steps(torch, lambda i0, n, f=run_bl: [f() for _ in range(n)], reps,
                             max(3, warmup // 10), chunk=reps)
            us_bl = ms_bl * 1e3 / (reps * L)
            out.append({"M": M, "N": N, "K": K, "us_per_call": round(us, 2), "int8_TOPS": round(tops, 1),
                        "frac_int8_peak": round(tops / int8_peak_tops, 4),
                        "GBps": round(gemv_bytes(M, N, K) / (us * 1e-6) / 1e9, 1),
                        "bitlinear_us_per_call": round(us_bl, 2),
                        "bitlinear_TOPS": round(2.0 * M * N * K / (us_bl * 1e-6) / 1e12, 1)})
    return out


def measure_bf16_context(torch, shapes, warmup, l2_bytes, reps=30):
    """Context only (the pages compare their kernel with torch.matmul in bf16):
    cuBLAS bf16 GEMV [1, K] x [K, N] for the sweep shapes, weights rotating as
    for the W2A8 calls, mean per-call time in a graph of back-to-back calls."""
    out = []
    for (N, K) in shapes:
        w = torch.randn((K, N), device="cuda", dtype=torch.bfloat16)
        C = rotation_copies(w.numel() * 2, l2_bytes)
        ws = [w] + [w.clone() for _ in range(C - 1)]
        x = torch.randn((1, K), device="cuda", dtype=torch.bfloat16)
        y = torch.empty((1, N), device="cuda", dtype=torch.bfloat16)
        L = 4 * C

        def run():
            for i in range(L):
                torch.matmul(x, ws[i % C], out=y)
        ms = timed_steps(torch, lambda i0, n, f=run: [f() for _ in range(n)], reps,
                         max(3, warmup // 10), chunk=reps)
        us = ms * 1e3 / (reps * L)
        out.append({"N": N, "K": K, "bf16_us_per_call": round(us, 3),
                    "GBps": round((2 * N * K + 2 * K + 2 * N) / (us * 1e-6) / 1e9, 1)})
        del ws
        torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, dist):
    import torch
    import ternary_weight_bit_w2a8_b200 as bn
    from ternary_weight_bit_w2a8_b200 import build
    if rank == 0 or not os.path.exists(bn.LIB_PATH):
        build.build()
    if dist is not None:
        dist.barrier()
    dev = torch.cuda.current_device()
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 0) or L2_BYTES_DEFAULT
    peaks = load_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    int8_peak = 2.0 * float(peaks["bf16_tflops"])  # dense int8 = 2x dense bf16 (nominal ratio)

    gs = GemvSet(torch, bn, synth.SWEEP_SHAPES, synth.uniform_int8_ternary, seed=rank, l2_bytes=l2)
    clocks = ClockSampler(gpu_id_for(torch, dev)) if rank == 0 else None
    ms, launches_per_step, clk = measure_gemv_set(torch, bn, gs, args.steps, args.warmup, dist, clocks)
    per_shape_us = per_launch_us(torch, bn, gs, args.warmup)
    ms_per_step = ms / args.steps
    value = job_gbps(gs.bytes_per_step, args.steps, ms, world)
    kern_us = sum(per_shape_us)
    achieved = gs.bytes_per_step / (kern_us * 1e-6) / 1e9

    e2e_steps = max(3, min(args.steps, 300))
    e2e_ms, h2d, d2h = e2e_sweep(torch, bn, gs, e2e_steps)
    e2e_ms = max_over_ranks(torch, e2e_ms, dist, "cuda")
    e2e_value = job_gbps(gs.bytes_per_step, e2e_steps, e2e_ms, world)
    e2e_c_ms = max_over_ranks(torch, e2e_sweep_c(torch, bn, gs, e2e_steps), dist, "cuda")
    e2e_c_value = job_gbps(gs.bytes_per_step, e2e_steps, e2e_c_ms, world)

    details = {"sweep": [{"N": N, "K": K, "us_per_call": round(u, 3),
                          "GBps": round(gemv_bytes(1, N, K) / (u * 1e-6) / 1e9, 1),
                          "frac_hbm": round(gemv_bytes(1, N, K) / (u * 1e-6) / 1e9 / hbm_peak, 4)}
                         for (N, K), u in zip(synth.SWEEP_SHAPES, per_shape_us)]}
    del gs
    torch.cuda.empty_cache()
    if not args.quick and rank == 0:
        gl = GemvSet(torch, bn, synth.LARGE_SHAPES, synth.sparse_ternary_normal_int8, seed=0, l2_bytes=l2)
        us_l = per_launch_us(torch, bn, gl, args.warmup)
        details["large"] = [{"N": N, "K": K, "us_per_call": round(u, 3),
                             "GBps": round(gemv_bytes(1, N, K) / (u * 1e-6) / 1e9, 1),
                             "frac_hbm": round(gemv_bytes(1, N, K) / (u * 1e-6) / 1e9 / hbm_peak, 4)}
                            for (N, K), u in zip(synth.LARGE_SHAPES, us_l)]
        del gl
        torch.cuda.empty_cache()
        details["bitlinear_decode"] = measure_bitlinear_decode(torch, bn, synth.BITLINEAR_DECODE_SHAPES,
                                                               args.warmup, l2)
        details["small_batch"] = measure_small_batch(torch, bn, synth.BITLINEAR_DECODE_SHAPES, [2, 4, 8, 12, 16, 32, 64],
                                                     args.warmup, l2)
        details["prefill"] = measure_prefill(torch, bn, synth.PREFILL_M, synth.PREFILL_SHAPES, args.warmup, int8_peak)
        bf = measure_bf16_context(torch, synth.SWEEP_SHAPES, args.warmup, l2)
        for row, ours in zip(bf, details["sweep"]):
            row["w2a8_us_per_call"] = ours["us_per_call"]
            row["speedup_w2a8_vs_bf16"] = round(row["bf16_us_per_call"] / ours["us_per_call"], 2)
        details["bf16_matmul_context"] = bf
        details["int8_peak_tops"] = {"value": round(int8_peak, 1),
                                     "basis": f"{peaks['source']} bf16 dense x 2 (nominal int8/bf16 ratio)"}

    err = bn.bitnet_get_device_error()
    traffic = read_traffic()
    if traffic is not None:
        traffic = round(traffic, 1)
    return {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8xint2->int32", "data": "synthetic",
        "config": {"workload": "W2A8 GEMV M=1 shape sweep, 8 (N,K) shapes, int32 out",
                   "shapes": [list(s) for s in synth.SWEEP_SHAPES],
                   "l2": f"weights rotate over {len(synth.SWEEP_SHAPES)}-shape sets, "
                         f"{rotation_copies(sum(N * K // 4 for N, K in synth.SWEEP_SHAPES), l2)} copies "
                         f"(> 2x L2 of {l2 // 2**20} MiB between reuses)",
                   "step": "the 8 bitnet_w2a8_gemm calls over one rotation copy; CUDA graphs of one step per "
                           "copy, run as one graph of all copies in turn plus single steps for the remainder",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "seed": "rank"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                     "traffic_source": "profiles/traffic_gemv_tma_sweep.json (ncu dram__bytes_read.sum + "
                                       "dram__bytes_write.sum, mean over the 8 sweep launches); null when the "
                                       "kernel sources changed since that capture",
                     "kernel": "gemv_tma_kernel", "peak_source": peaks["source"],
                     "per_launch_bytes": "N*K/4 + K + 4N per shape, mean over the 8 shapes",
                     "duration": "mean per-call time of each shape in a graph of back-to-back calls over rotating "
                                 "weight copies (CUDA events)"},
        "clocks": clk,
        "e2e": {"value": round(e2e_c_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "us_per_step": round(e2e_c_ms * 1e3 / e2e_steps, 2),
                "note": "through the C ABI with host buffers (bench_e2e.cu): every step copies the eight shapes' "
                        "int8 activations in from pinned host memory (one copy), makes the eight bitnet_w2a8_gemm "
                        "calls, copies their int32 results out to pinned host memory (one copy) and synchronises "
                        "the stream; packed weights resident",
                "python": {"value": round(e2e_value, 2), "unit": "GB/s",
                           "us_per_step": round(e2e_ms * 1e3 / e2e_steps, 2),
                           "note": "the same step through the Python binding (torch tensors, ctypes)"}},
        "gpu_launches": int(launches_per_step * args.steps),
        "device_error": err,
        "details": details,
    }


# ----------------------------------------------------------------------------- CPU arms
def oracle_sweep_step(shapes_data, frac, step):
    """One oracle pass over a row sample of every sweep shape; returns algorithmic bytes processed."""
    import oracle
    done = 0.0
    for (q, w, N, K) in shapes_data:
        rows = max(1, int(N * frac))
        r0 = (step * rows) % N
        first = min(rows, N - r0)
        oracle.gemm_i32(q, w[r0:r0 + first])  # contiguous row blocks: no copy
        if first < rows:
            oracle.gemm_i32(q, w[:rows - first])
        done += gemv_bytes(1, rows, K)
    return done


def cpu_threads():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else (os.cpu_count() or 1)


def cpu_baseline_one_thread(budget_s=4.0):
    """The same oracle sample on one host thread: a child process with
    OMP_NUM_THREADS=1 (the OpenMP thread count is fixed when a process first
    uses it)."""
    env = dict(os.environ)
    env["OMP_NUM_THREADS"] = "1"
    r = subprocess.run([sys.executable, os.path.abspath(__file__), "--cpu-baseline-only",
                        "--cpu-budget", str(budget_s)], env=env, capture_output=True, text=True, timeout=600)
    if r.returncode != 0:
        return {"error": r.stderr.strip().splitlines()[-1:] or ["failed"]}
    return json.loads(r.stdout.strip().splitlines()[-1])


def cpu_baseline(budget_s=4.0):
    """The oracle, as it stands, on a bounded row sample of the sweep."""
    import oracle
    oracle._lib()
    data = []
    for (N, K) in synth.SWEEP_SHAPES:
        q, w = synth.uniform_int8_ternary(N, K, seed=0)
        data.append((q, w, N, K))
    frac = 1.0 / 16
    t0 = time.perf_counter()
    oracle_sweep_step(data, frac, 0)
    t1 = time.perf_counter()
    reps = max(1, int(budget_s / max(t1 - t0, 1e-6)))
    done = 0.0
    t0 = time.perf_counter()
    for i in range(reps):
        done += oracle_sweep_step(data, frac, i + 1)
    dt = time.perf_counter() - t0
    return {"value": round(done / dt / 1e9, 3), "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{reps} passes over 1/16 of the rows of each of the 8 sweep shapes "
                      f"(algorithmic bytes of the rows processed), {dt:.1f} s"}


def run_reference(args):
    import oracle
    oracle._lib()
    data = []
    for (N, K) in synth.SWEEP_SHAPES:
        q, w = synth.uniform_int8_ternary(N, K, seed=0)
        data.append((q, w, N, K))
    t0 = time.perf_counter()
    oracle_sweep_step(data, 1.0 / 64, 0)
    t_probe = (time.perf_counter() - t0) * 64  # seconds for one full sweep
    budget = args.ref_budget / max(1, args.steps + args.warmup)  # whole run within the budget
    frac = min(1.0, budget / max(t_probe, 1e-9))
    for i in range(args.warmup):
        oracle_sweep_step(data, frac, i)
    done = 0.0
    t0 = time.perf_counter()
    for i in range(args.steps):
        done += oracle_sweep_step(data, frac, args.warmup + i)
    dt = time.perf_counter() - t0
    value = done / dt / 1e9
    sample = f"each step: {frac:.3g} of the rows of each of the 8 sweep shapes"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8xint2->int32",
            "data": "synthetic",
            "config": {"workload": "W2A8 GEMV M=1 shape sweep, 8 (N,K) shapes, int32 out",
                       "shapes": [list(s) for s in synth.SWEEP_SHAPES]},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "kind": "oracle", "cores": cpu_threads(),
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


TRAFFIC_DATA = os.path.join(ROOT, "profiles", "traffic_gemv_tma_sweep.json")
TRAFFIC_SOURCES = ("common.cuh", "quant.cuh", "gemv.cuh", "gemv_tma.cuh")
# the tensor-core GEMM's section of the translation unit (not part of the GEMV)
TC_SECTION = ("// ------------------------------------------------------------------ tcgen05 GEMM (M > 1)",
              "// ------------------------------------------------------------------ dispatch")


def kernel_source_hash():
    """sha256 over the sources that decide the GEMV kernel and its launch: its
    headers and the translation unit without the tensor-core GEMM's section."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "ternary_weight_bit_w2a8_b200", "csrc")
    for name in TRAFFIC_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    with open(os.path.join(csrc, "bitnet_b200.cu"), encoding="utf-8") as f:
        tu = f.read()
    a = tu.find(TC_SECTION[0])
    b = tu.find(TC_SECTION[1], a + 1) if a >= 0 else -1
    if a >= 0 and b > a:
        tu = tu[:a] + tu[b:]
    h.update(tu.encode("utf-8"))
    return h.hexdigest()


def read_traffic(path=TRAFFIC_DATA):
    """DRAM bytes per launch (read + write, mean over the sweep's launches) from
    the committed ncu capture's data file, or None when the kernel sources
    changed since that capture."""
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("source_sha256") != kernel_source_hash() or d.get("traffic_bytes_per_launch") is None:
        return None
    return float(d["traffic_bytes_per_launch"])


def run_profile(args):
    """`warmup + steps` plain calls, no graphs: the int32 contraction of one
    problem (M,N,K) over rotating weight copies, of each sweep shape at M = 1
    in order (`sweep`), the activation quantisation (`quant,M,K`) or the
    BitLinear forward (`bitlinear,M,N,K`)."""
    import torch
    import ternary_weight_bit_w2a8_b200 as bn
    if args.profile == "sweep":
        l2 = torch.cuda.get_device_properties(0).L2_cache_size
        gs = GemvSet(torch, bn, synth.SWEEP_SHAPES, synth.uniform_int8_ternary, seed=0, l2_bytes=l2)
        for i in range(args.warmup + args.steps):
            gs.run(i % len(gs.copies))
        torch.cuda.synchronize()
        print(json.dumps({"profile": "sweep", "calls": (args.warmup + args.steps) * len(gs.shapes),
                          "device_error": bn.bitnet_get_device_error()}))
        return 0
    parts = args.profile.split(",")
    if parts[0] in ("quant", "bitlinear"):
        # bf16 activations: the quantisation pass alone (quant,M,K) or the whole
        # BitLinear forward (bitlinear,M,N,K), weights ternarised on the GPU
        M, K = int(parts[1]), int(parts[-1])
        x = bf16_dev(torch, synth.bf16_activations(M, K, seed=0, outlier_p=0.0))
        if parts[0] == "quant":
            q, s, r = bn.bitnet_quant_act(x)
            fn = lambda: bn.bitnet_quant_act(x, q=q, s=s, rowsum=r)  # noqa: E731
        else:
            N = int(parts[2])
            Wd = bf16_dev(torch, synth.bf16_weights(N, K, seed=1))
            gamma = bn.bitnet_absmean(Wd)
            packed = bn.bitnet_pack_weights(bn.bitnet_ternarize(Wd, gamma))
            del Wd
            y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            ws = bn.workspace(M, N, K)
            fn = lambda: bn.bitnet_bitlinear(x, packed, gamma, N, y=y, ws=ws)  # noqa: E731
        for _ in range(args.warmup + args.steps):
            fn()
        torch.cuda.synchronize()
        print(json.dumps({"profile": parts, "calls": args.warmup + args.steps,
                          "device_error": bn.bitnet_get_device_error()}))
        return 0
    M, N, K = (int(v) for v in parts)
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    gen = synth.sparse_ternary_normal_int8 if (N, K) in synth.LARGE_SHAPES else synth.uniform_int8_ternary
    q, w = gen(N, K, seed=0, M=M)
    qd = to_dev(torch, q)
    packed = bn.bitnet_pack_weights(to_dev(torch, w))
    del w
    copies = [packed] + [packed.clone() for _ in range(rotation_copies(packed.numel(), l2) - 1)]
    y = torch.empty((M, N), dtype=torch.int32, device="cuda")
    ws = bn.workspace(M, N, K)
    for i in range(args.warmup + args.steps):
        bn.bitnet_w2a8_gemm(qd, copies[i % len(copies)], N, y=y, ws=ws)
    torch.cuda.synchronize()
    print(json.dumps({"profile": [M, N, K], "calls": args.warmup + args.steps,
                      "device_error": bn.bitnet_get_device_error()}))
    return 0


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true", help="headline only (skip the details workloads)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=90.0,
                    help="seconds of oracle work for the whole --impl reference run")
    ap.add_argument("--cpu-baseline-only", action="store_true",
                    help="print the oracle's CPU baseline (the threads OMP_NUM_THREADS allows) and exit")
    ap.add_argument("--cpu-budget", type=float, default=4.0, help="seconds of oracle work for the CPU baseline")
    ap.add_argument("--profile", metavar="M,N,K|sweep|quant,M,K|bitlinear,M,N,K",
                    help="profiling mode (for ncu): `warmup + steps` plain calls of bitnet_w2a8_gemm on one "
                         "problem or on each sweep shape, of bitnet_quant_act, or of bitnet_bitlinear")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.cpu_baseline_only:
        print(json.dumps(cpu_baseline(args.cpu_budget)), flush=True)
        return 0

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    if args.profile:
        return run_profile(args)

    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the CUDA path has no CPU fallback)")
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    try:
        res = run_ours(args, rank, world, dist)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(args.cpu_budget)
            res["cpu_baseline"]["host_cpu_count"] = os.cpu_count()
            res["cpu_baseline"]["one_thread"] = cpu_baseline_one_thread(args.cpu_budget)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
