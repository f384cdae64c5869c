#!/usr/bin/env python
"""Benchmark of the B200 W4A16 quantized linear layer.

Headline (one JSON line on rank 0): decode GEMV throughput in GB/s of algorithmic traffic on
the Llama-3-8B linear shapes (K x N = 4096x6144, 4096x4096, 4096x28672, 14336x4096) at
M = 1, 4, 8, 16 tokens, W4 g128 weights packed by the library's own quantize kernel.  One
step is the 16 GEMV calls of that sweep, replayed as a CUDA graph.  Each (shape, M) call
uses its own copy of the packed weights, so a step touches 453 MB, well above the 126 MB
L2.  Extra keys report the prefill GEMM (TFLOP/s) on the same shapes at M = 512, 2048 and
8192, and the quantize kernel (GB/s).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 runs one process per GPU (torchrun); the path does not shard, so every rank runs an
independent replica of the workload ("scaling": "weak").  Time is the max over ranks.
--impl reference times the CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "W4A16 GEMV achieved GB/s (% HBM peak); GEMM TFLOPS (% bf16 TC peak)"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATA = "synthetic: seeded N(0, 0.02^2) weights, lognormal-channel activations (no checkpoints)"
GEMV_SHAPES = workloads.LLAMA3_8B
GEMV_MS = workloads.DECODE_SWEEP["Ms"]
GEMM_MS = workloads.PREFILL_SWEEP["Ms"]
WORKLOAD = ("decode GEMV sweep, Llama-3-8B linear shapes (K x N = 4096x6144, 4096x4096, 4096x28672, "
            "14336x4096) x M in {1, 4, 8, 16}, W4 g128 (alpha 0.5)")


def gemv_bytes(N: int, K: int, M: int) -> int:
    """Algorithmic bytes of one GEMV call: packed weights + bf16 x + bf16 y."""
    return workloads.packed_bytes(N, K) + 2 * M * K + 2 * M * N


def sweep_config(world: int) -> dict:
    """The workload's `config`, the same for both arms."""
    step_bytes = sum(gemv_bytes(N, K, M) for _, K, N in GEMV_SHAPES for M in GEMV_MS)
    return {"workload": WORKLOAD, "M": GEMV_MS, "step": "16 GEMV calls (4 shapes x 4 M), one CUDA graph",
            "l2": "inputs larger than L2: one packed-weight copy per call, %.0f MB per step" % (step_bytes / 1e6),
            "parallelism": f"replicas x{world}"}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK}, "measured"
    return dict(FALLBACK), "fallback"


# ------------------------------------------------------------------ distributed plumbing --

def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(value: float, world: int) -> float:
    """Max over ranks (the timed region's length of the slowest replica)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(ms_local: float, bytes_local: float, world: int):
    """Whole-job throughput: the units all ranks processed over the max time of any rank."""
    ms = reduce_max(ms_local, world)
    return ms, bytes_local * world / (ms * 1e-3) / 1e9


# ------------------------------------------------------------------ clocks -----------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.sel = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.sel = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.sel:
            cmd += ["-i", self.sel]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
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
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------ CPU oracle timing ------

def oracle_sample(budget_s: float):
    """Time the CPU oracle on sampled outputs of the GEMV sweep for about budget_s seconds.
    Returns (GB/s-equivalent, seconds, outputs, description).  Each sampled output (m, n) of a
    call accounts for bytes_call / (M * N) algorithmic bytes."""
    import oracle
    oracle.build()
    rng = np.random.default_rng(12345)
    calls = []
    for si, (name, K, N) in enumerate(GEMV_SHAPES):
        L = workloads.make_layer(workloads.seed_of(1, si), K=K, N=N)
        qw, sc, z, _ = oracle.awq_quantize_g128(L.W, L.act_absmean, workloads.ALPHA)
        for M in GEMV_MS:
            x = workloads.make_activations(workloads.seed_of(1, si), M, L.mult)
            calls.append((K, N, M, qw, sc, z, x))

    def run(P):
        t, b = 0.0, 0.0
        for K, N, M, qw, sc, z, x in calls:
            m = rng.integers(0, M, P)
            n = rng.integers(0, N, P)
            t0 = time.perf_counter()
            oracle.linear_at(x, qw, sc, z, N, m, n)
            t += time.perf_counter() - t0
            b += gemv_bytes(N, K, M) / (M * N) * P
        return t, b

    t_cal, _ = run(64)
    P = int(max(64, min(1 << 20, 64 * budget_s / max(t_cal, 1e-6))))
    t, b = run(P)
    desc = (f"oracle.linear_at (C, fp64 accumulation, OpenMP over outputs): {P} sampled outputs of each of "
            f"the 16 calls of the sweep ({16 * P} outputs); each output counts call bytes / (M*N)")
    return b / t / 1e9, t, 16 * P, desc


def omp_threads() -> int:
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v and v.isdigit() else (os.cpu_count() or 1)


# ------------------------------------------------------------------ reference arm ----------

def run_reference(args, world, rank):
    if rank != 0:
        return
    import oracle
    oracle.build()
    # one layer of the sweep per step, rotating; a fixed number of sampled outputs per step,
    # sized so that warmup + steps take about two minutes
    layers = []
    for si, (name, K, N) in enumerate(GEMV_SHAPES):
        L = workloads.make_layer(workloads.seed_of(1, si), K=K, N=N)
        qw, sc, z, _ = oracle.awq_quantize_g128(L.W, L.act_absmean, workloads.ALPHA)
        xs = {M: workloads.make_activations(workloads.seed_of(1, si), M, L.mult) for M in GEMV_MS}
        layers.append((K, N, qw, sc, z, xs))
    rng = np.random.default_rng(7)

    def one_step(i, P):
        K, N, qw, sc, z, xs = layers[i % len(layers)]
        M = GEMV_MS[(i // len(layers)) % len(GEMV_MS)]
        m = rng.integers(0, M, P)
        n = rng.integers(0, N, P)
        t0 = time.perf_counter()
        oracle.linear_at(xs[M], qw, sc, z, N, m, n)
        return time.perf_counter() - t0, gemv_bytes(N, K, M) / (M * N) * P

    dt, _ = one_step(0, 512)
    per_out = dt / 512
    budget = args.ref_budget
    P = int(max(16, min(1 << 16, budget / max(args.steps + args.warmup, 1) / per_out)))
    for i in range(args.warmup):
        one_step(i, P)
    t_tot, b_tot = 0.0, 0.0
    for i in range(args.steps):
        dt, b = one_step(i, P)
        t_tot += dt
        b_tot += b
    value = b_tot / t_tot / 1e9
    line = {"metric": METRIC, "impl": "reference", "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_tot / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": DATA,
            "config": sweep_config(world),
            "sample": f"each step: {P} sampled outputs of one (layer, M) of the sweep, computed by the oracle",
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": omp_threads(), "kind": "oracle",
                             "sample": f"{P} sampled GEMV outputs per step over {args.steps} steps"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm ---------------

def build_gemv_workload(torch, w4):
    calls = []
    quant = []
    for si, (name, K, N) in enumerate(GEMV_SHAPES):
        L = workloads.make_layer(workloads.seed_of(1, si), K=K, N=N)
        W = torch.from_numpy(L.W).cuda()
        act = torch.from_numpy(L.act_absmean).cuda()
        qw, sc, z, s = w4.awq_quantize_g128(W, act, workloads.ALPHA)
        w4.check_device_status()
        quant.append((W, act, N, K))
        for j, M in enumerate(GEMV_MS):
            if j == 0:
                packed = (qw, sc, z)
            else:
                packed = (qw.clone(), sc.clone(), z.clone())
            xh = workloads.make_activations(workloads.seed_of(1, si), M, L.mult)
            x = torch.from_numpy(xh.view(np.int16)).view(torch.bfloat16).cuda()
            y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            calls.append(dict(x=x, w=packed, y=y, M=M, N=N, K=K, bytes=gemv_bytes(N, K, M)))
    return calls, quant


STEPS_PER_GRAPH = 8


def capture_steps(torch, fn, n):
    """A CUDA graph of n consecutive calls of fn (fn has run eagerly before)."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        for _ in range(n):
            fn()
    return g


def time_steps(torch, fn, steps, warmup):
    """ms per call of fn, replayed as graphs of STEPS_PER_GRAPH calls (plus single ones)."""
    fn()
    torch.cuda.synchronize()
    g_many, g_one = capture_steps(torch, fn, STEPS_PER_GRAPH), capture_steps(torch, fn, 1)
    for _ in range(warmup):
        g_one.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps // STEPS_PER_GRAPH):
        g_many.replay()
    for _ in range(steps % STEPS_PER_GRAPH):
        g_one.replay()
    e1.record()
    torch.cuda.synchronize()
    del g_many, g_one
    return e0.elapsed_time(e1) / steps


def time_graph(torch, fn, steps, warmup):
    """Capture fn() once, replay warmup + steps times; CUDA-event ms per replay."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        fn()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, g


def run_gpu(args, world, rank, local):
    import torch

    import w4a16_gemm_awq_b200 as w4
    pk, pk_kind = peaks()
    calls, quant = build_gemv_workload(torch, w4)
    # one zeroed workspace, reused by every call in stream order (each call leaves it zeroed)
    ws = torch.zeros(max(w4.workspace_bytes(16, c["N"], c["K"]) for c in calls), dtype=torch.uint8,
                     device="cuda")

    def step():
        for c in calls:
            qw, sc, z = c["w"]
            w4.w4a16_gemv(c["x"], qw, sc, z, out=c["y"], workspace=ws)

    step_bytes = sum(c["bytes"] for c in calls)
    # warmup (eager, then graph), then the timed region: barrier + sync on both sides
    for _ in range(max(args.warmup, 3)):
        step()
    w4.check_device_status()
    # Graphs of STEPS_PER_GRAPH steps (and of one step for the remainder), so that the gap
    # between graph launches is paid once per several steps, as in a decode loop; exactly
    # args.steps steps run inside the timed region.
    g_many, g_one = capture_steps(torch, step, STEPS_PER_GRAPH), capture_steps(torch, step, 1)
    for _ in range(args.warmup):
        g_one.replay()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    e0.record(stream)
    for _ in range(args.steps // STEPS_PER_GRAPH):
        g_many.replay()
    for _ in range(args.steps % STEPS_PER_GRAPH):
        g_one.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    w4.check_device_status()
    ms_local = e0.elapsed_time(e1) / args.steps
    ms, gbs = aggregate(ms_local, step_bytes, world)
    del g_many, g_one

    # End to end through the public API with host buffers: the step's activations go from one
    # pinned host buffer to the device in one copy, the 16 GEMVs run, and their outputs come
    # back in one copy (a decode step moves its batch once, not once per layer call).
    xs_n = [c["x"].numel() for c in calls]
    ys_n = [c["y"].numel() for c in calls]
    hx_all = torch.cat([c["x"].reshape(-1).cpu() for c in calls]).pin_memory()
    hy_all = torch.empty(sum(ys_n), dtype=torch.bfloat16).pin_memory()
    dx_all = torch.empty(sum(xs_n), dtype=torch.bfloat16, device="cuda")
    dy_all = torch.empty(sum(ys_n), dtype=torch.bfloat16, device="cuda")
    xe, ye, ox, oy = [], [], 0, 0
    for c, nx, ny in zip(calls, xs_n, ys_n):
        xe.append(dx_all[ox:ox + nx].view(c["x"].shape))   # offsets stay 16-byte aligned: K, N multiples of 8
        ye.append(dy_all[oy:oy + ny].view(c["y"].shape))
        ox += nx
        oy += ny

    def e2e_step():
        dx_all.copy_(hx_all, non_blocking=True)
        for c, x_, y_ in zip(calls, xe, ye):
            qw, sc, z = c["w"]
            w4.w4a16_gemv(x_, qw, sc, z, out=y_, workspace=ws)
        hy_all.copy_(dy_all, non_blocking=True)

    e2e_steps = max(1, min(args.steps, 2000))
    ms_e2e = time_steps(torch, e2e_step, e2e_steps, max(args.warmup, 3))
    ms_e2e = reduce_max(ms_e2e, world)
    h2d = dx_all.numel() * 2
    d2h = dy_all.numel() * 2

    # The same sweep on raw activations with the 1/s fold [AWQ translation, section 3.2]
    # inside the GEMV's x load, against awq_fold_activations as a separate launch before each
    # call (x' in a scratch buffer).  The bytes counted are the sweep's, as above.
    finfo = None
    if not args.skip_fold:
        s_of = {}
        for c in calls:
            if c["K"] not in s_of:
                g_ = torch.Generator(device="cuda").manual_seed(c["K"])
                s_of[c["K"]] = torch.rand(c["K"], device="cuda", generator=g_) * 4.0 + 0.25
        xp = [torch.empty_like(c["x"]) for c in calls]

        def fused_step():
            for c in calls:
                qw, sc, z = c["w"]
                w4.w4a16_gemv_folded(c["x"], s_of[c["K"]], qw, sc, z, out=c["y"], workspace=ws)

        def separate_step():
            for c, xb in zip(calls, xp):
                qw, sc, z = c["w"]
                w4.awq_fold_activations(c["x"], s_of[c["K"]], out=xb)
                w4.w4a16_gemv(xb, qw, sc, z, out=c["y"], workspace=ws)

        ms_f = time_steps(torch, fused_step, 400, 5)
        ms_s = time_steps(torch, separate_step, 400, 5)
        w4.check_device_status()
        finfo = {"fused": {"value": step_bytes / (ms_f * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms_f},
                 "separate": {"value": step_bytes / (ms_s * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms_s},
                 "workload": "the decode sweep on raw activations: w4a16_gemv_folded, against "
                             "awq_fold_activations + w4a16_gemv per call"}
        del xp

    # prefill GEMM on the same shapes (weights of the M = 1 copy; M = 512, 2048, 8192)
    gemm = None
    if not args.skip_gemm:
        flops, t_ms = 0.0, 0.0
        per = []
        # one zeroed workspace for the split-K partial tiles and counters of every call
        wsg = torch.zeros(max(w4.workspace_bytes(M, c["N"], c["K"], csr=False) for c in calls for M in GEMM_MS),
                          dtype=torch.uint8, device="cuda")
        for ci in range(0, len(calls), len(GEMV_MS)):
            c = calls[ci]
            qw, sc, z = c["w"]
            for M in GEMM_MS:
                x = torch.randn(M, c["K"], device="cuda").to(torch.bfloat16)
                y = torch.empty(M, c["N"], dtype=torch.bfloat16, device="cuda")
                ms1, gg = time_graph(torch, lambda: w4.w4a16_gemm(x, qw, sc, z, out=y, workspace=wsg), 20, 3)
                del gg
                f = 2.0 * M * c["N"] * c["K"]
                flops += f
                t_ms += ms1
                per.append({"K": c["K"], "N": c["N"], "M": M, "tflops": round(f / ms1 / 1e9, 1)})
                del x, y
        w4.check_device_status()
        tf = flops / t_ms / 1e9
        peak = pk["bf16_tflops"]
        gemm = {"value": tf, "unit": "TFLOP/s", "workload": "prefill GEMM, Llama-3-8B shapes x M in {512, 2048, "
                "8192}", "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                                      "frac": tf / peak, "peak_kind": f"{pk_kind} bf16 burst"},
                "per_call": per}

    # quantize throughput on the four layers (fp32 W -> packed), algorithmic 4.5195 B/weight
    qinfo = None
    if not args.skip_quant:
        qb, qms = 0.0, 0.0
        for W, act, N, K in quant:
            ms1, gq = time_graph(torch, lambda: w4.awq_quantize_g128(W, act, workloads.ALPHA), 10, 2)
            del gq
            qb += N * K * 4 + workloads.packed_bytes(N, K) + K * 4
            qms += ms1
        qinfo = {"value": qb / qms / 1e6, "unit": "GB/s", "workload": "awq_quantize_g128 on the four Llama-3-8B "
                 "layers (218 M fp32 weights)", "frac_of_hbm": qb / qms / 1e6 / pk["hbm_gbs"]}

    # GPU dense-and-sparse split on the Llama-2-13B layers (0.45% outliers);
    # algorithmic bytes: read W and a, write W_dense and the CSR
    sinfo = None
    if not args.skip_split:
        sb, sms_ = 0.0, 0.0
        per_split = []
        for si, (name, K, N) in enumerate(workloads.DENSE_SPARSE_13B["shapes"]):
            L = workloads.make_layer(workloads.seed_of(3, si), K=K, N=N)
            W = torch.from_numpy(L.W).cuda()
            act = torch.from_numpy(L.act_absmean).cuda()
            nnz = workloads.outlier_nnz(N, K)
            outs = (torch.empty_like(W), torch.empty(N + 1, dtype=torch.int32, device="cuda"),
                    torch.empty(nnz, dtype=torch.int32, device="cuda"), torch.empty(nnz, dtype=torch.int16, device="cuda"))
            wsp = torch.empty(w4.lib().awq_split_outliers_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
            ms1, gs = time_graph(torch, lambda: w4.awq_split_outliers(W, act, workloads.ALPHA, nnz, out=outs,
                                                                      workspace=wsp), 10, 2)
            del gs
            w4.check_device_status()
            b = 8 * N * K + 4 * K + 6 * nnz + 4 * (N + 1)
            sb += b
            sms_ += ms1
            per_split.append({"K": K, "N": N, "nnz": nnz, "ms": round(ms1, 4), "GB/s": round(b / ms1 / 1e6, 1)})
            del W, act, outs, wsp
        sinfo = {"value": sb / sms_ / 1e6, "unit": "GB/s", "workload": "awq_split_outliers on the Llama-2-13B "
                 "layers 5120x5120 and 5120x13824, 0.45% fp16 outliers", "frac_of_hbm": sb / sms_ / 1e6 / pk["hbm_gbs"],
                 "per_layer": per_split}

    # AWQ alpha search: an 11-point grid on the 4096x4096 layer with 128 calibration tokens
    # (quantize + fold + W4A16 GEMM + error per alpha, one fp32 reference product)
    ainfo = None
    if not args.skip_search:
        K, N, Mc = 4096, 4096, 128
        L = workloads.make_layer(workloads.seed_of(1, 1), K=K, N=N)
        W = torch.from_numpy(L.W).cuda()
        act = torch.from_numpy(L.act_absmean).cuda()
        xc = torch.from_numpy(workloads.make_activations(99, Mc, L.mult, alpha=0.0).view(np.int16)).view(
            torch.bfloat16).cuda()
        grid = [i / 10 for i in range(11)]
        wsa = torch.empty(w4.lib().awq_search_alpha_workspace_bytes(Mc, N, K, len(grid)), dtype=torch.uint8,
                          device="cuda")
        w4.awq_search_alpha(W, act, xc, grid, workspace=wsa)
        reps = 5
        t0 = time.perf_counter()
        for _ in range(reps):
            err, best = w4.awq_search_alpha(W, act, xc, grid, workspace=wsa)
        ms_total = (time.perf_counter() - t0) / reps * 1e3
        ainfo = {"value": ms_total, "unit": "ms per search", "ms_per_alpha": ms_total / len(grid),
                 "workload": f"awq_search_alpha, K x N = {K}x{N}, {Mc} calibration tokens, alpha in 0..1 step 0.1",
                 "best_alpha": grid[best], "errors": [round(e, 6) for e in err]}
        del W, act, xc, wsa

    # One group per row (group size = K) [SqueezeLLM article, section 4.1]: quantize the four
    # layers, then the decode sweep's 16 calls on per-row parameters (own weights per call)
    rinfo = None
    if not args.skip_groups:
        rq_b, rq_ms = 0.0, 0.0
        rcalls = []
        for W, act, N, K in quant:
            ms1, gq = time_graph(torch, lambda: w4.awq_quantize(W, act, workloads.ALPHA, K), 5, 2)
            del gq
            rq_b += N * K * 4 + N * K // 2 + N * 2 + N // 8 * 4 + K * 4
            rq_ms += ms1
            qw, sc, z, _ = w4.awq_quantize(W, act, workloads.ALPHA, K)
            for j, M in enumerate(GEMV_MS):
                packed = (qw, sc, z) if j == 0 else (qw.clone(), sc.clone(), z.clone())
                x = torch.randn(M, K, device="cuda").to(torch.bfloat16)
                rcalls.append((x, packed, torch.empty(M, N, dtype=torch.bfloat16, device="cuda"), K,
                               N * K // 2 + N * 2 + N // 8 * 4 + 2 * M * K + 2 * M * N))
        w4.check_device_status()

        def rstep():
            for x, (qw, sc, z), y, K, _ in rcalls:
                w4.w4a16_linear_ex(x, qw, sc, z, out=y, workspace=ws, group_size=K)

        ms_r, gr = time_graph(torch, rstep, 200, 5)
        del gr
        w4.check_device_status()
        rb = sum(c[4] for c in rcalls)
        rinfo = {"gemv": {"value": rb / (ms_r * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms_r,
                          "frac_of_hbm": rb / (ms_r * 1e-3) / 1e9 / pk["hbm_gbs"],
                          "workload": "the decode sweep (4 Llama-3-8B shapes x M in {1, 4, 8, 16}) with one "
                                      "quantization group per row, own weights per call"},
                 "quantize": {"value": rq_b / rq_ms / 1e6, "unit": "GB/s",
                              "workload": "awq_quantize with group size K on the four Llama-3-8B layers"}}
        del rcalls

    # 3-bit codes [SqueezeLLM article, sections 2.1-2.2]: quantize the four layers with eight
    # levels, then the decode sweep's 16 calls through w3a16_gemv (own weights per call)
    tinfo = None
    if not args.skip_3bit:
        tq_b, tq_ms = 0.0, 0.0
        tcalls = []
        for W, act, N, K in quant:
            ms1, gq = time_graph(torch, lambda: w4.awq_quantize3(W, act, workloads.ALPHA, 128), 5, 2)
            del gq
            pb = N * (3 * K // 32) * 4 + (K // 128) * N * 2 + (K // 128) * (N // 8) * 4
            tq_b += N * K * 4 + pb + K * 4
            tq_ms += ms1
            qw, sc, z, _ = w4.awq_quantize3(W, act, workloads.ALPHA, 128)
            for j, M in enumerate(GEMV_MS):
                packed = (qw, sc, z) if j == 0 else (qw.clone(), sc.clone(), z.clone())
                x = torch.randn(M, K, device="cuda").to(torch.bfloat16)
                tcalls.append((x, packed, torch.empty(M, N, dtype=torch.bfloat16, device="cuda"),
                               pb + 2 * M * K + 2 * M * N))
        w4.check_device_status()

        def tstep():
            for x, (qw, sc, z), y, _ in tcalls:
                w4.w3a16_gemv(x, qw, sc, z, out=y, workspace=ws)

        ms_t, gt = time_graph(torch, tstep, 200, 5)
        del gt
        w4.check_device_status()
        tb = sum(c[3] for c in tcalls)
        # NVFP4 weights on the same four layers (quantizer only; W is read twice, once for the
        # tensor amax, but the rate counts it once)
        nq_b, nq_ms = 0.0, 0.0
        for W, act, N, K in quant:
            ms1, gq = time_graph(torch, lambda: w4.awq_quantize_nvfp4(W, act, workloads.ALPHA), 5, 2)
            del gq
            nq_b += N * K * 4 + N * K // 2 + N * K // 16 + 4 + 2 * K * 4
            nq_ms += ms1
        w4.check_device_status()
        tinfo_nv = {"value": nq_b / nq_ms / 1e6, "unit": "GB/s",
                    "workload": "awq_quantize_nvfp4 on the four Llama-3-8B layers"}
        # the decode sweep on NVFP4 weights (own weights per call)
        ncalls = []
        for W, act, N, K in quant:
            qn, sn, gn, _ = w4.awq_quantize_nvfp4(W, act, workloads.ALPHA)
            for j, M in enumerate(GEMV_MS):
                packed = (qn, sn, gn) if j == 0 else (qn.clone(), sn.clone(), gn.clone())
                x = torch.randn(M, K, device="cuda").to(torch.bfloat16)
                ncalls.append((x, packed, torch.empty(M, N, dtype=torch.bfloat16, device="cuda"),
                               N * K // 2 + N * K // 16 + 4 + 2 * M * K + 2 * M * N))
        w4.check_device_status()

        def nstep():
            for x, (qn, sn, gn), y, _ in ncalls:
                w4.w4a16_gemv_nvfp4(x, qn, sn, gn, out=y)

        ms_n, gnv = time_graph(torch, nstep, 200, 5)
        del gnv
        w4.check_device_status()
        nb = sum(c[3] for c in ncalls)
        tinfo_nvg = {"value": nb / (ms_n * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms_n,
                     "frac_of_hbm": nb / (ms_n * 1e-3) / 1e9 / pk["hbm_gbs"],
                     "workload": "the decode sweep (4 Llama-3-8B shapes x M in {1, 4, 8, 16}) on NVFP4 weights "
                                 "(w4a16_gemv_nvfp4), own weights per call"}
        del ncalls
        tinfo = {"gemv": {"value": tb / (ms_t * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms_t,
                          "frac_of_hbm": tb / (ms_t * 1e-3) / 1e9 / pk["hbm_gbs"],
                          "workload": "the decode sweep (4 Llama-3-8B shapes x M in {1, 4, 8, 16}) on 3-bit "
                                      "codes (w3a16_gemv), own weights per call"},
                 "quantize": {"value": tq_b / tq_ms / 1e6, "unit": "GB/s",
                              "workload": "awq_quantize3 (g128) on the four Llama-3-8B layers"},
                 "nvfp4_quantize": tinfo_nv, "nvfp4_gemv": tinfo_nvg}
        del tcalls

    cinfo = None
    if not args.skip_configs:
        cinfo = run_configs(torch, w4, pk, pk_kind, quant)

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.skip_cpu:
        v, secs, outs, desc = oracle_sample(args.cpu_budget)
        cpu = {"value": v, "unit": "GB/s", "cores": omp_threads(), "kind": "oracle", "sample": desc,
               "seconds": round(secs, 2)}
    traffic, traffic_note = profile_traffic()
    per_gpu_gbs = step_bytes / (ms_local * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": DATA,
        "config": sweep_config(world),
        "roofline": {"bound": "hbm", "achieved": per_gpu_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": per_gpu_gbs / pk["hbm_gbs"], "traffic": traffic, "peak_kind": f"{pk_kind} HBM copy",
                     "kernel": "gemv_w4a16_kernel", "bytes_per_launch": step_bytes / len(calls),
                     **({"traffic_note": traffic_note} if traffic_note else {})},
        "cpu_baseline": cpu,
        "e2e": {"value": step_bytes * world / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e},
        "gpu_launches": len(calls) * args.steps,
        "clocks": clocks,
        "gemm": gemm,
        "quantize": qinfo,
        "outlier_split": sinfo,
        "alpha_search": ainfo,
        "per_row_groups": rinfo,
        "three_bit": tinfo,
        "fold_in_gemv": finfo,
        "configs": cinfo,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ the other configs -------

L2_BYTES = 126e6


def _copies(nbytes: float) -> int:
    """Weight copies a timed loop cycles through so that its weights do not stay in L2."""
    return max(1, int(np.ceil(2.5 * L2_BYTES / nbytes)))


def _gpu_layer(torch, seed: int, K: int, N: int):
    """(W fp32 [N][K], act_absmean [K], mult [K]) on the device: the workloads recipe, with W
    drawn on the device (N(0, 0.02^2), seeded) for layers too large to draw on the host."""
    mult, act = workloads.make_act_absmean(seed, K)
    g = torch.Generator(device="cuda").manual_seed(seed)
    W = torch.randn(N, K, device="cuda", generator=g) * 0.02
    return W, torch.from_numpy(act).cuda(), mult


def _x(torch, seed: int, M: int, mult):
    return torch.from_numpy(workloads.make_activations(seed, M, mult).view(np.int16)).view(torch.bfloat16).cuda()


def _rate(nbytes=None, flops=None, ms=None, pk=None, pk_kind=""):
    out = {"us": round(ms * 1e3, 2)}
    if nbytes is not None:
        gbs = nbytes / (ms * 1e-3) / 1e9
        out.update({"GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / pk["hbm_gbs"], 4)})
    if flops is not None:
        tf = flops / (ms * 1e-3) / 1e12
        out.update({"TFLOP/s": round(tf, 1), "frac_of_bf16": round(tf / pk["bf16_tflops"], 4)})
    return out


def _time_calls(torch, calls, reps=20):
    """ms per call: the calls in order inside one graph, replayed reps times."""
    ms = time_steps(torch, lambda: [c() for c in calls], reps, 3)
    return ms / len(calls)


def run_configs(torch, w4, pk, pk_kind, quant8b):
    """Every workload config besides the headline sweep and the prefill GEMM: the single layer
    (config 0), the dense-and-sparse 13B layers (config 3), the 70B layers (config 4) and the
    quantize pass over all eight layers (config 4's C4q).  GEMV timings cycle weight copies
    (> 2x L2); GEMM timings reuse one copy (compute-bound)."""
    out = {}
    # one zeroed workspace, created before any graph capture, for every call below (each call
    # leaves its counters zero): the largest need of configs 0, 3 and 4
    need = [w4.workspace_bytes(1, 4096, 4096)]
    need += [w4.workspace_bytes(M, N, K) for _, K, N in workloads.DENSE_SPARSE_13B["shapes"]
             for M in workloads.DENSE_SPARSE_13B["Ms"]]
    need += [w4.workspace_bytes(M, N, K, csr=False) for _, K, N in workloads.LLAMA2_70B
             for M in workloads.LARGE_LAYERS_70B["Ms"]]
    ws = torch.zeros(max(need), dtype=torch.uint8, device="cuda")
    # ---- config 0: single layer 4096x4096, M = 1: quantize, then the GEMV
    L = workloads.make_layer(workloads.seed_of(0, 0), K=4096, N=4096)
    W, act = torch.from_numpy(L.W).cuda(), torch.from_numpy(L.act_absmean).cuda()
    ms_q = _time_calls(torch, [lambda: w4.awq_quantize_g128(W, act, workloads.ALPHA)], 10)
    qw, sc, z, _ = w4.awq_quantize_g128(W, act, workloads.ALPHA)
    packs = [(qw, sc, z)] + [(qw.clone(), sc.clone(), z.clone()) for _ in range(_copies(workloads.packed_bytes(4096, 4096)) - 1)]
    x = _x(torch, workloads.seed_of(0, 0), 1, L.mult)
    y = torch.empty(1, 4096, dtype=torch.bfloat16, device="cuda")
    ms_g = _time_calls(torch, [lambda p=p: w4.w4a16_gemv(x, *p, out=y, workspace=ws) for p in packs])
    out["config0_single_layer"] = {
        "workload": "4096x4096, M=1: awq_quantize_g128 then w4a16_gemv",
        "quantize": _rate(nbytes=4096 * 4096 * 4 + workloads.packed_bytes(4096, 4096) + 4096 * 4, ms=ms_q, pk=pk),
        "gemv": _rate(nbytes=gemv_bytes(4096, 4096, 1), ms=ms_g, pk=pk)}
    del W, act, packs

    # ---- config 3: dense-and-sparse 13B layers, the CSR term against nnz = 0
    rows = []
    for si, (name, K, N) in enumerate(workloads.DENSE_SPARSE_13B["shapes"]):
        L = workloads.make_layer(workloads.seed_of(3, si), K=K, N=N)
        W, act = torch.from_numpy(L.W).cuda(), torch.from_numpy(L.act_absmean).cuda()
        nnz = workloads.outlier_nnz(N, K)
        Wd, (rp, ci, vals) = w4.awq_split_outliers(W, act, workloads.ALPHA, nnz)
        qw, sc, z, _ = w4.awq_quantize_g128(Wd, act, workloads.ALPHA)
        w4.check_device_status()
        nc = _copies(workloads.packed_bytes(N, K))
        packs = [(qw, sc, z, (rp, ci, vals))] + [(qw.clone(), sc.clone(), z.clone(), (rp.clone(), ci.clone(), vals.clone()))
                                                 for _ in range(nc - 1)]
        csr_bytes = 6 * nnz + 4 * (N + 1)
        for M in workloads.DENSE_SPARSE_13B["Ms"]:
            x = _x(torch, workloads.seed_of(3, si), M, L.mult)
            y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            if M <= 16:
                ms_c = _time_calls(torch, [lambda p=p: w4.w4a16_gemv(x, *p[:3], csr=p[3], out=y, workspace=ws)
                                           for p in packs])
                ms_0 = _time_calls(torch, [lambda p=p: w4.w4a16_gemv(x, *p[:3], out=y, workspace=ws) for p in packs])
                b0 = gemv_bytes(N, K, M)
                rows.append({"K": K, "N": N, "M": M, "nnz": nnz, "kernel": "gemv",
                             "csr": _rate(nbytes=b0 + csr_bytes, ms=ms_c, pk=pk), "no_csr": _rate(nbytes=b0, ms=ms_0, pk=pk),
                             "csr_cost": round(ms_c / ms_0 - 1.0, 4)})
            else:
                p = packs[0]
                ms_c = _time_calls(torch, [lambda: w4.w4a16_gemm(x, *p[:3], csr=p[3], out=y, workspace=ws)])
                ms_0 = _time_calls(torch, [lambda: w4.w4a16_gemm(x, *p[:3], out=y, workspace=ws)])
                f0 = 2.0 * M * N * K
                rows.append({"K": K, "N": N, "M": M, "nnz": nnz, "kernel": "gemm",
                             "csr": _rate(flops=f0 + 2.0 * M * nnz, ms=ms_c, pk=pk), "no_csr": _rate(flops=f0, ms=ms_0, pk=pk),
                             "csr_cost": round(ms_c / ms_0 - 1.0, 4)})
        del W, act, Wd, packs
    out["config3_dense_sparse_13b"] = {"workload": "Llama-2-13B layers with the 0.45% fp16 CSR, M in {1, 16, 1024}",
                                       "per_call": rows}

    # ---- config 4: 70B layers at M = 1, 64, 4096; the quantize pass over all eight layers
    rows, qb, qms = [], 0.0, 0.0
    for W8, act8, N8, K8 in quant8b:
        qms += _time_calls(torch, [lambda: w4.awq_quantize_g128(W8, act8, workloads.ALPHA)], 5)
        qb += N8 * K8 * 4 + workloads.packed_bytes(N8, K8) + K8 * 4
    for si, (name, K, N) in enumerate(workloads.LLAMA2_70B):
        W, act, mult = _gpu_layer(torch, workloads.seed_of(4, si), K, N)
        qms += _time_calls(torch, [lambda: w4.awq_quantize_g128(W, act, workloads.ALPHA)], 5)
        qb += N * K * 4 + workloads.packed_bytes(N, K) + K * 4
        qw, sc, z, _ = w4.awq_quantize_g128(W, act, workloads.ALPHA)
        w4.check_device_status()
        del W
        nb = workloads.packed_bytes(N, K)
        packs = [(qw, sc, z)] + [(qw.clone(), sc.clone(), z.clone()) for _ in range(_copies(nb) - 1)]
        for M in workloads.LARGE_LAYERS_70B["Ms"]:
            x = _x(torch, workloads.seed_of(4, si), M, mult)
            y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            if M <= 16:
                ms = _time_calls(torch, [lambda p=p: w4.w4a16_gemv(x, *p, out=y, workspace=ws) for p in packs])
                rows.append({"K": K, "N": N, "M": M, "kernel": "gemv", **_rate(nbytes=gemv_bytes(N, K, M), ms=ms, pk=pk)})
            else:
                use = packs if M <= 256 else packs[:1]  # the ridge point streams its weights: cycle copies
                ms = _time_calls(torch, [lambda p=p: w4.w4a16_linear(x, *p, out=y, workspace=ws) for p in use], 10)
                r = {"K": K, "N": N, "M": M, "kernel": "gemm"}
                if M <= 256:  # near the ridge: both rooflines
                    r.update(_rate(nbytes=gemv_bytes(N, K, M), flops=2.0 * M * N * K, ms=ms, pk=pk))
                else:
                    r.update(_rate(flops=2.0 * M * N * K, ms=ms, pk=pk))
                rows.append(r)
        del packs, qw, sc, z
    out["config4_large_70b"] = {"workload": "Llama-2-70B layers (W drawn on the device), M in {1, 64, 4096}",
                                "per_call": rows}
    out["c4q_quantize_eight_layers"] = {
        "workload": "awq_quantize_g128 over the four Llama-3-8B and the four Llama-2-70B layers (1.074 G weights)",
        "value": qb / (qms * 1e-3) / 1e9, "unit": "GB/s", "frac_of_hbm": qb / (qms * 1e-3) / 1e9 / pk["hbm_gbs"],
        "algorithmic_bytes": qb, "ms": round(qms, 3)}
    w4.check_device_status()
    return out


GEMV_SOURCE = os.path.join(ROOT, "w4a16_gemm_awq_b200", "csrc", "gemv.cu")
GEMV_PROFILE = os.path.join(ROOT, "profiles", "gemv_w4a16_llama3_8b_decode.md")


def code_digest_text(text: str) -> str:
    """16 hex digits of the sha256 of C/CUDA source text without its comments and whitespace:
    it changes with the code, not with comments or formatting."""
    import hashlib
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return hashlib.sha256(re.sub(r"\s+", "", text).encode()).hexdigest()[:16]


def code_digest(path: str) -> str:
    with open(path) as f:
        return code_digest_text(f.read())


def traffic_from_summary(lines, current_digest: str):
    """(DRAM bytes per GEMV launch, note) from the lines of an ncu summary:
    'traffic_bytes_per_launch: <int>' and 'kernel_code_digest: <hex>'.  The bytes are
    returned only while the digest matches the kernel code as it is now; counters taken on
    other code give (None, why)."""
    fields = {}
    for line in lines:
        if ":" in line and line.split(":", 1)[0] in ("traffic_bytes_per_launch", "kernel_code_digest"):
            k, v = line.split(":", 1)
            fields[k] = v.strip()
    try:
        traffic = int(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None, "no traffic line in the ncu summary"
    if fields.get("kernel_code_digest") != current_digest:
        return None, (f"the ncu counters ({traffic} B per launch) were taken on other kernel code "
                      f"(digest {fields.get('kernel_code_digest')}, now {current_digest})")
    return traffic, None


def profile_traffic():
    """traffic_from_summary for the committed GEMV summary and the current gemv.cu."""
    if not os.path.exists(GEMV_PROFILE):
        return None, "no ncu summary"
    with open(GEMV_PROFILE) as f:
        return traffic_from_summary(f.readlines(), code_digest(GEMV_SOURCE))


def run_case(args):
    """One kernel on one layer, launched eagerly (for ncu): --case gemv|gemm|quantize."""
    import torch

    import w4a16_gemm_awq_b200 as w4
    torch.cuda.set_device(0)
    K, N, M = args.K, args.N, args.M
    L = workloads.make_layer(seed=99, K=K, N=N)
    W = torch.from_numpy(L.W).cuda()
    act = torch.from_numpy(L.act_absmean).cuda()
    qw, sc, z, _ = w4.awq_quantize_g128(W, act, workloads.ALPHA)
    copies = max(1, int(np.ceil(2 * 126e6 / workloads.packed_bytes(N, K)))) if args.case != "quantize" else 1
    packs = [(qw, sc, z)] + [(qw.clone(), sc.clone(), z.clone()) for _ in range(copies - 1)]
    x = torch.from_numpy(workloads.make_activations(99, M, L.mult).view(np.int16)).view(torch.bfloat16).cuda()
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    sched = {"auto": w4.GEMV_AUTO, "stream_k": w4.GEMV_STREAM_K, "cluster": w4.GEMV_CLUSTER}[args.schedule]
    fn = {"gemv": lambda *a, **k: w4.w4a16_gemv_ex(*a, **k, schedule=sched), "gemm": w4.w4a16_gemm}.get(args.case)
    ws = torch.zeros(max(256, w4.workspace_bytes(M, N, K, csr=False)), dtype=torch.uint8, device="cuda")

    def once(i):
        if args.case == "quantize":
            w4.awq_quantize_g128(W, act, workloads.ALPHA, out=(qw, sc, z, _s))
        else:
            a, b, c = packs[i % len(packs)]
            fn(x, a, b, c, out=y, workspace=ws)

    _s = torch.empty(K, device="cuda")
    for i in range(args.warmup):
        once(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        once(i)
    e1.record()
    torch.cuda.synchronize()
    w4.check_device_status()
    ms = e0.elapsed_time(e1) / args.steps
    if args.case == "quantize":
        b = N * K * 4 + workloads.packed_bytes(N, K) + K * 4
        print(json.dumps({"case": "quantize", "K": K, "N": N, "ms": ms, "GB/s": b / ms / 1e6}))
    elif args.case == "gemv":
        print(json.dumps({"case": "gemv", "K": K, "N": N, "M": M, "ms": ms, "copies": copies,
                          "plan": w4.gemv_plan(M, N, K, sched), "GB/s": gemv_bytes(N, K, M) / ms / 1e6}))
    else:
        print(json.dumps({"case": "gemm", "K": K, "N": N, "M": M, "ms": ms, "TFLOP/s": 2.0 * M * N * K / ms / 1e9}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="seconds of oracle work for --impl reference (warm-up and timed steps together)")
    ap.add_argument("--skip-gemm", action="store_true")
    ap.add_argument("--skip-quant", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-split", action="store_true")
    ap.add_argument("--skip-search", action="store_true")
    ap.add_argument("--skip-groups", action="store_true")
    ap.add_argument("--skip-3bit", action="store_true")
    ap.add_argument("--skip-fold", action="store_true")
    ap.add_argument("--skip-configs", action="store_true")
    ap.add_argument("--case", choices=["gemv", "gemm", "quantize"], help="time one kernel on one layer (ncu)")
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--N", type=int, default=28672)
    ap.add_argument("--M", type=int, default=16)
    ap.add_argument("--schedule", default="auto", choices=["auto", "stream_k", "cluster"],
                    help="GEMV schedule of --case gemv")
    args = ap.parse_args()
    if args.case:
        run_case(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        # the CPU oracle needs no process group: rank 0 alone runs, the other ranks exit 0
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup()
    try:
        run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
