#!/usr/bin/env python
"""Benchmark of the W4A16 g128 path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--sections all|none|decode_small_m,prefill,quantize]

Headline workload (one "step"): the decode layer set M = 1, K = 4096,
N in {4096, 11008, 12288}, asymmetric INT4 g128, fp16 activations: three
W4A16 GEMVs through w4a16_gemm.  `value` is the algorithmic bytes of the
step (packed codes + fp32 scales and zeros + X + Y) over the device time of
exactly K steps, in TB/s.  Every step reads a different copy of the packed
weights (enough copies to exceed three times the L2), so each step streams
its weights from HBM.  The other rows of the path are timed in `sections`:
small-M decode (M in {4, 8, 16, 32}, K = 8192, N = 28672, symmetric), the
prefill GEMM (M = 2048, K = 4096, N = 11008, bf16, asymmetric) and the
quantizer over a 7B-shaped stack (32 layers x 4 projections, AWQ factor
folded, asymmetric).

`--impl reference` times the CPU oracle (plain C, OpenMP over rows) on the
same workload instead: the one reference implementation there is.

Multi-GPU (torchrun, one process per GPU): every rank runs the same
workload on its own GPU with its own seeds (independent decode streams, weak
scaling); no data-path collective.  Time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "W4A16 g128 dequant-GEMM TB/s (decode) & TFLOPS (prefill) vs B200 roofline"
GROUP = 128

# DRAM traffic of one decode launch (M=1, K=4096, N=12288: the dominant
# kernel of the step, gemv1_kernel of csrc/w4_gemv1.cu) from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum; profiles/gemv1_kernel_m1_k4096_n12288.md),
# valid only for the kernel source it was taken on: reported as null once
# that source has changed.
DECODE_SRC = "w4_gemv1.cu"
DECODE_TRAFFIC = {"bytes": 28367104, "source_sha256_16": "11fbfdde0bc4a12d"}


# ---------------------------------------------------------------------------- helpers

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d["bf16_tflops_sustained"]), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def dist_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def barrier():
    if torch.distributed.is_initialized():
        torch.distributed.barrier()


def max_over_ranks(x: float) -> float:
    if torch.distributed.is_initialized():
        t = torch.tensor([x], dtype=torch.float64,
                         device="cuda" if torch.cuda.is_available() else "cpu")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())
    return x


def sum_over_ranks(x: float) -> float:
    if torch.distributed.is_initialized():
        t = torch.tensor([x], dtype=torch.float64,
                         device="cuda" if torch.cuda.is_available() else "cpu")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
        return float(t.item())
    return x


def aggregate_rate(bytes_local: float, ms_local: float) -> float:
    """Whole-job throughput in TB/s: the bytes all ranks processed divided by
    the slowest rank's time (every rank calls this, in the same order)."""
    ms = max_over_ranks(ms_local)
    total = sum_over_ranks(bytes_local)
    return total / (ms * 1e-3) / 1e12


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.f = None

    def start(self):
        try:
            self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [l.strip().split(",") for l in self.f.read().splitlines() if l.strip()]
        os.unlink(self.f.name)
        sm, smax, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
                pw.append(float(r[3]))
            except ValueError:
                continue
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        # under load: samples drawing more than the idle floor
        floor = min(pw) + 0.25 * (max(pw) - min(pw)) if pw else 0
        load = [s for s, p in zip(sm, pw) if p >= floor] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm), "power_w_max": max(pw)}


def timed(fn_step, steps: int, warmup: int, stream=None, sampler=None):
    """Runs warmup + exactly `steps` calls of fn_step(i); returns device ms over the steps."""
    for i in range(warmup):
        fn_step(i)
    torch.cuda.synchronize()
    barrier()
    if sampler:
        sampler.start()
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        fn_step(warmup + i)
    e1.record()
    e1.synchronize()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    return e0.elapsed_time(e1), clocks


def timed_block(run_steps, steps: int, warmup: int, sampler=None):
    """Like timed(), with run_steps(n) enqueueing n steps at once."""
    run_steps(warmup)
    torch.cuda.synchronize()
    barrier()
    if sampler:
        sampler.start()
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    run_steps(steps)
    e1.record()
    e1.synchronize()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler else None
    return e0.elapsed_time(e1), clocks


def kernel_ms(graph_fns, reps: int = 20):
    """Average device ms of one replay of each graph (graphs alternate over copies)."""
    for g in graph_fns:
        g.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for r in range(reps):
        for g in graph_fns:
            g.replay()
    e1.record()
    e1.synchronize()
    return e0.elapsed_time(e1) / (reps * len(graph_fns))


def n_copies(set_bytes: int, l2_bytes: int) -> int:
    return max(2, math.ceil(3 * l2_bytes / max(set_bytes, 1)) + 1)


def decode_bytes(M, K, N, sym, xbytes=2):
    G = K // GROUP
    sz = 4 if sym else 8  # fp32 scales (+ fp32 zeros when asymmetric)
    return N * K // 2 + N * G * sz + xbytes * M * K + xbytes * M * N


# ---------------------------------------------------------------------------- our arm

def make_layer(w4, N, K, sym, seed, tensor_id, dtype="f16", std=0.02, w_outlier=0.0):
    W = synth.weights(N, K, std, seed, outlier_frac=w_outlier, dtype=dtype, device="cuda",
                      tensor_id=tensor_id)
    packed, scales, zeros = w4.w4_quantize(W, GROUP, sym=sym)
    del W
    return packed, scales, (None if sym else zeros)


def clone_set(layers):
    return [(p.clone(), s.clone(), None if z is None else z.clone()) for p, s, z in layers]


def run_ours(args, ws_, rank, local):
    import weight_only_int4_pack_b200 as w4
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w4.load()
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20)
    pk = peaks()
    c = synth.DECODE_M1
    K, Ns = c["K"], c["Ns"]
    seed = c["seed"] + 1000 * rank
    launches_per_step = len(Ns)

    # --- headline: decode M = 1 over three layer shapes -------------------------------
    base = [make_layer(w4, N, K, c["sym"], seed, 4 + i, w_outlier=c["w_outlier"])
            for i, N in enumerate(Ns)]
    step_bytes = sum(decode_bytes(1, K, N, c["sym"]) for N in Ns)
    copies = n_copies(sum(p.numel() + s.numel() * 8 for p, s, _ in base), l2)
    sets = [base] + [clone_set(base) for _ in range(copies - 1)]
    X = synth.activations(1, K, seed, salient_frac=c["x_salient"], dtype="f16", device=dev)
    # the three outputs are slices of one buffer, so one copy brings a step's
    # results to the host
    Yall = torch.empty((1, sum(Ns)), dtype=torch.float16, device=dev)
    offs = [sum(Ns[:i]) for i in range(len(Ns))]
    Ys = [Yall[:, o:o + N] for o, N in zip(offs, Ns)]
    wsp = w4.Workspace()
    wsp.get(max(w4.w4a16_workspace_bytes(1, K, N) for N in Ns), dev)

    def step_eager(cidx, xin=X, outs=Ys):
        for (p, s, z), Y in zip(sets[cidx], outs):
            w4.w4a16_gemm(xin, p, s, z, out=Y, workspace=wsp)

    step_eager(0)
    torch.cuda.synchronize()
    block = copies * max(1, 64 // copies)
    # single-step graphs (one per weight copy) and a block graph of B steps
    # cycling through the copies, so that host replay cost stays far below
    # the device time of the steps it launches
    graphs = []
    for ci in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step_eager(ci)
        graphs.append(g)
    gblock = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gblock):
        for i in range(block):
            step_eager(i % copies)
    # per-layer block graphs (B launches of one layer over the copies) for the
    # per-kernel timing
    layer_graphs = []
    for li in range(len(Ns)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(block):
                p, s, z = sets[i % copies][li]
                w4.w4a16_gemm(X, p, s, z, out=Ys[li], workspace=wsp)
        layer_graphs.append(g)

    def run_steps(n):
        for _ in range(n // block):
            gblock.replay()
        for i in range(n % block):
            graphs[i % copies].replay()

    ms_local, clocks = timed_block(run_steps, args.steps, args.warmup, sampler=ClockSampler(local))
    value_tbs = aggregate_rate(step_bytes * args.steps, ms_local)
    ms = max_over_ranks(ms_local)

    per_layer = []
    for li, N in enumerate(Ns):
        kms = kernel_ms([layer_graphs[li]], reps=10) / block
        b = decode_bytes(1, K, N, c["sym"])
        per_layer.append({"N": N, "us": kms * 1e3, "bytes": b, "gbs": b / (kms * 1e-3) / 1e9})
    dom = max(per_layer, key=lambda d: d["us"])
    src = os.path.join(ROOT, "weight_only_int4_pack_b200", "csrc", DECODE_SRC)
    cur = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] if os.path.exists(src) else ""
    traffic = DECODE_TRAFFIC["bytes"] if (cur == DECODE_TRAFFIC["source_sha256_16"]
                                          and dom["N"] == 12288) else None
    roof = {"bound": "hbm", "kernel": "gemv1_kernel (w4a16_gemm, M=1)",
            "achieved": round(dom["gbs"], 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(dom["gbs"] / pk["hbm_gbs"], 4), "traffic": traffic,
            "peak_source": pk["source"], "bytes_per_launch": dom["bytes"],
            "launch_us": round(dom["us"], 3), "per_layer": per_layer}

    # e2e through the public API: pinned host X -> device, three layers, Y -> pinned host
    Xh = X.cpu().pin_memory()
    Yh = torch.empty((1, sum(Ns)), dtype=torch.float16).pin_memory()
    Xd = torch.empty_like(X)

    def step_e2e(i):
        Xd.copy_(Xh, non_blocking=True)
        step_eager(i % copies, Xd)
        Yh.copy_(Yall, non_blocking=True)

    e2e_steps = min(args.steps, 2000)
    e2e_ms_local, _ = timed(step_e2e, e2e_steps, args.warmup)
    e2e_value = aggregate_rate(step_bytes * e2e_steps, e2e_ms_local)
    e2e_ms = max_over_ranks(e2e_ms_local)
    e2e = {"value": round(e2e_value, 4),
           "unit": "TB/s", "h2d_bytes_per_step": int(X.numel() * 2),
           "d2h_bytes_per_step": int(sum(N * 2 for N in Ns)),
           "ms_per_step": round(e2e_ms / e2e_steps, 5)}

    sections = {}
    if rank == 0:
        want = set(args.sections.split(",")) if args.sections not in ("all", "none") else (
            {"decode_small_m", "prefill", "quantize", "awq", "w8a8", "gptq"}
            if args.sections == "all"
            else set())
        del graphs, layer_graphs, gblock
        cpu_ok = args.n_gpus == 1 and not args.no_cpu
        if "decode_small_m" in want:
            sections["decode_small_m"] = section_small_m(w4, dev, l2, pk, cpu_ok)
        if "prefill" in want:
            sections["prefill"] = section_prefill(w4, dev, pk, cpu_ok)
        if "quantize" in want:
            sections["quantize_7b_stack"] = section_quantize(w4, dev, pk, cpu_ok)
        if "awq" in want:
            sections["awq_search"] = section_awq(w4, dev, pk)
        if "w8a8" in want:
            sections["w8a8"] = section_w8a8(w4, dev, pk)
        if "gptq" in want:
            sections["gptq"] = section_gptq(w4, dev, pk)

    cpu = None
    if rank == 0 and args.n_gpus == 1 and not args.no_cpu:
        cpu = cpu_baseline(sets[0], X, step_bytes)

    return dict(value=value_tbs, ms=ms, clocks=clocks, roofline=roof, e2e=e2e,
                sections=sections, cpu=cpu, copies=copies, step_bytes=step_bytes,
                gpu_launches=launches_per_step * args.steps)


def section_small_m(w4, dev, l2, pk, cpu=False):
    c = synth.DECODE_SMALLM
    K, N = c["K"], c["N"]
    base = [make_layer(w4, N, K, c["sym"], c["seed"], 4, std=c["std"])]
    copies = n_copies(base[0][0].numel() + base[0][1].numel() * 4, l2)
    sets = [base] + [clone_set(base) for _ in range(copies - 1)]
    out = []
    wsp = w4.Workspace()
    for M in c["Ms"]:
        X = synth.activations(M, K, c["seed"], salient_frac=c["x_salient"], device=dev)
        Y = torch.empty((M, N), dtype=torch.float16, device=dev)
        ws = wsp.get(w4.w4a16_workspace_bytes(M, K, N), dev)
        w4.w4a16_gemm(X, *sets[0][0], out=Y, workspace=wsp)
        blk = copies * max(1, 32 // copies)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(blk):
                w4.w4a16_gemm(X, *sets[i % copies][0], out=Y, workspace=wsp)
        kms = kernel_ms([g], reps=5) / blk
        b = decode_bytes(M, K, N, True)
        gbs = b / (kms * 1e-3) / 1e9
        out.append({"M": M, "us": round(kms * 1e3, 2), "gbs": round(gbs, 1),
                    "tflops": round(2 * M * N * K / (kms * 1e-3) / 1e12, 2),
                    "frac_hbm": round(gbs / pk["hbm_gbs"], 4)})
        del g, ws
    res = {"workload": f"decode M in {list(c['Ms'])}, K={K}, N={N}, symmetric g128 fp16",
           "bound": "hbm", "peak_gbs": pk["hbm_gbs"], "copies": copies, "per_m": out}
    if cpu:
        p, sc, _ = host_layers([sets[0][0]])[0]
        res["cpu_baseline"] = cpu_small_m(p, sc, K, N, c)
    return res


def section_prefill(w4, dev, pk, cpu=False):
    c = synth.PREFILL
    M, K, N = c["M"], c["K"], c["N"]
    p, s, z = make_layer(w4, N, K, c["sym"], c["seed"], 4, dtype="bf16", std=c["std"])
    X = synth.activations(M, K, c["seed"], salient_frac=c["x_salient"], dtype="bf16", device=dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    try:
        w4.w4a16_gemm(X, p, s, z, out=Y)
    except w4.W4Error as e:
        return {"unavailable": str(e)}
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        w4.w4a16_gemm(X, p, s, z, out=Y)
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    times = []
    for r in range(23):
        flush.zero_()  # evict the weights and X from L2 between launches
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        e1.synchronize()
        if r >= 3:
            times.append(e0.elapsed_time(e1))
    kms = statistics.median(times)
    tf = 2 * M * N * K / (kms * 1e-3) / 1e12
    res = {"workload": f"prefill M={M} K={K} N={N} asymmetric g128 bf16", "bound": "tensor",
           "us": round(kms * 1e3, 1), "tflops": round(tf, 1), "peak_tflops": pk["bf16_tflops"],
           "frac": round(tf / pk["bf16_tflops"], 4), "l2": "flushed between launches"}
    if cpu:
        hp, hs, hz = host_layers([(p, s, z)])[0]
        res["cpu_baseline"] = cpu_prefill(X.cpu(), hp, hs, hz, M, K, N)
    return res


def section_quantize(w4, dev, pk, cpu=False):
    c = synth.STACK_7B
    Xcal = synth.activations(c["calib_M"], 4096, c["seed"], salient_frac=c["x_salient"],
                             tensor_id=2, device=dev)
    cs = synth.awq_col_scale(Xcal)
    layer = []
    for li, (name, out_f, in_f) in enumerate(c["shapes"]):
        layer.append(synth.weights(out_f, in_f, c["std"], c["seed"], outlier_frac=c["w_outlier"],
                                   device=dev, tensor_id=16 + li))
    # 32 layers: distinct buffers holding the same seeded layer (identical values
    # do not change the work; distinct addresses keep every read in HBM)
    Ws = [[w.clone() for w in layer] for _ in range(c["layers"])]
    outs = []
    for lw in Ws:
        lo = []
        for w in lw:
            N, K = w.shape
            lo.append((torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                       torch.empty((N, K // GROUP), dtype=torch.float32, device=dev),
                       torch.empty((N, K // GROUP), dtype=torch.float32, device=dev)))
        outs.append(lo)

    def run():
        for lw, lo in zip(Ws, outs):
            for w, (p, s, z) in zip(lw, lo):
                col = cs if w.shape[1] == 4096 else None
                w4.w4_quantize_into(w, p, s, z, GROUP, sym=False, col_scale=col)

    run()
    torch.cuda.synchronize()
    times = []
    for r in range(5):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    kms = statistics.median(times)
    nw = sum(w.numel() for lw in Ws for w in lw)
    b = nw * (2 + 0.5 + 8 / GROUP)
    gbs = b / (kms * 1e-3) / 1e9
    res = {"workload": "quantize 32 x {qkv 12288x4096, o 4096x4096, gate_up 22016x4096, "
                       "down 4096x11008}, AWQ factor folded (in=4096), asymmetric g128",
           "bound": "hbm", "weights": nw, "ms": round(kms, 3), "gbs": round(gbs, 1),
           "frac": round(gbs / pk["hbm_gbs"], 4), "launches": len(Ws) * 4,
           "bytes_per_weight": 2 + 0.5 + 8 / GROUP}
    if cpu:
        host = [w.cpu() for w in layer]
        del Ws, outs
        res["cpu_baseline"] = cpu_quantize(host, cs.cpu(), c["layers"])
    return res


def awq_inputs(dev):
    c = synth.AWQ_SEARCH
    W = synth.weights(c["N"], c["K"], c["std"], c["seed"], outlier_frac=c["w_outlier"],
                      dtype=c["dtype"], device=dev)
    X = synth.activations(c["Mc"], c["K"], c["seed"], salient_frac=c["x_salient"],
                          dtype=c["dtype"], device=dev)
    alphas = [i / (c["n_alpha"] - 1) for i in range(c["n_alpha"])]
    return c, W, X, alphas


def section_awq(w4, dev, pk):
    """One AWQ alpha search per step: 11 alphas on a 12288 x 4096 layer with
    512 calibration rows.  Ideal time = the bytes every pass must move at the
    measured HBM bandwidth plus the two GEMMs' flops at the measured bf16
    tensor peak (fp16 runs at the same rate)."""
    c, W, X, alphas = awq_inputs(dev)
    Mc, K, N, A = c["Mc"], c["K"], c["N"], len(alphas)
    ws = torch.empty(w4.w4_awq_search_workspace_bytes(Mc, K, N), dtype=torch.uint8, device=dev)
    try:
        w4.w4_awq_search(W, X, alphas, sym=c["sym"], workspace=ws)
    except w4.W4Error as e:
        return {"unavailable": str(e)}
    torch.cuda.synchronize()
    times = []
    for r in range(8):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        w4.w4_awq_search(W, X, alphas, sym=c["sym"], workspace=ws)
        e1.record()
        e1.synchronize()
        if r >= 3:
            times.append(e0.elapsed_time(e1))
    ms = statistics.median(times)
    G = K // GROUP
    once_bytes = 2 * N * K + 2 * Mc * K + 4 * Mc * N          # statistics, Yref write
    per_alpha_bytes = (2 * N * K + N * K / 2 + 8 * N * G      # quantize: read W, write Q
                       + 4 * Mc * K                           # X / s
                       + N * K / 2 + 8 * N * G + 2 * Mc * N   # layer: read Q, write Yq
                       + 6 * Mc * N)                          # error: read Yq, Yref
    flops = 2 * Mc * N * K * (A + 1)
    ideal_ms = ((once_bytes + A * per_alpha_bytes) / (pk["hbm_gbs"] * 1e9)
                + flops / (pk["bf16_tflops"] * 1e12)) * 1e3
    return {"workload": f"AWQ alpha search, {A} alphas, Mc={Mc} calibration rows, "
                        f"layer N={N} K={K}, asymmetric g128 fp16",
            "bound": "hbm+tensor", "ms": round(ms, 3), "ms_per_alpha": round(ms / A, 4),
            "alphas_per_s": round(A / (ms * 1e-3), 1), "ideal_ms": round(ideal_ms, 3),
            "frac": round(ideal_ms / ms, 4),
            "launches_per_search": 4 + 1 + 6 * A + 1}


def w8a8_inputs(w4, dev, fmt):
    c = synth.W8A8
    X = synth.activations(c["M"], c["K"], c["seed"], salient_frac=c["x_salient"],
                          dtype=c["dtype"], device=dev)
    W = synth.weights(c["N"], c["K"], c["std"], c["seed"], dtype=c["dtype"], device=dev)
    s = w4.w8_smooth_scales(X, W, c["alpha"]) if fmt == w4.W8_INT8 else None
    wq, sw = w4.w8_quantize(W, fmt, s, w4.W8_COL_MUL if s is not None else w4.W8_COL_NONE)
    xq, sx = w4.w8_quantize(X, fmt, s, w4.W8_COL_DIV if s is not None else w4.W8_COL_NONE)
    return c, X, s, wq, sw, xq, sx


def section_w8a8(w4, dev, pk):
    """The W8A8 layer at M = 2048, K = 4096, N = 11008 (bf16 in and out):
    SmoothQuant INT8 and FP8 E4M3.  `gemm` times the 8-bit tcgen05 GEMM alone
    on quantized operands, `linear` the layer with the on-the-fly activation
    quantization; L2 is flushed between launches.  The 8-bit dense peak is the
    measured bf16 peak x 2 (the nominal int8 / fp8 : bf16 ratio)."""
    peak8 = 2 * pk["bf16_tflops"]
    out = {"workload": "W8A8 M=2048 K=4096 N=11008 bf16, per-tensor scales "
                       "(INT8 with SmoothQuant alpha=0.5; FP8 E4M3)",
           "bound": "tensor", "peak_tops": peak8,
           "peak_note": "measured bf16 burst x 2 (nominal 8-bit : bf16 ratio)"}
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    for name, fmt in (("int8", w4.W8_INT8), ("fp8_e4m3", w4.W8_E4M3)):
        try:
            c, X, s, wq, sw, xq, sx = w8a8_inputs(w4, dev, fmt)
            M, K, N = c["M"], c["K"], c["N"]
            Y = torch.empty((M, N), dtype=X.dtype, device=dev)
            ws = torch.empty(w4.w8a8_workspace_bytes(M, K), dtype=torch.uint8, device=dev)
            w4.w8_gemm(xq, sx, wq, sw, fmt, X.dtype, out=Y)
            w4.w8a8_linear(X, wq, sw, fmt, s=s, out=Y, workspace=ws)
        except w4.W4Error as e:
            out[name] = {"unavailable": str(e)}
            continue
        torch.cuda.synchronize()
        res = {}
        for part, fn in (("gemm", lambda: w4.w8_gemm(xq, sx, wq, sw, fmt, X.dtype, out=Y)),
                         ("linear", lambda: w4.w8a8_linear(X, wq, sw, fmt, s=s, out=Y,
                                                           workspace=ws))):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            times = []
            for r in range(23):
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                g.replay()
                e1.record()
                e1.synchronize()
                if r >= 3:
                    times.append(e0.elapsed_time(e1))
            kms = statistics.median(times)
            tops = 2 * M * N * K / (kms * 1e-3) / 1e12
            res[part] = {"us": round(kms * 1e3, 1), "tops": round(tops, 1),
                         "frac": round(tops / peak8, 4)}
            del g
        out[name] = res
    return out


def gptq_inputs(dev):
    c = synth.GPTQ
    W = synth.weights(c["N"], c["K"], c["std"], c["seed"], outlier_frac=c["w_outlier"],
                      dtype=c["dtype"], device=dev)
    X = synth.activations(c["Mc"], c["K"], c["seed"], salient_frac=c["x_salient"],
                          dtype=c["dtype"], device=dev)
    return c, W, X


def section_gptq(w4, dev, pk):
    """GPTQ of the qkv projection of a 7B layer (12288 x 4096) with 512
    calibration rows.  `whole` = w4_gptq (Hessian, damping, factorization --
    which synchronizes once -- and the column loop); `column_loop` =
    w4_gptq_quantize alone.  The loop is bound by the fp32 FMAs of its lazy
    updates, N * 128^2 * G (G - 1) / 2 for G = K / 128 blocks, against the
    fp32 FMA peak from the unit counts: 148 SMs x 128 lanes x 2 flops x the
    maximum SM clock (1965 MHz)."""
    c, W, X = gptq_inputs(dev)
    N, K, Mc = c["N"], c["K"], c["Mc"]
    ws = torch.empty(w4.w4_gptq_workspace_bytes(Mc, K, N), dtype=torch.uint8, device=dev)
    try:
        p, s, z, U = w4.w4_gptq(W, X, sym=c["sym"], percdamp=c["percdamp"], return_u=True,
                                workspace=ws)
    except w4.W4Error as e:
        return {"unavailable": str(e)}
    torch.cuda.synchronize()
    res = {}
    for part, fn in (("whole", lambda: w4.w4_gptq(W, X, sym=c["sym"], percdamp=c["percdamp"],
                                                  workspace=ws)),
                     ("column_loop", lambda: w4.w4_gptq_quantize(W, U, sym=c["sym"],
                                                                 workspace=ws))):
        times = []
        for r in range(6):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            if r >= 1:
                times.append(e0.elapsed_time(e1))
        res[part] = {"ms": round(statistics.median(times), 3)}
    G = K // GROUP
    lazy_flops = 2.0 * N * GROUP * GROUP * G * (G - 1) / 2
    peak = 148 * 128 * 2 * 1965e6 / 1e12  # clocks.max.sm of the B200: 1965 MHz
    tf = lazy_flops / (res["column_loop"]["ms"] * 1e-3) / 1e12
    return {"workload": f"GPTQ N={N} K={K}, {Mc} calibration rows, asymmetric g128 fp16, "
                        f"percdamp {c['percdamp']}",
            "bound": "alu", "whole_ms": res["whole"]["ms"],
            "column_loop_ms": res["column_loop"]["ms"],
            "lazy_update_tflops": round(tf, 2), "peak_fp32_tflops": round(peak, 1),
            "frac": round(tf / peak, 4),
            "peak_note": "fp32 FMA lanes x max clock (148 x 128 x 2 x 1965 MHz)"}


# ---------------------------------------------------------------------------- oracle arms

def oracle_step(layer_sets_host, Xbits, dtype):
    import oracle
    for packed, scales, zeros in layer_sets_host:
        K = Xbits.shape[1]
        What = oracle.dequant(packed, scales, zeros, K, GROUP)
        oracle.linear(Xbits, dtype, What)


def host_layers(layers):
    return [(p.cpu().numpy(), s.cpu().numpy(), None if z is None else z.cpu().numpy())
            for p, s, z in layers]


def _cpu_info():
    import oracle
    model = ""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"cores": oracle.threads(), "nproc": os.cpu_count(), "cpu_model": model}


def _one_core(fn):
    """Runs fn() with the oracle on one thread; returns its result."""
    import oracle
    n = oracle.threads()
    oracle.set_threads(1)
    try:
        return fn()
    finally:
        oracle.set_threads(n)


def cpu_small_m(packed, scales, K, N, c):
    """The oracle on the small-M decode layers (K = 8192, N = 28672,
    symmetric): fp64 dequantization + naive fp64 product, every M in full on
    all cores; on one core the M = 4 layer on its first 1024 weight rows,
    scaled to the full N (labelled)."""
    import oracle
    info = _cpu_info()
    out = []
    for M in c["Ms"]:
        X = synth.activations(M, K, c["seed"], salient_frac=c["x_salient"])
        xb = X.contiguous().view(torch.int16).numpy().view(np.uint16)
        t0 = time.perf_counter()
        W2 = oracle.dequant(packed, scales, None, K, GROUP)
        oracle.linear(xb, oracle.F16, W2)
        el = time.perf_counter() - t0
        b = decode_bytes(M, K, N, True)
        out.append({"M": M, "s": round(el, 3), "gbs": round(b / el / 1e9, 3)})
        del W2
    X = synth.activations(4, K, c["seed"], salient_frac=c["x_salient"])
    xb = X.contiguous().view(torch.int16).numpy().view(np.uint16)
    rows = 1024

    def one():
        t0 = time.perf_counter()
        Wr = oracle.dequant(packed[:rows], scales[:rows], None, K, GROUP)
        oracle.linear(xb, oracle.F16, Wr)
        return time.perf_counter() - t0
    el1 = _one_core(one) * N / rows
    return dict(info, kind="oracle", unit="GB/s", value=out[0]["gbs"], per_m=out,
                sample="every M of the layer in full (all cores)",
                one_core={"M": 4, "s_extrapolated": round(el1, 2),
                          "gbs": round(decode_bytes(4, K, N, True) / el1 / 1e9, 4),
                          "sample": f"first {rows} of {N} rows, time scaled by {N}/{rows}"})


def cpu_prefill(X, packed, scales, zeros, M, K, N):
    """The oracle on the prefill layer (M = 2048, K = 4096, N = 11008): fp64
    dequantization and the naive fp64 product on a seeded sample of 256 rows of
    X (all N), all cores; 32 of those rows on one core.  The full-size time is
    the sample's scaled by the rows (labelled as an extrapolation)."""
    import oracle
    info = _cpu_info()
    xb = X.contiguous().view(torch.int16).numpy().view(np.uint16)
    rows = np.sort(np.random.default_rng(4).choice(M, 256, replace=False))
    t0 = time.perf_counter()
    What = oracle.dequant(packed, scales, zeros, K, GROUP)
    oracle.linear(xb, oracle.BF16, What, rows=rows)
    el = time.perf_counter() - t0
    full = el * M / len(rows)
    tf = 2 * M * N * K / full / 1e12

    def one():
        t0 = time.perf_counter()
        oracle.linear(xb, oracle.BF16, What, rows=rows[:32])
        return time.perf_counter() - t0
    el1 = _one_core(one) * M / 32
    return dict(info, kind="oracle", unit="TFLOP/s", value=round(tf, 6),
                sample=f"256 of {M} rows of X, all N; full-size time extrapolated "
                       f"({full:.1f} s) from the sample's {el:.2f} s",
                one_core={"tflops": round(2 * M * N * K / el1 / 1e12, 7),
                          "s_extrapolated": round(el1, 1),
                          "sample": f"32 of {M} rows, scaled by {M}/32"})


def cpu_quantize(layer, cs, nlayers):
    """The oracle quantizer on the 7B stack: the seeded layer (4 projections,
    AWQ factor folded where in = 4096, asymmetric) quantized 32 times -- the
    same work as the GPU section's 32 layers -- on all cores; one projection
    (o, 4096 x 4096) on one core, scaled to the stack (labelled)."""
    import oracle
    info = _cpu_info()
    hb = [w.contiguous().view(torch.int16).numpy().view(np.uint16) for w in layer]
    csn = cs.numpy().astype(np.float32)
    nw = sum(w.size for w in hb) * nlayers
    t0 = time.perf_counter()
    for _ in range(nlayers):
        for w in hb:
            oracle.quantize(w, oracle.F16, GROUP, False, csn if w.shape[1] == 4096 else None)
    el = time.perf_counter() - t0
    b = nw * (2 + 0.5 + 8 / GROUP)
    o = hb[1]

    def one():
        t0 = time.perf_counter()
        oracle.quantize(o, oracle.F16, GROUP, False, csn)
        return time.perf_counter() - t0
    el1 = _one_core(one) * nw / o.size
    return dict(info, kind="oracle", unit="GB/s", value=round(b / el / 1e9, 3), s=round(el, 2),
                sample=f"the whole stack ({nlayers} x the seeded layer, {nw} weights)",
                one_core={"gbs": round(b / el1 / 1e9, 4), "s_extrapolated": round(el1, 1),
                          "sample": "the o projection (4096 x 4096), scaled to the stack"})


def cpu_baseline(layers, X, step_bytes):
    """The oracle, as it stands, on the host cores: full decode steps on all
    cores, and the same step on one core (both reported; the headline fields
    are the all-core run)."""
    import oracle
    hl = host_layers(layers)
    xb = X.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    cores = oracle.threads()

    def timed_steps(limit_s, max_reps):
        reps, t0 = 0, time.perf_counter()
        while True:
            oracle_step(hl, xb, oracle.F16)
            reps += 1
            el = time.perf_counter() - t0
            if el > limit_s or reps >= max_reps:
                return reps, el

    reps, el = timed_steps(10, 5)
    v = step_bytes * reps / el / 1e12
    one = None
    if cores > 1:
        oracle.set_threads(1)
        try:
            r1, e1 = timed_steps(8, 2)
        finally:
            oracle.set_threads(cores)
        one = {"value": step_bytes * r1 / e1 / 1e12, "unit": "TB/s", "cores": 1,
               "sample": f"{r1} full decode step(s) in {e1:.1f} s"}
    return {"value": v, "unit": "TB/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} full decode step(s) (3 layers, M=1, K=4096) in {el:.1f} s: "
                      "fp64 dequantization + naive fp64 GEMV",
            "one_core": one}


def run_reference(args, rank):
    """The oracle, as it stands, on the headline workload (rank 0 only)."""
    import oracle
    c = synth.DECODE_M1
    K, Ns = c["K"], c["Ns"]
    layers = []
    for i, N in enumerate(Ns):
        W = synth.weights(N, K, c["std"], c["seed"], outlier_frac=c["w_outlier"], tensor_id=4 + i)
        wb = W.view(torch.int16).numpy().view(np.uint16)
        p, s, z = oracle.quantize(wb, oracle.F16, GROUP, c["sym"])
        layers.append((p, s, None if c["sym"] else z))
    X = synth.activations(1, K, c["seed"], salient_frac=c["x_salient"])
    xb = X.view(torch.int16).numpy().view(np.uint16)
    step_bytes = sum(decode_bytes(1, K, N, c["sym"]) for N in Ns)
    for _ in range(args.warmup):
        oracle_step(layers, xb, oracle.F16)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(layers, xb, oracle.F16)
    el = time.perf_counter() - t0
    v = step_bytes * args.steps / el / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TB/s", "n_gpus": args.n_gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(),
            "cpu_baseline": {"value": v, "unit": "TB/s", "cores": oracle.threads(), "kind": "oracle",
                             "sample": f"{args.steps} full decode steps (3 layers, M=1, K=4096)"},
            "e2e": {"value": v, "unit": "TB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


def workload_config():
    c = synth.DECODE_M1
    return {"workload": f"decode GEMV M=1, K={c['K']}, N in {list(c['Ns'])}, asymmetric INT4 g128, "
                        "fp16 X, W ~N(0,0.02) with 0.1% entries x10, X ~N(0,1) with 1% channels x20",
            "global_batch": 1, "group": GROUP,
            "l2": "inputs larger than L2: every step reads its own copy of the packed weights",
            "parallelism": "independent replicas per GPU"}


# ---------------------------------------------------------------------------- main

def run_profile_case(args):
    """Runs `--launches` launches of one kernel on its workload, untimed: the
    command the ncu summaries under profiles/ were taken with."""
    import weight_only_int4_pack_b200 as w4
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w4.load()
    case = args.profile
    if case.startswith("decode"):
        if case in ("decode_m1", "decode_m1_n4096"):
            c = synth.DECODE_M1
            M, K, N, sym = 1, c["K"], c["Ns"][0 if case.endswith("4096") else -1], c["sym"]
        else:
            c = synth.DECODE_SMALLM
            M, K, N, sym = int(case.split("_m")[-1]), c["K"], c["N"], c["sym"]
        p, s, z = make_layer(w4, N, K, sym, c["seed"], 4, std=c["std"])
        X = synth.activations(M, K, c["seed"], salient_frac=0.01, device=dev)
        Y = torch.empty((M, N), dtype=torch.float16, device=dev)
        torch.cuda.synchronize()
        for _ in range(args.launches):
            w4.w4a16_gemm(X, p, s, z, out=Y)
    elif case == "prefill":
        c = synth.PREFILL
        p, s, z = make_layer(w4, c["N"], c["K"], c["sym"], c["seed"], 4, dtype="bf16", std=c["std"])
        X = synth.activations(c["M"], c["K"], c["seed"], salient_frac=0.01, dtype="bf16", device=dev)
        torch.cuda.synchronize()
        for _ in range(args.launches):
            w4.w4a16_gemm(X, p, s, z)
    elif case == "quantize":
        # the largest projection of the 7B stack (gate_up, 22016 x 4096), AWQ factor folded
        c = synth.STACK_7B
        W = synth.weights(22016, 4096, c["std"], c["seed"], outlier_frac=c["w_outlier"], device=dev,
                          tensor_id=18)
        cs = synth.awq_col_scale(synth.activations(c["calib_M"], 4096, c["seed"],
                                                   salient_frac=c["x_salient"], tensor_id=2,
                                                   device=dev))
        torch.cuda.synchronize()
        for _ in range(args.launches):
            w4.w4_quantize(W, GROUP, sym=False, col_scale=cs)
    elif case in ("w8a8_int8", "w8a8_fp8"):
        fmt = w4.W8_INT8 if case.endswith("int8") else w4.W8_E4M3
        c, X, s, wq, sw, xq, sx = w8a8_inputs(w4, dev, fmt)
        torch.cuda.synchronize()
        for _ in range(args.launches):
            w4.w8_gemm(xq, sx, wq, sw, fmt, X.dtype)
    elif case == "gptq":
        c, W, X = gptq_inputs(dev)
        torch.cuda.synchronize()
        for _ in range(args.launches):
            w4.w4_gptq(W, X, sym=c["sym"], percdamp=c["percdamp"])
    elif case == "awq":
        c, W, X, alphas = awq_inputs(dev)
        torch.cuda.synchronize()
        for _ in range(args.launches):
            w4.w4_awq_search(W, X, alphas, sym=c["sym"])
    else:
        raise SystemExit(f"unknown --profile case {case}")
    torch.cuda.synchronize()
    print(f"profile case {case}: {args.launches} launches done")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=1000)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--sections", default="all")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--profile", default=None,
                    help="decode_m1 | decode_m4..decode_m32 | prefill | quantize | awq | gptq | w8a8_int8 | "
                         "w8a8_fp8: run "
                         "--launches launches of that kernel (awq: searches) untimed (for ncu)")
    ap.add_argument("--launches", type=int, default=3)
    args = ap.parse_args()
    if args.profile:
        run_profile_case(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    ws_, rank, local = dist_info()
    args.n_gpus = ws_
    if ws_ > 1:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        import datetime
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank)), flush=True)
        if torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()
        return

    r = run_ours(args, ws_, rank, local)
    if rank == 0:
        cpu = r["cpu"]
        line = {
            "metric": METRIC, "value": round(r["value"], 4), "unit": "TB/s", "n_gpus": ws_,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(r["ms"] / args.steps, 6), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": dict(workload_config(), weight_copies=r["copies"],
                           bytes_per_step=r["step_bytes"]),
            "roofline": r["roofline"],
            "cpu_baseline": cpu, "e2e": r["e2e"], "clocks": r["clocks"],
            "gpu_launches": r["gpu_launches"], "sections": r["sections"],
        }
        print(json.dumps(line), flush=True)
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
