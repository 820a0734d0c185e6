#!/usr/bin/env python
"""Benchmark of the rotated low-bit linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the hot path over one batch: the rotated linears of the
bit-width-coverage workload (out 12288, in 4096, group-128 codes at 2, 3 and 8
bits, zero point 2^(b-1), fp16 activations N(0,1), batch 1), each one call of
the C ABI's hq_linear (rotation, unpack, dequantisation and contraction).
Metric: effective weight GB/s = (packed-code + scale bytes) / time, whole job.

Weights are cycled over enough distinct copies that every step reads HBM, not
L2 (inputs larger than L2 between uses of a copy).  Steps are replayed from
CUDA graphs and timed with CUDA events on the launching stream, bracketed by a
barrier and a device synchronisation; the job time is the max over ranks.

Under torchrun every rank runs the same workload on its own GPU with its own
weights (weak scaling); there is no collective on the data path.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_hadamard_rotated_b200 import dist, synth  # noqa: E402

METRIC = "rotated 2/3/4-bit linear: weight GB/s (% HBM peak) at B=1; TFLOP/s at B=64"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
WORKLOAD = "rotated linear M=12288 K=4096, bits 2/3/8, batch 1"
LAYERS = [(12288, 4096, 2), (12288, 4096, 3), (12288, 4096, 8)]
B64 = (28672, 8192, 2, 64)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS,
                bf16_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------- clocks during the timed region
class Clocks:
    Q = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.uuid = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for line in out.splitlines():
            f = [c.strip() for c in line.split(",")]
            if len(f) < 10:
                continue
            if self.uuid and self.uuid.replace("GPU-", "") not in f[1]:
                continue
            rows.append(f)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i] == "Active"})
        loaded = [s for s in sm if s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows),
                "power_w_max": max(float(r[4]) for r in rows
                                   if r[4].replace(".", "").isdigit())}


# ---------------------------------------------------------------- workload
def build_layers(device, copies, seed):
    """copies x layers of packed weights; copy 0 from the seeded host generator,
    the others drawn on the device from a seeded torch generator (same laws)."""
    from bit_hadamard_rotated_b200 import RotatedLinear
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    base = [synth.linear(M, K, b, 1, seed=seed) for (M, K, b) in LAYERS]
    xs = [torch.from_numpy(d["x"]).to(device) for d in base]
    layers = []
    for c in range(copies):
        row = []
        for d in base:
            M, K, b = d["M"], d["K"], d["bits"]
            if c == 0:
                q = torch.from_numpy(d["q"].view(np.int32)).to(device)
                sc = torch.from_numpy(d["scales"]).to(device)
            else:
                q = torch.randint(-2**31, 2**31 - 1, (M, K * b // 32), dtype=torch.int32,
                                  device=device, generator=gen)
                sc = (torch.rand((M, K // 128), device=device, generator=gen) * 0.015 + 0.005
                      ).to(torch.float16)
            s = torch.from_numpy(d["signs"]).to(device)
            row.append(RotatedLinear(q, sc, s, b, d["zero"], max_batch=1))
        layers.append(row)
    return layers, xs


def weight_bytes(M, K, b):
    return M * K * b // 8 + M * (K // 128) * 2


def algorithmic_bytes(M, K, b, N):
    """Bytes the linear must move at least once: codes, scales, signs, x, y."""
    return weight_bytes(M, K, b) + K + N * K * 2 + N * M * 4


def run_ours(a):
    rank, local_rank, world = dist.env_world()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dist.init("nccl")
    import bit_hadamard_rotated_b200 as hq
    from bit_hadamard_rotated_b200 import _lib
    _lib.lib()  # fail loudly if the CUDA library is missing

    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 126 * 2**20)
    step_w = sum(weight_bytes(M, K, b) for (M, K, b) in LAYERS)
    copies = max(2, math.ceil(4 * l2 / step_w))
    layers, xs = build_layers(device, copies, seed=1234 + rank)
    ys = [torch.empty((1, M), dtype=torch.float32, device=device) for (M, K, b) in LAYERS]
    stream = torch.cuda.Stream(device)

    def step(c):
        for li in range(len(LAYERS)):
            layers[c][li](xs[li], out=ys[li])

    with torch.cuda.stream(stream):
        for i in range(max(a.warmup, 3)):
            step(i % copies)
    torch.cuda.synchronize(device)
    for row in layers:
        for lin in row:
            lin.check_status(stream)

    # One graph per weight copy (one step each) and one block graph of `rep` rounds.
    rep = 8
    g1 = []
    n0 = hq.hq_launch_count()
    with torch.cuda.stream(stream):
        for c in range(copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step(c)
            g1.append(g)
        launches_per_step = (hq.hq_launch_count() - n0) // copies
        gb = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gb, stream=stream):
            for _ in range(rep):
                for c in range(copies):
                    step(c)
    block = rep * copies
    for i in range(a.warmup):
        with torch.cuda.stream(stream):
            g1[i % copies].replay()
    torch.cuda.synchronize(device)

    clocks = Clocks(device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier(device)
    torch.cuda.synchronize(device)
    clocks.start()
    time.sleep(0.3)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        done = 0
        while a.steps - done >= block:
            gb.replay()
            done += block
        while done < a.steps:
            g1[done % copies].replay()
            done += 1
        ev1.record(stream)
    torch.cuda.synchronize(device)
    ck = clocks.stop()
    dist.barrier(device)
    ms = ev0.elapsed_time(ev1)
    ms_max = dist.max_over_ranks(ms, device)
    for row in layers:
        for lin in row:
            lin.check_status(stream)

    total_w = step_w * a.steps * world
    value = total_w / (ms_max / 1e3) / 1e9
    pk = peaks()
    alg = sum(algorithmic_bytes(M, K, b, 1) for (M, K, b) in LAYERS)
    achieved = alg / ((ms / a.steps) / 1e3) / 1e9

    # per-bit-width breakdown (each layer's own graph, same protocol)
    per_bits = {}
    for li, (M, K, b) in enumerate(LAYERS):
        gs = []
        with torch.cuda.stream(stream):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(rep):
                    for c in range(copies):
                        layers[c][li](xs[li], out=ys[li])
            gs.append(g)
            reps = max(1, 2000 // block)
            g.replay()
            torch.cuda.synchronize(device)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize(device)
        us = e0.elapsed_time(e1) * 1e3 / (reps * block)
        per_bits[str(b)] = {"us_per_linear": round(us, 3),
                            "weight_gbs": round(weight_bytes(M, K, b) / (us * 1e-6) / 1e9, 1),
                            "frac_hbm": round(weight_bytes(M, K, b) / (us * 1e-6) / 1e9
                                              / pk["hbm"], 4)}

    b64 = measure_b64(device, stream, pk) if a.b64 else None
    configs = measure_configs(device, stream, pk, l2) if a.b64 else None
    e2e = measure_e2e(device, layers, xs, a)
    e2e_ms = dist.max_over_ranks(e2e.pop("ms"), device)
    e2e["value"] = round(step_w * e2e["steps"] * world / (e2e_ms * 1e-3) / 1e9, 3)

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(a.cpu_seconds)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms_max / a.steps, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded; uniform codes, fp16 scales U[0.005,0.02], x ~ N(0,1))",
        "config": {"workload": WORKLOAD, "layers": [f"{M}x{K} b{b}" for (M, K, b) in LAYERS],
                   "batch": 1, "group": 128, "weight_bytes_per_step": step_w,
                   "weight_copies": copies, "l2_bytes": l2,
                   "l2_policy": f"{copies} weight copies cycled; {copies * step_w / 2**20:.0f} MiB "
                                f"> L2 between reuses of a copy",
                   "parallelism": f"replicas x{world} (weak scaling, no data-path collective)"},
        "frac_hbm": round(value / world / pk["hbm"], 4),
        "roofline": {"bound": "hbm",
                     "kernel": "gemv_kernel, rotation fused in (one launch per linear at "
                               "batch 1; aggregate over the step's three linears)",
                     "achieved": round(achieved, 1), "peak": pk["hbm"], "unit": "GB/s",
                     "frac": round(achieved / pk["hbm"], 4), "traffic": None,
                     "peak_source": pk["source"] + " (MEASURED_PEAKS.json hbm_gbs)"},
        "per_bits": per_bits,
        "b64": b64,
        "configs": configs,
        "e2e": e2e,
        "gpu_launches": int(launches_per_step * a.steps),
        "launches_per_step": int(launches_per_step),
        "clocks": ck,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g1, gb
    dist.finish()


def measure_b64(device, stream, pk):
    """TFLOP/s of the large dense MLP linear (28672x8192, 2-bit) at batch 64 (and 16; batch 1
    on the GEMV, weight GB/s)."""
    from bit_hadamard_rotated_b200 import RotatedLinear
    M, K, b, N = B64
    d = synth.linear(M, K, b, N, seed=77, scale_dist="loguniform", outlier_frac=0.01)
    lin = RotatedLinear(torch.from_numpy(d["q"].view(np.int32)).to(device),
                        torch.from_numpy(d["scales"]).to(device),
                        torch.from_numpy(d["signs"]).to(device), b, d["zero"], max_batch=N)
    flush = torch.empty(2 * 126 * 2**20 // 4, dtype=torch.float32, device=device)
    out = {}
    for n in (N, 16, 1):
        x = torch.from_numpy(np.ascontiguousarray(d["x"][:n])).to(device)
        y = torch.empty((n, M), dtype=torch.float32, device=device)
        with torch.cuda.stream(stream):
            for _ in range(3):
                lin(x, out=y)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                lin(x, out=y)
            torch.cuda.synchronize(device)
            times = []
            for _ in range(20):
                flush.zero_()  # L2 flush between timed calls (outside the timed interval)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                torch.cuda.synchronize(device)
                times.append(e0.elapsed_time(e1))
        ms = statistics.median(times)
        tflops = 2.0 * M * K * n / (ms * 1e-3) / 1e12
        out[n] = {"ms": round(ms, 4), "tflops": round(tflops, 2),
                  "frac_bf16_peak": round(tflops / pk["bf16"], 4),
                  "weight_gbs": round(weight_bytes(M, K, b) / (ms * 1e-3) / 1e9, 1),
                  "frac_hbm": round(weight_bytes(M, K, b) / (ms * 1e-3) / 1e9 / pk["hbm"], 4),
                  "launches": lin.launches(n)}
    r = {"workload": f"rotated linear M={M} K={K} b{b} batch {N}", **out[N],
         "timing": "CUDA-graph replay of one call, median of 20, L2 flushed before each",
         "batch16": out[16], "batch1": out[1]}
    return r


def _graph_us(stream, device, calls, reps=5):
    """Median per-call time (us) of one CUDA graph holding `calls` back to back."""
    with torch.cuda.stream(stream):
        for c in calls:
            c()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for c in calls:
                c()
        g.replay()
        torch.cuda.synchronize(device)
        times = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize(device)
            times.append(e0.elapsed_time(e1) * 1e3 / len(calls))
    return statistics.median(times)


def _device_copies(device, M, K, b, n, gen):
    """n weight copies drawn on the device (uniform codes, fp16 scales U[0.005, 0.02])."""
    out = []
    for _ in range(n):
        q = torch.randint(-2**31, 2**31 - 1, (M, K * b // 32), dtype=torch.int32, device=device,
                          generator=gen)
        sc = (torch.rand((M, K // 128), device=device, generator=gen) * 0.015 + 0.005).half()
        out.append((q, sc))
    return out


def measure_configs(device, stream, pk, l2):
    """The other workloads of the metric: the 4096x4096 4-bit linear at batch 1,
    the 256-expert MoE layer (32 tokens, top-8) and the M=K=8192 sweep over
    widths and batches (GEMV up to batch 8, tensor cores from 16).  Weights are
    cycled over enough copies that every call reads HBM; each point is the
    median over 5 replays of a graph of back-to-back calls."""
    from bit_hadamard_rotated_b200 import (RotatedLinear, expert_table, hq_moe_experts,
                                           hq_moe_workspace_size)
    gen = torch.Generator(device=device)
    gen.manual_seed(4242)
    res = {}

    def linear_point(M, K, b, N):
        wb = weight_bytes(M, K, b)
        copies = max(2, math.ceil(4 * l2 / wb))
        signs = torch.from_numpy(synth.linear(16, K, b, 1, seed=5)["signs"]).to(device)
        lins = [RotatedLinear(q, sc, signs, b, 1 << (b - 1), max_batch=N)
                for (q, sc) in _device_copies(device, M, K, b, copies, gen)]
        x = torch.randn((N, K), device=device, generator=gen).half()
        y = torch.empty((N, M), dtype=torch.float32, device=device)
        us = _graph_us(stream, device, [lambda l=l: l(x, out=y) for l in lins])
        gbs = wb / (us * 1e-6) / 1e9
        tf = 2.0 * M * K * N / (us * 1e-6) / 1e12
        r = {"us": round(us, 3), "weight_gbs": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm"], 4),
             "tflops": round(tf, 2), "frac_bf16_peak": round(tf / pk["bf16"], 4),
             "path": "tensor cores" if lins[0].uses_tensor_cores(N) else "GEMV",
             "launches": lins[0].launches(N)}
        del lins
        return r

    res["cfg_4096x4096_b4_n1"] = linear_point(4096, 4096, 4, 1)

    # MoE layer: two copies of the expert weights, alternated, so calls read HBM
    m = synth.moe(seed=1)
    E, H, I, T, k = len(m["experts"]), m["hidden"], m["inter"], m["T"], m["k"]

    def put(v):
        return torch.from_numpy(np.ascontiguousarray(v)).to(device)

    tables = []
    for cpy in range(2):
        ex = []
        for e in m["experts"]:
            d = dict(bits=e["bits"], zero=e["zero"])
            for n in ("q_gate", "q_up", "q_down"):
                d[n] = put(e[n].view(np.int32)) if cpy == 0 else torch.randint(
                    -2**31, 2**31 - 1, e[n].shape, dtype=torch.int32, device=device, generator=gen)
            for n in ("s_gate", "s_up", "s_down"):
                d[n] = put(e[n])
            ex.append(d)
        tables.append((expert_table(ex, device), ex))
    x, ids, w = put(m["x"]), put(m["topk_ids"].astype(np.int32)), put(m["topk_w"].astype(np.float32))
    s_in, s_mid = put(m["s_in"]), put(m["s_mid"])
    ws = torch.zeros(hq_moe_workspace_size(E, H, I, T, k), dtype=torch.uint8, device=device)
    out = torch.empty((T, H), dtype=torch.float32, device=device)
    us = _graph_us(stream, device, [lambda t=t: hq_moe_experts(t[0], E, H, I, x, ids, w, s_in, s_mid,
                                                               out=out, workspace=ws)
                                    for t in tables] * 4)
    tb = synth.touched_weight_bytes(m)
    res["moe_256x2048x512_t32_top8"] = {
        "us": round(us, 2), "tokens_per_s": round(T / (us * 1e-6), 1),
        "touched_weight_bytes": tb, "weight_gbs": round(tb / (us * 1e-6) / 1e9, 1),
        "frac_hbm": round(tb / (us * 1e-6) / 1e9 / pk["hbm"], 4), "launches": 5}
    del tables

    sweep = {}
    for b in (2, 3, 4, 8):
        for N in (1, 2, 4, 8, 16, 32, 64, 128):
            sweep[f"b{b}_n{N}"] = linear_point(8192, 8192, b, N)
    res["sweep_8192x8192"] = sweep
    return res


class _Rt:
    """Async copies and event waits on raw stream handles through the CUDA
    runtime that PyTorch loaded (a few hundred ns of host time each, against
    several us for the tensor-level calls), or the tensor-level calls when that
    library cannot be found."""

    def __init__(self):
        import ctypes
        import glob
        self.rt = None
        here = os.path.dirname(torch.__file__)
        for c in glob.glob(os.path.join(here, "..", "nvidia", "cuda_runtime", "lib", "libcudart.so*")) + \
                ["libcudart.so.12", "libcudart.so"]:
            try:
                self.rt = ctypes.CDLL(c)
                break
            except OSError:
                continue
        if self.rt is not None:
            vp, sz = ctypes.c_void_p, ctypes.c_size_t
            self.rt.cudaMemcpyAsync.argtypes = [vp, vp, sz, ctypes.c_int, vp]
            self.rt.cudaEventRecord.argtypes = [vp, vp]
            self.rt.cudaStreamWaitEvent.argtypes = [vp, vp, ctypes.c_uint]
        self.ctypes = ctypes

    def event(self):
        ev = torch.cuda.Event()
        if self.rt is not None:
            ev.record()  # creates the event; its handle is then fixed
            torch.cuda.synchronize()
        return ev

    def copy(self, dst, src, stream, kind):
        if self.rt is None:
            with torch.cuda.stream(stream):
                dst.copy_(src, non_blocking=True)
            return
        n = src.numel() * src.element_size()
        if self.rt.cudaMemcpyAsync(dst.data_ptr(), src.data_ptr(), n, kind, stream.cuda_stream):
            raise RuntimeError("cudaMemcpyAsync failed")

    def record(self, ev, stream):
        if self.rt is None:
            ev.record(stream)
        elif self.rt.cudaEventRecord(ev.cuda_event, stream.cuda_stream):
            raise RuntimeError("cudaEventRecord failed")

    def wait(self, stream, ev):
        if self.rt is None:
            stream.wait_event(ev)
        elif self.rt.cudaStreamWaitEvent(stream.cuda_stream, ev.cuda_event, 0):
            raise RuntimeError("cudaStreamWaitEvent failed")


def measure_e2e(device, layers, xs, a):
    """Same metric through the public Python API with host buffers: every step
    copies the step's activations (the three layers' inputs, one pinned host
    buffer) to the device in one copy, runs the layers (RotatedLinear launchers
    prepared once on their buffers, each call one hq_linear call), and reads
    their outputs back to a pinned host buffer in one copy, all inside the timed
    region.  The copies run on two copy streams, double-buffered, so step
    i + 1's upload and step i's download overlap the layers of the neighbouring
    steps (a serving loop's pipelining); every step moves its own bytes both
    ways."""
    copies = len(layers)
    xsz = [x.numel() for x in xs]
    ysz = [M for (M, K, b) in LAYERS]
    xh = torch.cat([x.reshape(-1).cpu() for x in xs]).pin_memory()
    NB = 2  # buffer sets in flight
    xd = [torch.empty_like(xh, device=device) for _ in range(NB)]
    yd = [torch.empty(sum(ysz), dtype=torch.float32, device=device) for _ in range(NB)]
    yh = [torch.empty(sum(ysz), dtype=torch.float32).pin_memory() for _ in range(NB)]
    comp = torch.cuda.current_stream(device)
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    launch = []  # [copy][buffer set] -> the three layers' launchers
    for c in range(copies):
        per_b = []
        for b in range(NB):
            fns, ox, oy = [], 0, 0
            for li, (M, _K, _b) in enumerate(LAYERS):
                fns.append(layers[c][li].prepare(xd[b][ox:ox + xsz[li]].view(1, -1),
                                                 yd[b][oy:oy + M].view(1, -1), stream=comp))
                ox += xsz[li]
                oy += M
            per_b.append(fns)
        launch.append(per_b)
    steps = min(a.steps, 2000)
    rt = _Rt()
    x_in, y_out, y_read = ([rt.event() for _ in range(NB)] for _ in range(3))
    H2D, D2H = 1, 2  # cudaMemcpyKind

    def upload(i):
        b = i % NB
        if i >= NB:
            rt.wait(up, y_out[b])  # the layers of step i - NB have read xd[b]
        rt.copy(xd[b], xh, up, H2D)
        rt.record(x_in[b], up)

    def step(i):
        b = i % NB
        rt.wait(comp, x_in[b])
        if i >= NB:
            rt.wait(comp, y_read[b])  # step i - NB's download has read yd[b]
        for fn in launch[i % copies][b]:
            fn()
        rt.record(y_out[b], comp)
        rt.wait(down, y_out[b])
        rt.copy(yh[b], yd[b], down, D2H)
        rt.record(y_read[b], down)

    def run(n, start=None):
        if start is not None:
            rt.wait(up, start)
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            step(i)
        rt.wait(comp, y_read[(n - 1) % NB])  # the last download is inside the region

    run(3)
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    run(steps, start=e0)
    e1.record(comp)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1)
    return {"ms": ms, "value": None, "unit": "GB/s", "steps": steps,
            "h2d_bytes_per_step": int(xh.numel() * 2), "d2h_bytes_per_step": int(yh[0].numel() * 4),
            "api": "RotatedLinear.prepare launchers -> hq_linear (C ABI), eager, one call per "
                   "layer per step; one H2D and one D2H copy per step on two copy streams, "
                   "double-buffered against the layers" +
                   ("" if rt.rt is not None else " (tensor-level copies)")}


# ---------------------------------------------------------------- CPU oracle baseline
def cpu_baseline(seconds: float):
    """The fp64 oracle as it stands, on this host's cores (rows split across
    threads), over a bounded sample: whole passes over the workload's three
    layers at batch 1, repeated until about `seconds` of wall time."""
    import oracle
    cores = os.cpu_count() or 1
    ds = [synth.linear(M, K, b, 1, seed=99) for (M, K, b) in LAYERS]
    passes = 0
    t0 = time.perf_counter()
    while True:
        for d in ds:
            oracle.linear(d["bits"], d["M"], d["K"], d["zero"], d["q"], d["scales"], d["signs"],
                          d["x"], threads=cores)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    wb = passes * sum(weight_bytes(M, K, b) for (M, K, b) in LAYERS)
    return {"value": round(wb / dt / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{passes} full passes over the 3 layers (12288x4096 at b2, b3, b8), "
                      f"batch 1, {dt:.1f} s wall on {cores} threads"}


def run_reference(a):
    rank, _, world = dist.env_world()
    if rank != 0:
        return
    import oracle
    cores = os.cpu_count() or 1
    ds = [synth.linear(M, K, b, 1, seed=99) for (M, K, b) in LAYERS]
    rows = a.ref_rows
    for _ in range(max(a.warmup, 0)):
        for d in ds:
            oracle.linear(d["bits"], d["M"], d["K"], d["zero"], d["q"], d["scales"], d["signs"],
                          d["x"], 0, rows, threads=cores)
    t0 = time.perf_counter()
    for _ in range(a.steps):
        for d in ds:
            oracle.linear(d["bits"], d["M"], d["K"], d["zero"], d["q"], d["scales"], d["signs"],
                          d["x"], 0, rows, threads=cores)
    dt = time.perf_counter() - t0
    wb = a.steps * sum(rows * (K * b // 8 + (K // 128) * 2) for (M, K, b) in LAYERS)
    v = wb / dt / 1e9
    sample = f"each step: first {rows} of 12288 rows of each layer (b2, b3, b8), batch 1"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(v, 5), "unit": "GB/s",
        "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": round(dt * 1e3 / a.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": sample},
        "cpu_baseline": {"value": round(v, 5), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(v, 5), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-b64", dest="b64", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-rows", type=int, default=256)
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
