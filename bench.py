#!/usr/bin/env python
"""Benchmark of the rotated low-bit linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the hot path over one batch: the large dense MLP linear
(out 28672, in 8192, 2-bit group-128 codes, zero point 2, fp16 scales
log-uniform in [0.003, 0.03], fp16 activations N(0,1) with 1 % outlier
channels x20, random signs) at batch 1, one call of the C ABI's hq_linear
(rotation, unpack, dequantisation and contraction in one kernel).
Metric: effective weight GB/s = (packed-code + scale bytes) / time, whole job;
the same weights at batch 16 and 64 are reported in TFLOP/s beside it.

Weights are cycled over enough distinct copies that every call reads HBM, not
L2 (inputs larger than L2 between uses of a copy).  The K timed calls are one
CUDA graph (a few, past 2048 calls), so the time per call does not depend on K;
CUDA events on the launching stream, a barrier and a device synchronisation
on both sides; the job time is the max over ranks.

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
HEAD = (28672, 8192, 2)  # M, K, bits of the dense MLP linear
WORKLOAD = "rotated dense MLP linear M=28672 K=8192, 2-bit group-128, batch 1"
GRAPH_CALLS = 2048       # calls per captured graph at most
# Files the GEMV kernel is built from: the ncu traffic figure in the profile
# summary is reported only while their hash matches the one it was taken at.
GEMV_SOURCES = ["gemv.cu", "gemv_frag.cuh", "fwht.cuh", "hq_common.cuh", "hq_internal.h", "hq_io.cuh",
                "hq_launch.cuh", "hq_layout.cuh"]
TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "gemv_kernel_28672x8192_b2_n1.md")


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
def weight_bytes(M, K, b):
    return M * K * b // 8 + M * (K // 128) * 2


def algorithmic_bytes(M, K, b, N):
    """Bytes the linear must move at least once: codes, scales, signs, x, y."""
    return weight_bytes(M, K, b) + K + N * K * 2 + N * M * 4


def gemv_source_hash():
    import hashlib
    h = hashlib.sha256()
    for f in GEMV_SOURCES:
        with open(os.path.join(ROOT, "bit_hadamard_rotated_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch of the batch-1 GEMV from the committed ncu summary,
    or None if the summary is missing or the kernel's sources changed since."""
    try:
        txt = open(TRAFFIC_PROFILE).read()
    except OSError:
        return None, "no profile summary"
    import re
    t = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", txt)
    s = re.search(r"source_sha16:\s*([0-9a-f]{16})", txt)
    if not t or not s:
        return None, "profile summary without traffic"
    if s.group(1) != gemv_source_hash():
        return None, "kernel changed since the profile"
    return int(t.group(1)), os.path.relpath(TRAFFIC_PROFILE, ROOT)


def head_copies(device, copies, seed):
    """copies of the dense MLP linear's packed weights: copy 0 from the seeded
    host generator, the others drawn on the device from a seeded torch
    generator with the same laws (uniform code bits, log-uniform fp16 scales)."""
    from bit_hadamard_rotated_b200 import RotatedLinear
    M, K, b = HEAD
    d = synth.linear(M, K, b, 64, seed=seed, scale_dist="loguniform", outlier_frac=0.01)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    signs = torch.from_numpy(d["signs"]).to(device)
    lins = []
    for c in range(copies):
        if c == 0:
            q = torch.from_numpy(d["q"].view(np.int32)).to(device)
            sc = torch.from_numpy(d["scales"]).to(device)
        else:
            q = torch.randint(-2**31, 2**31 - 1, (M, K * b // 32), dtype=torch.int32, device=device,
                              generator=gen)
            u = torch.rand((M, K // 128), device=device, generator=gen, dtype=torch.float64)
            sc = torch.exp(math.log(0.003) + u * (math.log(0.03) - math.log(0.003))).half()
        lins.append(RotatedLinear(q, sc, signs, b, d["zero"], max_batch=64))
    return lins, torch.from_numpy(d["x"]).to(device)


def capture(stream, calls):
    """One CUDA graph of the given calls back to back."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in calls:
            c()
    return g


def timed_calls(stream, device, lins, x, y, steps, warmup, copies):
    """Time `steps` calls (call i on weight copy i mod copies) replayed from
    graphs of up to GRAPH_CALLS calls (a multiple of `copies`, so the cycle
    continues across replays); returns (ms, graphs) after W warm-up calls."""
    def calls(n, start=0):
        return [lambda l=lins[(start + i) % copies]: l(x, out=y) for i in range(n)]

    with torch.cuda.stream(stream):
        for c in calls(max(warmup, 3)):
            c()
        if steps <= GRAPH_CALLS:
            plan = [(capture(stream, calls(steps)), 1)]
        else:
            per = max(copies, GRAPH_CALLS // copies * copies)
            plan = [(capture(stream, calls(per)), steps // per)]
            if steps % per:
                plan.append((capture(stream, calls(steps % per)), 1))
        # warm-up replays of the captured graphs (uploads them, warms the clocks)
        for g, _ in plan:
            g.replay()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier(device)
    torch.cuda.synchronize(device)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for g, reps in plan:
            for _ in range(reps):
                g.replay()
        e1.record(stream)
    torch.cuda.synchronize(device)
    dist.barrier(device)
    return e0.elapsed_time(e1), plan


def run_ours(a):
    rank, local_rank, world = dist.env_world()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dist.init("nccl")
    import bit_hadamard_rotated_b200 as hq
    from bit_hadamard_rotated_b200 import _lib
    _lib.lib()  # fail loudly if the CUDA library is missing

    M, K, b = HEAD
    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 126 * 2**20)
    wb = weight_bytes(M, K, b)
    copies = max(2, math.ceil(4 * l2 / wb))
    lins, x64 = head_copies(device, copies, seed=77 + rank)
    x1 = x64[:1].contiguous()
    y1 = torch.empty((1, M), dtype=torch.float32, device=device)
    stream = torch.cuda.Stream(device)
    pk = peaks()

    n0 = hq.hq_launch_count()
    with torch.cuda.stream(stream):
        lins[0](x1, out=y1)
    torch.cuda.synchronize(device)
    launches_per_step = hq.hq_launch_count() - n0

    clocks = Clocks(device)
    clocks.start()
    time.sleep(0.3)
    ms, plan = timed_calls(stream, device, lins, x1, y1, a.steps, a.warmup, copies)
    ck = clocks.stop()
    del plan
    ms_max = dist.max_over_ranks(ms, device)
    for lin in lins:
        lin.check_status(stream)

    value = wb * a.steps * world / (ms_max / 1e3) / 1e9
    alg = algorithmic_bytes(M, K, b, 1)
    achieved = alg / ((ms / a.steps) / 1e3) / 1e9
    traffic, traffic_src = profiled_traffic()

    # the same weights at batch 16 and 64 (tensor cores), back-to-back calls
    big = {}
    for n in (16, 64):
        xn = x64[:n].contiguous()
        yn = torch.empty((n, M), dtype=torch.float32, device=device)
        reps = max(copies, 4 * copies)
        ms_n, plan = timed_calls(stream, device, lins, xn, yn, reps, 3, copies)
        del plan
        ms_n = dist.max_over_ranks(ms_n, device)
        us = ms_n * 1e3 / reps
        tf = 2.0 * M * K * n / (us * 1e-6) / 1e12
        big[f"b{n}"] = {"us_per_call": round(us, 3), "tflops": round(tf, 2),
                        "frac_bf16_peak": round(tf / pk["bf16"], 4),
                        "weight_gbs": round(wb / (us * 1e-6) / 1e9, 1),
                        "frac_hbm": round(wb / (us * 1e-6) / 1e9 / pk["hbm"], 4),
                        "path": lins[0].path(n),
                        "launches_per_call": lins[0].launches(n),
                        "timing": f"{reps} back-to-back calls in one graph, {copies} weight "
                                  f"copies cycled"}

    configs = measure_configs(device, stream, pk, l2) if a.configs else None
    e2e = measure_e2e(device, lins, x1, a, copies)
    e2e_ms = dist.max_over_ranks(e2e.pop("ms"), device)
    e2e["value"] = round(wb * e2e["steps"] * world / (e2e_ms * 1e-3) / 1e9, 3)

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(a.cpu_seconds)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms_max / a.steps, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded; uniform 2-bit codes, fp16 scales log-uniform [0.003,0.03], "
                "x ~ N(0,1) fp16 with 1% outlier channels x20)",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "bits": b, "batch": 1, "group": 128,
                   "zero": 2, "weight_bytes_per_step": wb, "weight_copies": copies,
                   "l2_bytes": l2,
                   "l2_policy": f"{copies} weight copies cycled; {copies * wb / 2**20:.0f} MiB "
                                f"> L2 between reuses of a copy",
                   "timing": "the K calls replayed from one CUDA graph (graphs of up to "
                             f"{GRAPH_CALLS} calls past that)",
                   "parallelism": f"replicas x{world} (weak scaling, no data-path collective)"},
        "frac_hbm": round(value / world / pk["hbm"], 4),
        "tflops_b64": big["b64"]["tflops"],
        "frac_bf16_b64": big["b64"]["frac_bf16_peak"],
        "b16": big["b16"], "b64": big["b64"],
        "roofline": {"bound": "hbm",
                     "kernel": "gemv_kernel<2, 13, 1> (rotation fused in; the step's only kernel)",
                     "achieved": round(achieved, 1), "peak": pk["hbm"], "unit": "GB/s",
                     "frac": round(achieved / pk["hbm"], 4), "traffic": traffic,
                     "algorithmic_bytes_per_launch": alg,
                     "traffic_source": traffic_src,
                     "peak_source": pk["source"] + " (MEASURED_PEAKS.json hbm_gbs, copy)"},
        "configs": configs,
        "e2e": e2e,
        "gpu_launches": int(launches_per_step * a.steps),
        "launches_per_step": int(launches_per_step),
        "clocks": ck,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.finish()


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
    """The other workloads: the 4096x4096 4-bit linear at batch 1, the bit-width
    coverage linears (12288x4096 at 2, 3 and 8 bits, batch 1-8), the 256-expert
    MoE layer (32 tokens, top-8) and the M=K=8192 sweep over widths and batches.
    Weights are cycled over enough copies that every call reads HBM; each point
    is the median over 5 replays of a graph of back-to-back calls."""
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
             "path": lins[0].path(N),
             "launches": lins[0].launches(N)}
        del lins
        return r

    res["cfg_4096x4096_b4_n1"] = linear_point(4096, 4096, 4, 1)
    res["cfg_12288x4096"] = {f"b{b}_n{n}": linear_point(12288, 4096, b, n)
                             for b in (2, 3, 8) for n in (1, 2, 4, 8)}

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

    res["readout_157184x2048_top8"] = measure_readout(device, stream, pk, gen)
    res["kv_attend_32768x4x128_q32"] = measure_kv(device, stream, pk, l2)

    sweep = {}
    for b in (2, 3, 4, 8):
        for N in (1, 2, 4, 8, 16, 32, 64, 128):
            sweep[f"b{b}_n{N}"] = linear_point(8192, 8192, b, N)
    res["sweep_8192x8192"] = sweep
    return res


def measure_readout(device, stream, pk, gen):
    """The screened top-8 readout over the 157,184 x 2048 8-bit lm_head kept
    as nibble planes, batch 1, against the plain 8-bit linear over the same
    codes; two copies of the planes alternated (16-bit codes, 2 x 322 MB > L2)."""
    from bit_hadamard_rotated_b200 import RotatedLinear, ScreenedReadout, hq_split_nibbles
    V, K = 157184, 2048
    signs = torch.from_numpy(synth.signs(np.random.default_rng(1), K)).to(device)
    ros, lins = [], []
    for _ in range(2):
        q8 = torch.randint(-2**31, 2**31 - 1, (V, K // 4), dtype=torch.int32, device=device, generator=gen)
        sc = (torch.rand((V, K // 128), device=device, generator=gen) * 0.015 + 0.005).half()
        hi, lo = hq_split_nibbles(q8, K)
        ros.append(ScreenedReadout(hi, lo, sc, signs, 128, max_batch=1))
        lins.append(RotatedLinear(q8, sc, signs, 8, 128, max_batch=1))
    x = torch.randn((1, K), device=device, generator=gen).half()
    y = torch.empty((1, V), dtype=torch.float32, device=device)
    us_ro = _graph_us(stream, device, [lambda r=r: r.topk(x, 8, stream=stream) for r in ros] * 4)
    us_lin = _graph_us(stream, device, [lambda l=l: l(x, out=y) for l in lins] * 4)
    hi_bytes = V * K // 2 + V * (K // 128) * 2
    return {"us_screened_top8": round(us_ro, 2), "us_plain_8bit_linear": round(us_lin, 2),
            "high_plane_gbs": round(hi_bytes / (us_ro * 1e-6) / 1e9, 1),
            "frac_hbm_high_plane": round(hi_bytes / (us_ro * 1e-6) / 1e9 / pk["hbm"], 4),
            "launches": 5, "batch": 1}


def measure_kv(device, stream, pk, l2):
    """Attention of a 32-token block (16 heads, 4 kv heads of 128 channels)
    over a 32K-token int4 cache, and its quantisation of the block (append);
    enough caches cycled that every call reads HBM.  FLOPs: 4 R T d per kv
    head (scores and P.V, R = 128 query rows); bytes: the cache's codes,
    scales and minima."""
    from bit_hadamard_rotated_b200 import KVCache
    T, n_kv, d, n_q, n_heads = 32768, 4, 128, 32, 16
    cache_bytes = n_kv * T * d + n_kv * (T // 32) * d * 4 + n_kv * T * 4
    copies = max(2, math.ceil(3 * l2 / cache_bytes))
    caches = []
    for _ in range(copies):
        c = KVCache(n_kv, d, T, device)
        c.append(torch.randn((T, n_kv, d), device=device).half(), torch.randn((T, n_kv, d), device=device).half(), 0)
        caches.append(c)
    q = torch.randn((n_q, n_heads, d), device=device).half()
    out = torch.empty((n_q, n_heads, d), dtype=torch.float32, device=device)
    ws = torch.zeros(caches[0].workspace_size(T, n_q, n_heads), dtype=torch.uint8, device=device)
    us = _graph_us(stream, device, [lambda c=c: c.attend(q, T, out=out, workspace=ws, stream=stream)
                                    for c in caches])
    kb, vb = torch.randn((32, n_kv, d), device=device).half(), torch.randn((32, n_kv, d), device=device).half()
    us_app = _graph_us(stream, device, [lambda c=c: c.append(kb, vb, T - 32, stream=stream) for c in caches])
    flops = 4.0 * (n_q * n_heads // n_kv) * T * d * n_kv
    del caches
    return {"us": round(us, 2), "tflops": round(flops / (us * 1e-6) / 1e12, 2),
            "frac_bf16_peak": round(flops / (us * 1e-6) / 1e12 / pk["bf16"], 4),
            "cache_gbs": round(cache_bytes / (us * 1e-6) / 1e9, 1), "us_append_32_tokens": round(us_app, 2),
            "launches": 2}


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


def measure_e2e(device, lins, x1, a, copies):
    """Same metric through the public Python API with host buffers: every step
    copies the step's activations from a pinned host buffer to the device, runs
    the layer (a RotatedLinear launcher prepared once on its buffers: one
    hq_linear call), and reads its output back to a pinned host buffer, all
    inside the timed region.  The copies run on two copy streams,
    double-buffered, so step i + 1's upload and step i's download overlap the
    neighbouring steps' layer calls (a serving loop's pipelining); every step
    moves its own bytes both ways."""
    M = lins[0].M
    xh = x1.reshape(-1).cpu().pin_memory()
    NB = 2  # buffer sets in flight
    xd = [torch.empty_like(xh, device=device) for _ in range(NB)]
    yd = [torch.empty(M, dtype=torch.float32, device=device) for _ in range(NB)]
    yh = [torch.empty(M, dtype=torch.float32).pin_memory() for _ in range(NB)]
    comp = torch.cuda.current_stream(device)
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    launch = []  # [copy][buffer set] -> the layer's launcher
    for c in range(copies):
        launch.append([[lins[c].prepare(xd[b].view(1, -1), yd[b].view(1, -1), stream=comp)]
                       for b in range(NB)])
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
            "api": "RotatedLinear.prepare launcher -> hq_linear (C ABI), eager, one call per "
                   "step; one H2D and one D2H copy per step on two copy streams, "
                   "double-buffered against the layer calls" +
                   ("" if rt.rt is not None else " (tensor-level copies)")}


# ---------------------------------------------------------------- CPU oracle baseline
def cpu_baseline(seconds: float):
    """The fp64 oracle as it stands, on this host's cores (rows split across
    threads), over a bounded sample: whole passes over the workload's linear at
    batch 1, repeated until about `seconds` of wall time."""
    import oracle
    cores = os.cpu_count() or 1
    M, K, b = HEAD
    d = synth.linear(M, K, b, 1, seed=99, scale_dist="loguniform", outlier_frac=0.01)
    passes = 0
    t0 = time.perf_counter()
    while True:
        oracle.linear(d["bits"], d["M"], d["K"], d["zero"], d["q"], d["scales"], d["signs"],
                      d["x"], threads=cores)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    wb = passes * weight_bytes(M, K, b)
    return {"value": round(wb / dt / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{passes} full passes over the {M}x{K} 2-bit linear, batch 1, "
                      f"{dt:.1f} s wall on {cores} threads"}


def run_reference(a):
    rank, _, world = dist.env_world()
    if rank != 0:
        return
    import oracle
    cores = os.cpu_count() or 1
    M, K, b = HEAD
    d = synth.linear(M, K, b, 1, seed=99, scale_dist="loguniform", outlier_frac=0.01)
    rows = a.ref_rows
    for _ in range(max(a.warmup, 0)):
        oracle.linear(d["bits"], d["M"], d["K"], d["zero"], d["q"], d["scales"], d["signs"],
                      d["x"], 0, rows, threads=cores)
    t0 = time.perf_counter()
    for _ in range(a.steps):
        oracle.linear(d["bits"], d["M"], d["K"], d["zero"], d["q"], d["scales"], d["signs"],
                      d["x"], 0, rows, threads=cores)
    dt = time.perf_counter() - t0
    wb = a.steps * rows * (K * b // 8 + (K // 128) * 2)
    v = wb / dt / 1e9
    sample = f"each step: the first {rows} of {M} rows of the {M}x{K} 2-bit linear, batch 1"
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
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip the side workloads (other shapes, widths, the MoE layer)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-rows", type=int, default=512)
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
