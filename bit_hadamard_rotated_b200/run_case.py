"""Run one hq_linear (or one MoE layer, KV attention or screened readout) case a
few times on seeded synthetic inputs.

A reproducible target for profilers and quick timing:

    python -m bit_hadamard_rotated_b200.run_case --M 12288 --K 4096 --bits 2 --batch 1
    python -m bit_hadamard_rotated_b200.run_case --moe
    python -m bit_hadamard_rotated_b200.run_case --kv --tokens 8192
    python -m bit_hadamard_rotated_b200.run_case --readout
    python -m bit_hadamard_rotated_b200.run_case --M 8192 --K 8192 --batch 16 --tc-min-batch 1

Inputs come from bit_hadamard_rotated_b200.synth (seeded); every call goes
through the C ABI.  Prints the mean device time per call (CUDA events around
--reps back-to-back calls after --warmup calls) and checks the device status.
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from . import synth
from .hq import (KVCache, RotatedLinear, ScreenedReadout, expert_table, hq_check_status, hq_moe_experts,
                 hq_moe_workspace_size)


def _timed(fn, a):
    for _ in range(a.warmup):
        fn()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / max(a.reps, 1)


def run_kv(a):
    """Attention of a 32-token block (16 heads) over an int4 cache of --tokens
    tokens (4 kv heads of 128 channels), filled by hq_kv_append."""
    r = synth.kv(T=a.tokens, seed=a.seed)
    dev = torch.device("cuda", 0)
    c = KVCache(r["n_kv"], r["d"], r["T"], dev)
    c.append(torch.from_numpy(r["k"]).to(dev), torch.from_numpy(r["v"]).to(dev), 0)
    q = torch.from_numpy(r["q"]).to(dev)
    out = torch.empty((r["n_q"], r["n_heads"], r["d"]), dtype=torch.float32, device=dev)
    us = _timed(lambda: c.attend(q, r["T"], out=out), a)
    c.check_status()
    R = r["n_q"] * r["n_heads"] // r["n_kv"]
    flops = 4.0 * R * r["T"] * r["d"] * r["n_kv"]
    print(f"kv attend T={r['T']} kv heads {r['n_kv']} d={r['d']} query tokens {r['n_q']} x {r['n_heads']} heads: "
          f"{us:.2f} us/call ({flops / (us * 1e-6) / 1e12:.1f} TFLOP/s)")


def run_readout(a):
    """Screened top-8 readout over the 157,184 x 2048 8-bit lm_head (nibble planes), batch 1."""
    r = synth.readout(N=1, seed=a.seed)
    dev = torch.device("cuda", 0)
    hi = torch.from_numpy(r["hi"].view(np.int32)).to(dev)
    lo = torch.from_numpy(r["lo"].view(np.int32)).to(dev)
    ro = ScreenedReadout(hi, lo, torch.from_numpy(r["scales"]).to(dev), torch.from_numpy(r["signs"]).to(dev),
                         r["zero"], max_batch=1)
    x = torch.from_numpy(r["x"]).to(dev)
    us = _timed(lambda: ro.topk(x, 8), a)
    print(f"screened readout V={r['V']} K={r['K']} top-8 batch 1: {us:.2f} us/call")


def run_linear(a):
    d = synth.linear(a.M, a.K, a.bits, a.batch, seed=a.seed, scale_dist=a.scales)
    dev = torch.device("cuda", 0)
    lin = RotatedLinear(torch.from_numpy(d["q"].view(np.int32)).to(dev),
                        torch.from_numpy(d["scales"]).to(dev),
                        torch.from_numpy(d["signs"]).to(dev), a.bits, d["zero"], max_batch=a.batch)
    x = torch.from_numpy(d["x"]).to(dev)
    y = torch.empty((a.batch, a.M), dtype=torch.float32, device=dev)
    for _ in range(a.warmup):
        lin(x, out=y)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        lin(x, out=y)
    e1.record()
    torch.cuda.synchronize()
    lin.check_status()
    us = e0.elapsed_time(e1) * 1e3 / max(a.reps, 1)
    wb = d["q"].nbytes + d["scales"].nbytes
    print(f"linear M={a.M} K={a.K} b{a.bits} batch {a.batch}: {us:.2f} us/call "
          f"({wb / (us * 1e-6) / 1e9:.0f} GB/s weights, {lin.launches(a.batch)} launches/call, {lin.path(a.batch)})")


def run_moe(a):
    m = synth.moe(seed=a.seed)
    dev = torch.device("cuda", 0)

    def put(v):
        return torch.from_numpy(np.ascontiguousarray(v)).to(dev)

    experts = []
    for e in m["experts"]:
        d = dict(bits=e["bits"], zero=e["zero"])
        for n in ("q_gate", "q_up", "q_down"):
            d[n] = put(e[n].view(np.int32))
        for n in ("s_gate", "s_up", "s_down"):
            d[n] = put(e[n])
        experts.append(d)
    table = expert_table(experts, dev)
    E, H, I, T, k = len(experts), m["hidden"], m["inter"], m["T"], m["k"]
    x, ids = put(m["x"]), put(m["topk_ids"].astype(np.int32))
    w = put(m["topk_w"].astype(np.float32))
    s_in, s_mid = put(m["s_in"]), put(m["s_mid"])
    ws = torch.zeros(hq_moe_workspace_size(E, H, I, T, k), dtype=torch.uint8, device=dev)
    out = torch.empty((T, H), dtype=torch.float32, device=dev)
    for _ in range(a.warmup):
        hq_moe_experts(table, E, H, I, x, ids, w, s_in, s_mid, out=out, workspace=ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        hq_moe_experts(table, E, H, I, x, ids, w, s_in, s_mid, out=out, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    hq_check_status(ws)
    us = e0.elapsed_time(e1) * 1e3 / max(a.reps, 1)
    tb = synth.touched_weight_bytes(m)
    print(f"moe E={E} hidden={H} inter={I} tokens={T} top-{k}: {us:.2f} us/call "
          f"({tb / (us * 1e-6) / 1e9:.0f} GB/s over {tb / 1e6:.1f} MB of touched expert weights)")


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--M", type=int, default=12288)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--bits", type=int, default=2)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--scales", default="uniform", choices=["uniform", "loguniform"])
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--moe", action="store_true", help="run the MoE expert layer instead")
    ap.add_argument("--kv", action="store_true", help="run the int4 KV attention instead")
    ap.add_argument("--tokens", type=int, default=8192, help="cached tokens for --kv")
    ap.add_argument("--readout", action="store_true", help="run the screened readout instead")
    ap.add_argument("--gemv32-min-batch", type=int, default=0,
                    help="hq_set_gemv32_min_batch before the run (0: automatic)")
    ap.add_argument("--tc-min-batch", type=int, default=0, help="hq_set_tc_min_batch before the run (0: automatic)")
    a = ap.parse_args()
    if not torch.cuda.is_available():
        raise SystemExit("run_case needs a CUDA device")
    from .hq import hq_set_gemv32_min_batch, hq_set_tc_min_batch
    hq_set_gemv32_min_batch(a.gemv32_min_batch)
    hq_set_tc_min_batch(a.tc_min_batch)
    if a.moe:
        run_moe(a)
    elif a.kv:
        run_kv(a)
    elif a.readout:
        run_readout(a)
    else:
        run_linear(a)


if __name__ == "__main__":
    main()
