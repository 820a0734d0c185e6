"""Seeded synthetic inputs for the rotated low-bit linear and the MoE layer.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no rotation, no dequantisation, no contraction), so the
CUDA path and the CPU oracle can both consume what it produces without sharing
any computation.

Uniform codes are drawn as uniform random *bits* of the packed words: every
b-bit field of a uniformly random bit stream is uniform on [0, 2^b), so no
packing step is needed here.

Workloads (shapes and distributions of the pages' deployment: group-128 codes,
2/3/4-bit experts and 8-bit non-expert layers -- LLaDA2.2-mini Orin-Nano model
card, Properties table; a 32-token denoising block -- same card, "Measured
Throughput"):

* ``linear``: codes uniform, fp16 scales uniform in [0.005, 0.02] or
  log-uniform in [0.003, 0.03], zero point 2^(b-1), fp16 activations N(0, 1)
  with an optional seeded fraction of outlier channels scaled x20 (the same
  channels for every row), signs uniform on {-1, +1}.
* ``moe``: 256 experts of hidden 2048 / intermediate 512, bit widths drawn
  70/20/10 % from {2, 3, 4}, router logits N(0, 1) fp32, top-8 by logit (ties
  to the lower expert index), routing weights = softmax over the 8 selected
  logits.
"""
from __future__ import annotations

import numpy as np

GROUP = 128


def _rng(*seed_parts: int) -> np.random.Generator:
    return np.random.default_rng([int(s) & 0xFFFFFFFF for s in seed_parts])


def packed_words(rng: np.random.Generator, rows: int, K: int, bits: int) -> np.ndarray:
    """Uniform random packed codes: [rows][K*bits/32] uint32."""
    assert (K * bits) % 32 == 0
    return rng.integers(0, 2**32, size=(rows, K * bits // 32), dtype=np.uint64).astype(np.uint32)


def scales_uniform(rng, rows, K, lo=0.005, hi=0.02) -> np.ndarray:
    return rng.uniform(lo, hi, size=(rows, K // GROUP)).astype(np.float16)


def scales_loguniform(rng, rows, K, lo=0.003, hi=0.03) -> np.ndarray:
    return np.exp(rng.uniform(np.log(lo), np.log(hi), size=(rows, K // GROUP))).astype(np.float16)


def signs(rng, K) -> np.ndarray:
    return (rng.integers(0, 2, size=K, dtype=np.int8) * 2 - 1).astype(np.int8)


def activations(rng, N, K, outlier_frac=0.0, outlier_mult=20.0) -> np.ndarray:
    x = rng.standard_normal((N, K))
    if outlier_frac > 0:
        n_out = int(round(outlier_frac * K))
        ch = rng.choice(K, size=n_out, replace=False)
        x[:, ch] *= outlier_mult
    return x.astype(np.float16)


def linear(M: int, K: int, bits: int, N: int, seed: int = 0, scale_dist: str = "uniform",
           outlier_frac: float = 0.0) -> dict:
    """One rotated linear layer plus a batch of N activation rows."""
    rng = _rng(seed, M, K, bits, N)
    q = packed_words(rng, M, K, bits)
    sc = scales_uniform(rng, M, K) if scale_dist == "uniform" else scales_loguniform(rng, M, K)
    s = signs(rng, K)
    x = activations(rng, N, K, outlier_frac)
    return dict(bits=bits, M=M, K=K, N=N, zero=1 << (bits - 1), q=q, scales=sc, signs=s, x=x)


def expert_bits(rng, E, probs=(0.7, 0.2, 0.1), choices=(2, 3, 4)) -> np.ndarray:
    return rng.choice(np.array(choices), size=E, p=np.array(probs)).astype(np.int32)


def routing(rng, T, E, k):
    """Top-k of N(0,1) fp32 logits (ties -> lower index); weights = softmax over the k."""
    logits = rng.standard_normal((T, E)).astype(np.float32)
    # stable sort on -logit keeps the lower index first among equal logits
    order = np.argsort(-logits, axis=1, kind="stable")[:, :k].astype(np.int32)
    sel = np.take_along_axis(logits, order, axis=1).astype(np.float64)
    ex = np.exp(sel - sel.max(axis=1, keepdims=True))
    w = (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)
    return logits, order, w


def moe(seed: int = 0, E: int = 256, hidden: int = 2048, inter: int = 512, T: int = 32,
        k: int = 8, probs=(0.7, 0.2, 0.1), bits_choices=(2, 3, 4)) -> dict:
    """MoE expert layer: per-expert packed gate/up/down, activations and routing."""
    rng = _rng(seed, E, hidden, inter, T, k)
    eb = expert_bits(rng, E, probs, bits_choices)
    experts = []
    for e in range(E):
        b = int(eb[e])
        experts.append(dict(
            bits=b, zero=1 << (b - 1),
            q_gate=packed_words(rng, inter, hidden, b),
            q_up=packed_words(rng, inter, hidden, b),
            q_down=packed_words(rng, hidden, inter, b),
            s_gate=scales_uniform(rng, inter, hidden),
            s_up=scales_uniform(rng, inter, hidden),
            s_down=scales_uniform(rng, hidden, inter),
        ))
    x = activations(rng, T, hidden)
    logits, ids, w = routing(rng, T, E, k)
    return dict(E=E, hidden=hidden, inter=inter, T=T, k=k, experts=experts, x=x,
                logits=logits, topk_ids=ids, topk_w=w,
                s_in=signs(rng, hidden), s_mid=signs(rng, inter))


def touched_weight_bytes(inp: dict) -> int:
    """Packed-code plus scale bytes of the experts that the routing touches."""
    total = 0
    for e in np.unique(inp["topk_ids"]):
        ex = inp["experts"][int(e)]
        for n in ("q_gate", "q_up", "q_down", "s_gate", "s_up", "s_down"):
            total += ex[n].nbytes
    return total


def readout(V: int = 157184, K: int = 2048, N: int = 1, seed: int = 0) -> dict:
    """An 8-bit lm_head stored as high and low nibble planes (each a uniform
    4-bit packed matrix [V][K/8] words, so the 8-bit codes 16 hi + lo are
    uniform too), fp16 scales U[0.005, 0.02], zero point 128, signs, x ~ N(0, 1)
    fp16 [N][K].  Default sizes: a 157,184-token vocabulary over hidden 2048."""
    rng = _rng(seed, V, K, N, 8)
    hi = packed_words(rng, V, K, 4)
    lo = packed_words(rng, V, K, 4)
    return dict(V=V, K=K, N=N, zero=128, hi=hi, lo=lo, scales=scales_uniform(rng, V, K),
                signs=signs(rng, K), x=activations(rng, N, K))


def kv(T: int = 32768, n_kv: int = 4, d: int = 128, n_q: int = 32, n_heads: int = 16,
       seed: int = 0) -> dict:
    """One attention layer's keys and values for T tokens (fp16 [T][n_kv][d],
    N(0, 1); keys with a seeded 2 % of channels x8, the same for every token, as
    key caches usually have) and a block of n_q query tokens (fp16
    [n_q][n_heads][d], N(0, 1)).  Defaults: a 32K-token context, 4 kv heads of
    128 channels, 16 query heads, one 32-token denoising block."""
    rng = _rng(seed, T, n_kv, d, n_q, n_heads)
    k = rng.standard_normal((T, n_kv, d))
    ch = rng.choice(d, size=max(1, d // 50), replace=False)
    k[:, :, ch] *= 8.0
    v = rng.standard_normal((T, n_kv, d))
    q = rng.standard_normal((n_q, n_heads, d))
    return dict(T=T, n_kv=n_kv, d=d, n_q=n_q, n_heads=n_heads, k=k.astype(np.float16),
                v=v.astype(np.float16), q=q.astype(np.float16))
