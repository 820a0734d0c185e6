"""Plain fp64 CPU oracle for the rotated low-bit linear -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product library never loads it and shares no code with it: the arithmetic
lives in ``hq_oracle.c`` (scalar loops, double precision) and this module
only marshals numpy arrays into it.

The formulas and the readings of the pages they rest on are in
``hq_oracle.h``: the random-sign Hadamard rotation x' = H.diag(s).x/sqrt(K)
("group-128 GPTQ in a Hadamard-rotated basis" with "rotation signs":
LLaDA2.2-mini Orin-Nano model card, Properties table and file list), the
group-128 dequantisation w = scale.(q - z), the fp64 contraction, the
SwiGLU MoE expert composition, and the rotated round-to-nearest quantiser
that produces packed weights.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hq_oracle.c")
_HDR = os.path.join(_HERE, "hq_oracle.h")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile hq_oracle.c into oracle/liboracle.so with gcc (-O2, no fast-math)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < newest:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
             "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class Expert(ctypes.Structure):
    _fields_ = [
        ("bits", ctypes.c_int), ("zero", ctypes.c_int),
        ("q_gate", ctypes.c_void_p), ("q_up", ctypes.c_void_p), ("q_down", ctypes.c_void_p),
        ("s_gate", ctypes.c_void_p), ("s_up", ctypes.c_void_p), ("s_down", ctypes.c_void_p),
        ("signs_in", ctypes.c_void_p), ("signs_mid", ctypes.c_void_p),
    ]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
            L.hqo_f16_to_f64.argtypes = [ctypes.c_uint16]
            L.hqo_f16_to_f64.restype = ctypes.c_double
            L.hqo_unpack.argtypes = [vp, i, sz, vp]
            L.hqo_pack.argtypes = [vp, i, sz, vp]
            L.hqo_unpack_planes2.argtypes = [vp, sz, vp]
            L.hqo_pack_planes2.argtypes = [vp, sz, vp]
            L.hqo_fwht.argtypes = [vp, i]
            L.hqo_rotate.argtypes = [vp, vp, i, vp]
            L.hqo_rotate_f16.argtypes = [vp, vp, i, vp]
            L.hqo_dequant_dot.argtypes = [i, i, i, i, vp, vp, vp, vp, i, i, i, vp, vp]
            L.hqo_linear.argtypes = [i, i, i, i, vp, vp, vp, vp, vp, i, i, i, vp, vp]
            L.hqo_moe.argtypes = [vp, i, i, i, vp, i, vp, vp, i, vp, vp, i, i, vp, vp, vp]
            L.hqo_f64_to_f16.argtypes = [ctypes.c_double]
            L.hqo_f64_to_f16.restype = ctypes.c_uint16
            L.hqo_quantize.argtypes = [vp, i, i, i, vp, i, i, vp, vp, vp]
            L.hqo_kv_quant_group.argtypes = [vp, i, i, vp, vp, vp]
            L.hqo_kv_quantize.argtypes = [vp, vp, i, i, i, vp, vp, vp, vp, vp, vp]
            L.hqo_kv_attend.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, vp, i, i, vp, vp]
            L.hqo_readout.argtypes = [vp, vp, vp, vp, i, i, i, vp, i, i, ctypes.c_double, vp, vp, vp,
                                      vp, vp]
            for f in ("hqo_unpack", "hqo_pack", "hqo_unpack_planes2", "hqo_pack_planes2", "hqo_fwht", "hqo_rotate", "hqo_rotate_f16",
                      "hqo_dequant_dot", "hqo_linear", "hqo_moe", "hqo_quantize", "hqo_readout",
                      "hqo_kv_quant_group", "hqo_kv_quantize", "hqo_kv_attend"):
                getattr(L, f).restype = None
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def f16_to_f64(bits_u16: int) -> float:
    return lib().hqo_f16_to_f64(int(bits_u16))


def f64_to_f16(v: float) -> int:
    """binary16 bit pattern nearest to v (ties to even)."""
    return int(lib().hqo_f64_to_f16(float(v)))


def quantize(W, bits: int, signs=None, m_begin=0, m_end=None, want_rotated=False, threads=1):
    """Rotated round-to-nearest quantiser (hq_oracle.h).  W: [M][K] (any real
    dtype, read as float64).  Returns (qweight uint32 [M][K*bits/32], scales
    fp16 [M][K/128], rotated float64 [M][K] or None)."""
    Wd = _c(W, np.float64)
    M, K = Wd.shape
    s = _c(signs, np.int8)
    m_end = M if m_end is None else m_end
    q = np.zeros((M, K * bits // 32), np.uint32)
    sc = np.zeros((M, K // 128), np.uint16)
    r = np.zeros((M, K), np.float64) if want_rotated else None

    def run(lo, hi):
        lib().hqo_quantize(_p(Wd), M, K, bits, _p(s), lo, hi, _p(q), _p(sc), _p(r))

    if threads <= 1:
        run(m_begin, m_end)
    else:
        edges = np.linspace(m_begin, m_end, threads + 1).astype(int)
        ts = [threading.Thread(target=run, args=(int(edges[t]), int(edges[t + 1])))
              for t in range(threads)]
        for t in ts:
            t.start()
        for t in ts:
            t.join()
    return q, sc.view(np.float16), r


def unpack(words, bits: int, n_codes: int) -> np.ndarray:
    words = _c(words, np.uint32)
    assert words.size * 32 >= bits * n_codes
    out = np.empty(n_codes, np.uint8)
    lib().hqo_unpack(_p(words), bits, n_codes, _p(out))
    return out


def pack(codes, bits: int) -> np.ndarray:
    codes = _c(codes, np.uint8)
    n = codes.size
    out = np.empty((bits * n + 31) // 32, np.uint32)
    lib().hqo_pack(_p(codes), bits, n, _p(out))
    return out


def unpack_planes2(words, n_codes: int) -> np.ndarray:
    """2-bit codes from the bit-plane layout (hq_oracle.h, hqo_unpack_planes2)."""
    words = _c(words, np.uint32)
    assert n_codes % 32 == 0 and words.size * 16 >= n_codes
    out = np.empty(n_codes, np.uint8)
    lib().hqo_unpack_planes2(_p(words), n_codes, _p(out))
    return out


def pack_planes2(codes) -> np.ndarray:
    codes = _c(codes, np.uint8)
    assert codes.size % 32 == 0
    out = np.empty(codes.size // 16, np.uint32)
    lib().hqo_pack_planes2(_p(codes), codes.size, _p(out))
    return out


def planes_to_packed2(q, M, K) -> np.ndarray:
    """[M][K/16] bit-plane words -> the same codes in the packed 2-bit stream."""
    q = _c(q, np.uint32).reshape(M, K // 16)
    return np.stack([pack(unpack_planes2(q[m], K), 2) for m in range(M)])


def fwht(v) -> np.ndarray:
    v = np.array(v, dtype=np.float64, copy=True)
    lib().hqo_fwht(_p(v), v.size)
    return v


def rotate(x, signs=None) -> np.ndarray:
    """x: [..., K] float64 (or fp16 array) -> H.diag(s).x/sqrt(K) per row, float64."""
    x = np.asarray(x)
    K = x.shape[-1]
    rows = x.reshape(-1, K)
    s = _c(signs, np.int8)
    out = np.empty(rows.shape, np.float64)
    if rows.dtype == np.float16:
        r16 = np.ascontiguousarray(rows).view(np.uint16)
        for r in range(rows.shape[0]):
            lib().hqo_rotate_f16(_p(r16[r]), _p(s), K, _p(out[r]))
    else:
        rd = np.ascontiguousarray(rows, dtype=np.float64)
        for r in range(rows.shape[0]):
            lib().hqo_rotate(_p(rd[r]), _p(s), K, _p(out[r]))
    return out.reshape(x.shape)


def dequant_dot(bits, M, K, zero, q, scales, xr, m_begin=0, m_end=None, with_bound=True,
                zeros=None, planes=False):
    """y[n][m] = sum_k scale.(q - z).xr[n][k] for already-rotated xr [N][K]; z =
    zeros[m][k/128] (uint8 [M][K/128]) if given, else the scalar zero.
    planes: q holds 2-bit codes in the bit-plane layout."""
    q = planes_to_packed2(q, M, K) if planes else _c(q, np.uint32)
    zr = _c(zeros, np.uint8)
    sc = np.ascontiguousarray(scales).view(np.uint16) if np.asarray(scales).dtype == np.float16 \
        else _c(scales, np.uint16)
    xr = _c(xr, np.float64).reshape(-1, K)
    N = xr.shape[0]
    m_end = M if m_end is None else m_end
    y = np.zeros((N, M), np.float64)
    b = np.zeros((N, M), np.float64) if with_bound else None
    lib().hqo_dequant_dot(bits, M, K, zero, _p(zr), _p(q), _p(sc), _p(xr), N, m_begin, m_end, _p(y),
                          _p(b))
    return (y, b) if with_bound else y


def linear(bits, M, K, zero, q, scales, signs, x, m_begin=0, m_end=None, threads=1, zeros=None,
           planes=False):
    """Full rotated linear in fp64.  x: fp16 [N][K].  Returns (y, bound) float64 [N][M].
    zeros: per-group zero points uint8 [M][K/128] (else the scalar zero).
    planes: q holds 2-bit codes in the bit-plane layout (converted to the
    packed stream first: the codes, and so the result, are the same).

    threads > 1 splits the output rows across Python threads (the C call
    releases the GIL), each running the unchanged scalar code on its rows.
    """
    q = planes_to_packed2(q, M, K) if planes else _c(q, np.uint32)
    sc = np.ascontiguousarray(scales, dtype=np.float16).view(np.uint16)
    s = _c(signs, np.int8)
    zr = _c(zeros, np.uint8)
    x16 = np.ascontiguousarray(x, dtype=np.float16).reshape(-1, K).view(np.uint16)
    N = x16.shape[0]
    m_end = M if m_end is None else m_end
    y = np.zeros((N, M), np.float64)
    b = np.zeros((N, M), np.float64)

    def run(lo, hi):
        lib().hqo_linear(bits, M, K, zero, _p(zr), _p(q), _p(sc), _p(s), _p(x16), N, lo, hi, _p(y), _p(b))

    if threads <= 1:
        run(m_begin, m_end)
    else:
        edges = np.linspace(m_begin, m_end, threads + 1).astype(int)
        ts = [threading.Thread(target=run, args=(int(edges[t]), int(edges[t + 1])))
              for t in range(threads)]
        for t in ts:
            t.start()
        for t in ts:
            t.join()
    return y, b


def moe(experts, hidden, inter, x, topk_ids, topk_w, s_in, s_mid, t_begin=0, t_end=None,
        want_h=False, threads=1):
    """MoE expert layer in fp64.  experts: list of dicts with keys bits, zero,
    q_gate, q_up, q_down (uint32 arrays) and s_gate, s_up, s_down (fp16 arrays),
    and optionally the expert's own rotation signs signs_in, signs_mid (int8).
    Returns (y [T][hidden], bound [T][hidden], h [T*k][inter] or None)."""
    keep = []
    arr = (Expert * len(experts))()
    for i, e in enumerate(experts):
        qs = [_c(e[n], np.uint32) for n in ("q_gate", "q_up", "q_down")]
        ss = [np.ascontiguousarray(e[n], dtype=np.float16).view(np.uint16)
              for n in ("s_gate", "s_up", "s_down")]
        own = [_c(e.get(n), np.int8) for n in ("signs_in", "signs_mid")]
        keep += qs + ss + [o for o in own if o is not None]
        arr[i] = Expert(int(e["bits"]), int(e["zero"]), *[a.ctypes.data for a in qs + ss],
                        *[None if o is None else o.ctypes.data for o in own])
    x16 = np.ascontiguousarray(x, dtype=np.float16).reshape(-1, hidden).view(np.uint16)
    T = x16.shape[0]
    ids = _c(topk_ids, np.int32).reshape(T, -1)
    k = ids.shape[1]
    w = _c(topk_w, np.float32).reshape(T, k)
    si, sm = _c(s_in, np.int8), _c(s_mid, np.int8)
    t_end = T if t_end is None else t_end
    y = np.zeros((T, hidden), np.float64)
    b = np.zeros((T, hidden), np.float64)
    h = np.zeros((T * k, inter), np.float64) if want_h else None

    def run(lo, hi):
        lib().hqo_moe(ctypes.cast(arr, ctypes.c_void_p), len(experts), hidden, inter, _p(x16), T,
                      _p(ids), _p(w), k, _p(si), _p(sm), lo, hi, _p(y), _p(b), _p(h))

    if threads <= 1:
        run(t_begin, t_end)
    else:
        edges = np.linspace(t_begin, t_end, threads + 1).astype(int)
        ts = [threading.Thread(target=run, args=(int(edges[t]), int(edges[t + 1])))
              for t in range(threads)]
        for t in ts:
            t.start()
        for t in ts:
            t.join()
    del keep
    return y, b, h


def readout(hi, lo, scales, signs, V, K, zero, x, topk, beta=6.0, want_all=False):
    """Nibble-split screened readout (hq_oracle.h).  hi, lo: uint32 4-bit planes
    [V][K/8]; x fp16 [N][K].  Returns (ids int32 [N][topk], logits float64
    [N][topk], cand uint8 [N][V], y_all [N][V] or None, e [N][V] or None)."""
    hi, lo = _c(hi, np.uint32), _c(lo, np.uint32)
    sc = np.ascontiguousarray(scales, dtype=np.float16).view(np.uint16)
    s = _c(signs, np.int8)
    x16 = np.ascontiguousarray(x, dtype=np.float16).reshape(-1, K).view(np.uint16)
    N = x16.shape[0]
    ids = np.zeros((N, topk), np.int32)
    out = np.zeros((N, topk), np.float64)
    cand = np.zeros((N, V), np.uint8)
    ya = np.zeros((N, V), np.float64) if want_all else None
    ea = np.zeros((N, V), np.float64) if want_all else None
    lib().hqo_readout(_p(hi), _p(lo), _p(sc), _p(s), V, K, zero, _p(x16), N, topk, float(beta), _p(ids),
                      _p(out), _p(cand), _p(ya), _p(ea))
    return ids, out, cand, ya, ea


def kv_quantize(k, v):
    """int4 KV cache of one layer (hq_oracle.h).  k, v: fp16 [T][n_kv][d], T a
    multiple of 32.  Returns dict kc uint8 [n_kv][T/32][d][32], ks, km fp16
    [n_kv][T/32][d], vc uint8 [n_kv][T][d], vs, vm fp16 [n_kv][T] (codes one
    byte each)."""
    k16 = np.ascontiguousarray(k, dtype=np.float16)
    v16 = np.ascontiguousarray(v, dtype=np.float16)
    T, n_kv, d = k16.shape
    kb = k16.view(np.uint16)
    vb = v16.view(np.uint16)
    nb = T // 32
    kc = np.zeros((n_kv, nb, d, 32), np.uint8)
    ks = np.zeros((n_kv, nb, d), np.uint16)
    km = np.zeros((n_kv, nb, d), np.uint16)
    vc = np.zeros((n_kv, T, d), np.uint8)
    vs = np.zeros((n_kv, T), np.uint16)
    vm = np.zeros((n_kv, T), np.uint16)
    lib().hqo_kv_quantize(_p(kb), _p(vb), T, n_kv, d, _p(kc), _p(ks), _p(km), _p(vc), _p(vs), _p(vm))
    return dict(kc=kc, ks=ks.view(np.float16), km=km.view(np.float16), vc=vc, vs=vs.view(np.float16),
                vm=vm.view(np.float16))


def kv_attend(cache, T, q):
    """Attention of q fp16 [n_q][n_heads][d] over the first T tokens of a
    kv_quantize cache (T >= 1, any), fp64.  Returns (out, base) [n_q][n_heads][d]."""
    n_kv, _, d, _ = cache["kc"].shape
    nb = (T + 31) // 32
    kc = np.ascontiguousarray(cache["kc"][:, :nb])
    ks = np.ascontiguousarray(cache["ks"][:, :nb]).view(np.uint16)
    km = np.ascontiguousarray(cache["km"][:, :nb]).view(np.uint16)
    vc = np.ascontiguousarray(cache["vc"][:, :T])
    vs = np.ascontiguousarray(cache["vs"][:, :T]).view(np.uint16)
    vm = np.ascontiguousarray(cache["vm"][:, :T]).view(np.uint16)
    q16 = np.ascontiguousarray(q, dtype=np.float16)
    n_q, n_heads, _ = q16.shape
    out = np.zeros((n_q, n_heads, d), np.float64)
    base = np.zeros_like(out)
    lib().hqo_kv_attend(_p(kc), _p(ks), _p(km), _p(vc), _p(vs), _p(vm), n_kv, d, T, _p(q16.view(np.uint16)),
                        n_q, n_heads, _p(out), _p(base))
    return out, base
