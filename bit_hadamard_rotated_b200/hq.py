"""Python entry points with the C ABI's names (include/hq.h).

Each function checks tensor devices/dtypes/shapes, marshals pointers and the
current CUDA stream, and calls libhq.  Nothing is computed here.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import (HQ_BF16, HQ_F16, HQ_F32, HqError, HqExpert, HqKvCache, HqReadout, HqWeight, check,
                   lib)

_DT = {torch.float16: HQ_F16, torch.bfloat16: HQ_BF16, torch.float32: HQ_F32}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _raw_stream(stream, device_index):
    """The stream handle as an int: the given stream, else the current one of
    the device (read without building a Stream object)."""
    if stream is not None:
        return stream.cuda_stream
    get = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    return get(device_index) if get is not None else torch.cuda.current_stream().cuda_stream


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libhq takes CUDA tensors only (no CPU fallback)")


def hq_rotate(x: torch.Tensor, signs: torch.Tensor | None = None, out_dtype=torch.float32,
              out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """x' = H_K diag(s) x / sqrt(K) for every row of x ([..., K])."""
    _need_cuda(x, signs)
    K = x.shape[-1]
    x = x.contiguous()
    if out is None:
        out = torch.empty(x.shape, dtype=out_dtype, device=x.device)
    n_rows = x.numel() // K if K else 0
    st = lib().hq_rotate(_ptr(x), _DT[x.dtype], _ptr(out), _DT[out.dtype], n_rows, K,
                         _ptr(signs), _stream(stream))
    check(st, "hq_rotate")
    return out


def hq_quantize(W: torch.Tensor, bits: int, signs: torch.Tensor | None = None,
                qweight: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                stream=None):
    """Pack real weights W [M][K] (fp16/bf16/fp32) into (qweight int32 [M][K*bits/32],
    scales fp16 [M][K/128]) with the rotated round-to-nearest quantiser; the zero
    point of the result is 2^(bits-1)."""
    _need_cuda(W, signs)
    if W.dim() != 2 or W.dtype not in _DT or not W.is_contiguous():
        raise ValueError("W must be a contiguous [M][K] fp16, bf16 or fp32 tensor")
    M, K = W.shape
    with torch.cuda.device(W.device):
        if qweight is None:
            qweight = torch.empty((M, K * bits // 32), dtype=torch.int32, device=W.device)
        if scales is None:
            scales = torch.empty((M, K // 128), dtype=torch.float16, device=W.device)
        st = lib().hq_quantize(_ptr(W), _DT[W.dtype], M, K, bits, _ptr(signs), _ptr(qweight),
                               _ptr(scales), _stream(stream))
    check(st, "hq_quantize")
    return qweight, scales


def make_weight(qweight: torch.Tensor, scales: torch.Tensor, signs: torch.Tensor | None,
                bits: int, zero: int | None = None, zeros: torch.Tensor | None = None,
                planes: bool = False) -> HqWeight:
    """Weight descriptor; zeros: optional per-group zero points uint8 [M][K/128];
    planes: 2-bit codes in the bit-plane layout (hq_to_bitplanes)."""
    M = qweight.shape[0]
    K = qweight.shape[1] * 32 // bits
    z = (1 << (bits - 1)) if zero is None else int(zero)
    if zeros is not None and (zeros.dtype != torch.uint8 or tuple(zeros.shape) != (M, K // 128)
                              or not zeros.is_contiguous()):
        raise ValueError(f"zeros must be contiguous uint8 [{M}][{K // 128}]")
    return HqWeight(bits, M, K, z, qweight.data_ptr(), scales.data_ptr(),
                    None if signs is None else signs.data_ptr(),
                    None if zeros is None else zeros.data_ptr(), 1 if planes else 0)


def hq_linear_workspace_size(w: HqWeight, batch: int) -> int:
    return int(lib().hq_linear_workspace_size(ctypes.byref(w), batch))


def _check_linear_io(w: HqWeight, x: torch.Tensor, out: torch.Tensor | None, dev) -> None:
    """x must be contiguous fp16 [N][K] and out contiguous fp32 [N][M], both on
    the weight's device (the kernels read raw pointers: a wrong shape or
    stride would read out of bounds)."""
    if x.dtype != torch.float16 or x.dim() != 2 or x.shape[1] != w.K or not x.is_contiguous():
        raise ValueError(f"x must be contiguous fp16 [N][{w.K}], got {x.dtype} {tuple(x.shape)}")
    if x.device != dev:
        raise ValueError(f"x is on {x.device}, the weights on {dev}")
    if out is not None:
        N = x.shape[0]
        if out.dtype != torch.float32 or tuple(out.shape) != (N, w.M) or not out.is_contiguous():
            raise ValueError(f"out must be contiguous fp32 [{N}][{w.M}]")
        if out.device != dev:
            raise ValueError(f"out is on {out.device}, the weights on {dev}")


def hq_linear(qweight: torch.Tensor, scales: torch.Tensor, signs: torch.Tensor | None,
              x: torch.Tensor, bits: int, zero: int | None = None,
              out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
              stream=None, zeros: torch.Tensor | None = None, planes: bool = False) -> torch.Tensor:
    """y[n][m] = sum_k scale (q - zero) x'[n][k]; x fp16 [N][K] -> y fp32 [N][M]
    (zero per tensor, or per row and group with zeros uint8 [M][K/128];
    planes: 2-bit codes in the bit-plane layout)."""
    _need_cuda(qweight, scales, signs, x, zeros)
    w = make_weight(qweight, scales, signs, bits, zero, zeros, planes)
    _check_linear_io(w, x, out, qweight.device)
    N = x.shape[0]
    with torch.cuda.device(qweight.device):
        if out is None:
            out = torch.empty((N, w.M), dtype=torch.float32, device=x.device)
        need = hq_linear_workspace_size(w, N)
        if workspace is None:
            workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=x.device)
        st = lib().hq_linear(ctypes.byref(w), _ptr(x), N, _ptr(out), _ptr(workspace),
                             workspace.numel(), _stream(stream))
    check(st, "hq_linear")
    return out


def hq_linear_noalloc(qweight: torch.Tensor, scales: torch.Tensor, signs: torch.Tensor | None,
                      x: torch.Tensor, bits: int, zero: int | None = None,
                      out: torch.Tensor | None = None, stream=None,
                      zeros: torch.Tensor | None = None, planes: bool = False) -> torch.Tensor:
    """hq_linear without a workspace (the library's fixed device scratch is
    used instead; calls must not overlap on the GPU)."""
    _need_cuda(qweight, scales, signs, x, zeros)
    w = make_weight(qweight, scales, signs, bits, zero, zeros, planes)
    _check_linear_io(w, x, out, qweight.device)
    N = x.shape[0]
    with torch.cuda.device(qweight.device):
        if out is None:
            out = torch.empty((N, w.M), dtype=torch.float32, device=x.device)
        st = lib().hq_linear_noalloc(ctypes.byref(w), _ptr(x), N, _ptr(out), _stream(stream))
    check(st, "hq_linear_noalloc")
    return out


def hq_linear_noalloc_check_status(stream=None) -> None:
    """Raise HqError if the last hq_linear_noalloc call recorded a device error."""
    check(lib().hq_linear_noalloc_check_status(_stream(stream)), "hq_linear_noalloc status")


class RotatedLinear:
    """A packed, rotated linear layer bound to its device tensors and workspace."""

    def __init__(self, qweight, scales, signs, bits, zero=None, max_batch=64, zeros=None, planes=False):
        _need_cuda(qweight, scales, signs, zeros)
        self.qweight, self.scales, self.signs, self.bits, self.zeros = qweight, scales, signs, bits, zeros
        self.w = make_weight(qweight, scales, signs, bits, zero, zeros, planes)
        self.workspace = torch.zeros(max(hq_linear_workspace_size(self.w, max_batch), 256),
                                     dtype=torch.uint8, device=qweight.device)
        # per-call marshalling reduced to the two tensor pointers and the stream
        self._fn = lib().hq_linear
        self._wref = ctypes.byref(self.w)
        self._ws = self.workspace.data_ptr()
        self._ws_bytes = self.workspace.numel()
        self._dev = qweight.device.index if qweight.device.index is not None else torch.cuda.current_device()

    @property
    def M(self):
        return self.w.M

    @property
    def K(self):
        return self.w.K

    def launches(self, batch: int) -> int:
        return int(lib().hq_linear_launches(ctypes.byref(self.w), batch))

    def uses_tensor_cores(self, batch: int) -> bool:
        """Whether a call of this batch runs on the tensor-core GEMM (else a GEMV)."""
        return int(lib().hq_linear_uses_tensor_cores(ctypes.byref(self.w), batch)) == 1

    def path(self, batch: int) -> str:
        """The kernel family a call of this batch runs on: "GEMV", "tensor cores"
        or "GEMV32" (32-row tiles, up to 16 columns)."""
        p = int(lib().hq_linear_path(ctypes.byref(self.w), batch))
        return {0: "GEMV", 1: "tensor cores", 2: "GEMV32"}[p]

    def __call__(self, x, out=None, stream=None):
        N = x.shape[0]
        if out is None:
            out = torch.empty((N, self.w.M), dtype=torch.float32, device=x.device)
        st = self._fn(self._wref, x.data_ptr(), N, out.data_ptr(), self._ws, self._ws_bytes,
                      _raw_stream(stream, self._dev))
        if st:
            check(st, "hq_linear")
        return out

    def prepare(self, x, out, stream=None):
        """A zero-argument launcher of this layer on fixed buffers and a fixed
        stream (the current one if None), for loops that reuse them, such as a
        decode step: the buffers are checked once here, and each call is one
        hq_linear call with its arguments already marshalled."""
        _need_cuda(x, out)
        N = x.shape[0]
        if x.dtype != torch.float16 or x.dim() != 2 or x.shape[1] != self.w.K or not x.is_contiguous():
            raise ValueError(f"x must be contiguous fp16 [N][{self.w.K}]")
        if out.dtype != torch.float32 or tuple(out.shape) != (N, self.w.M) or not out.is_contiguous():
            raise ValueError(f"out must be contiguous fp32 [{N}][{self.w.M}]")
        if hq_linear_workspace_size(self.w, N) > self._ws_bytes:
            raise ValueError(f"batch {N} is larger than this layer's workspace allows")
        fn = self._fn
        args = (self._wref, ctypes.c_void_p(x.data_ptr()), ctypes.c_int(N),
                ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(self._ws),
                ctypes.c_size_t(self._ws_bytes), ctypes.c_void_p(_raw_stream(stream, self._dev)))

        def launch():
            st = fn(*args)
            if st:
                check(st, "hq_linear")

        launch.buffers = (self, x, out)  # keep them alive as long as the launcher
        return launch

    def check_status(self, stream=None):
        check(lib().hq_check_status(_ptr(self.workspace), _stream(stream)), "device status")


class ScreenedReadout:
    """An 8-bit lm_head kept as nibble planes (hi, lo: int32 [V][K/8] 4-bit
    layout; scales fp16 [V][K/128]; signs int8 [K] or None), with its own
    workspace for batches up to max_batch (<= 8)."""

    def __init__(self, hi, lo, scales, signs, zero=128, max_batch=8):
        _need_cuda(hi, lo, scales, signs)
        V, K = hi.shape[0], hi.shape[1] * 8
        self.tensors = (hi, lo, scales, signs)
        self.r = HqReadout(V, K, int(zero), hi.data_ptr(), lo.data_ptr(), scales.data_ptr(),
                           None if signs is None else signs.data_ptr())
        need = int(lib().hq_readout_workspace_size(ctypes.byref(self.r), max_batch))
        if need == 0:
            raise ValueError("unsupported readout shape or batch")
        self.workspace = torch.zeros(need, dtype=torch.uint8, device=hi.device)

    def topk(self, x, k, beta=6.0, stream=None):
        """(ids int32 [N][k], logits fp32 [N][k]) of the largest exact logits."""
        _need_cuda(x)
        N = x.shape[0]
        ids = torch.empty((N, k), dtype=torch.int32, device=x.device)
        out = torch.empty((N, k), dtype=torch.float32, device=x.device)
        check(lib().hq_readout_topk(ctypes.byref(self.r), _ptr(x.contiguous()), N, k, float(beta), _ptr(ids),
                                    _ptr(out), _ptr(self.workspace), self.workspace.numel(),
                                    _stream(stream)), "hq_readout_topk")
        return ids, out


class KVCache:
    """The int4 KV cache of one attention layer (layout: include/hq.h,
    hq_kv_cache), allocated on `device` for `capacity` tokens (a multiple of
    32) of n_kv_heads heads of head_dim channels."""

    def __init__(self, n_kv_heads: int, head_dim: int, capacity: int, device):
        if capacity % 32 != 0 or capacity < 32:
            raise ValueError("capacity must be a positive multiple of 32")
        nb, d = capacity // 32, head_dim
        dev = torch.device(device)
        if dev.type != "cuda":
            raise RuntimeError("KVCache lives in CUDA device memory")
        self.n_kv_heads, self.head_dim, self.capacity = n_kv_heads, head_dim, capacity
        self.k_codes = torch.zeros((n_kv_heads, nb, 32, d // 2), dtype=torch.uint8, device=dev)
        self.k_scale = torch.zeros((n_kv_heads, nb, d), dtype=torch.float16, device=dev)
        self.k_min = torch.zeros_like(self.k_scale)
        self.v_codes = torch.zeros((n_kv_heads, nb, d, 16), dtype=torch.uint8, device=dev)
        self.v_scale = torch.zeros((n_kv_heads, capacity), dtype=torch.float16, device=dev)
        self.v_min = torch.zeros_like(self.v_scale)
        self.c = HqKvCache(head_dim, n_kv_heads, capacity, self.k_codes.data_ptr(), self.k_scale.data_ptr(),
                           self.k_min.data_ptr(), self.v_codes.data_ptr(), self.v_scale.data_ptr(),
                           self.v_min.data_ptr())
        self._ws = None

    def append(self, k: torch.Tensor, v: torch.Tensor, pos: int, stream=None) -> None:
        """Quantise k, v (fp16 [n][n_kv_heads][head_dim], n a multiple of 32)
        into positions pos .. pos + n - 1."""
        _need_cuda(k, v)
        if k.dtype != torch.float16 or v.dtype != torch.float16 or k.shape != v.shape:
            raise ValueError("k and v must be fp16 tensors of one shape")
        k, v = k.contiguous(), v.contiguous()
        check(lib().hq_kv_append(ctypes.byref(self.c), _ptr(k), _ptr(v), int(pos), int(k.shape[0]),
                                 _stream(stream)), "hq_kv_append")

    def workspace_size(self, n_tokens: int, n_q: int, n_heads: int) -> int:
        return int(lib().hq_kv_attend_workspace_size(ctypes.byref(self.c), n_tokens, n_q, n_heads))

    def attend(self, q: torch.Tensor, n_tokens: int, out=None, workspace=None, stream=None) -> torch.Tensor:
        """Attention of q (fp16 [n_q][n_heads][head_dim]) over the first
        n_tokens cached tokens; returns fp32 [n_q][n_heads][head_dim]."""
        _need_cuda(q)
        if q.dtype != torch.float16 or q.dim() != 3 or q.shape[2] != self.head_dim:
            raise ValueError("q must be fp16 [n_q][n_heads][head_dim]")
        q = q.contiguous()
        n_q, n_heads = q.shape[0], q.shape[1]
        if out is None:
            out = torch.empty((n_q, n_heads, self.head_dim), dtype=torch.float32, device=q.device)
        if workspace is None:
            need = self.workspace_size(n_tokens, max(n_q, 1), n_heads)
            if self._ws is None or self._ws.numel() < need:
                self._ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=q.device)
            workspace = self._ws
        check(lib().hq_kv_attend(ctypes.byref(self.c), int(n_tokens), _ptr(q), n_q, n_heads, _ptr(out),
                                 _ptr(workspace), workspace.numel(), _stream(stream)), "hq_kv_attend")
        return out

    def check_status(self, workspace=None, stream=None) -> None:
        """Raise HqError if an attend call on this workspace recorded a device error."""
        ws = self._ws if workspace is None else workspace
        if ws is not None:
            check(lib().hq_check_status(_ptr(ws), _stream(stream)), "hq_kv_attend status")


def hq_to_bitplanes(q2: torch.Tensor, stream=None) -> torch.Tensor:
    """Packed 2-bit codes (int32 [..][K/16]) -> the same codes in the bit-plane
    layout (same shape)."""
    _need_cuda(q2)
    if q2.dtype != torch.int32 or not q2.is_contiguous():
        raise ValueError("q2 must be a contiguous int32 tensor")
    out = torch.empty_like(q2)
    check(lib().hq_to_bitplanes(_ptr(q2), q2.numel() * 16, _ptr(out), _stream(stream)), "hq_to_bitplanes")
    return out


def hq_split_nibbles(q8: torch.Tensor, K: int, stream=None):
    """(hi, lo) int32 [rows][K/8] nibble planes of 8-bit packed codes q8 [rows][K/4]."""
    _need_cuda(q8)
    rows = q8.shape[0]
    hi = torch.empty((rows, K // 8), dtype=torch.int32, device=q8.device)
    lo = torch.empty_like(hi)
    check(lib().hq_split_nibbles(_ptr(q8), rows, K, _ptr(hi), _ptr(lo), _stream(stream)), "hq_split_nibbles")
    return hi, lo


def hq_moe_workspace_size(n_experts, hidden, inter, T, k) -> int:
    return int(lib().hq_moe_workspace_size(n_experts, hidden, inter, T, k))


def expert_table(experts: list[dict], device) -> torch.Tensor:
    """Device array of hq_expert descriptors (bytes) for a list of expert dicts
    holding CUDA tensors q_gate, q_up, q_down, s_gate, s_up, s_down, and
    optionally the expert's own rotation signs signs_in, signs_mid."""
    arr = (HqExpert * len(experts))()
    for i, e in enumerate(experts):
        own = [e.get(n) for n in ("signs_in", "signs_mid")]
        arr[i] = HqExpert(int(e["bits"]), int(e["zero"]), *[e[n].data_ptr() for n in
                          ("q_gate", "q_up", "q_down", "s_gate", "s_up", "s_down")],
                          *[None if o is None else o.data_ptr() for o in own])
    raw = bytes(memoryview(arr).cast("B"))
    return torch.frombuffer(bytearray(raw), dtype=torch.uint8).to(device)


def hq_moe_experts(table: torch.Tensor, n_experts: int, hidden: int, inter: int,
                   x: torch.Tensor, topk_ids: torch.Tensor, topk_w: torch.Tensor,
                   signs_in: torch.Tensor | None, signs_mid: torch.Tensor | None,
                   out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    _need_cuda(table, x, topk_ids, topk_w, signs_in, signs_mid)
    T, k = topk_ids.shape
    if out is None:
        out = torch.empty((T, hidden), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.zeros(max(hq_moe_workspace_size(n_experts, hidden, inter, T, k), 256),
                                dtype=torch.uint8, device=x.device)
    st = lib().hq_moe_experts(_ptr(table), n_experts, hidden, inter, _ptr(x), T, _ptr(topk_ids),
                              _ptr(topk_w), k, _ptr(signs_in), _ptr(signs_mid), _ptr(out),
                              _ptr(workspace), workspace.numel(), _stream(stream))
    check(st, "hq_moe_experts")
    return out


def hq_check_status(workspace: torch.Tensor, stream=None) -> None:
    check(lib().hq_check_status(_ptr(workspace), _stream(stream)), "device status")


def hq_unpack_codes(packed: torch.Tensor, bits: int, n_codes: int,
                    out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _need_cuda(packed)
    if out is None:
        out = torch.empty(n_codes, dtype=torch.uint8, device=packed.device)
    check(lib().hq_unpack_codes(_ptr(packed), bits, n_codes, _ptr(out), _stream(stream)),
          "hq_unpack_codes")
    return out


def hq_launch_count() -> int:
    return int(lib().hq_launch_count())


def hq_set_tc_min_batch(n: int) -> int:
    return int(lib().hq_set_tc_min_batch(n))


def hq_set_gemv32_min_batch(n: int) -> int:
    return int(lib().hq_set_gemv32_min_batch(n))


__all__ = ["hq_to_bitplanes", "KVCache", "ScreenedReadout", "hq_split_nibbles", "hq_quantize", "hq_rotate", "hq_linear", "hq_linear_noalloc", "hq_linear_noalloc_check_status", "hq_linear_workspace_size", "RotatedLinear",
           "hq_moe_experts", "hq_moe_workspace_size", "expert_table", "hq_check_status",
           "hq_unpack_codes", "hq_launch_count", "hq_set_tc_min_batch", "hq_set_gemv32_min_batch", "HqError", "make_weight"]
