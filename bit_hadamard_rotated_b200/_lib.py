"""ctypes binding to libhq.so: argument marshalling only.

Every step of the computation runs in the CUDA kernels behind the C ABI
(include/hq.h).  Tensors are PyTorch CUDA tensors; PyTorch supplies device
memory and the current stream.  There is no CPU or PyTorch fallback: if the
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhq.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "hq.h")

HQ_OK, HQ_ERR_INVALID_ARG, HQ_ERR_UNSUPPORTED, HQ_ERR_WORKSPACE, HQ_ERR_CUDA, HQ_ERR_DATA, \
    HQ_ERR_TIMEOUT = range(7)
HQ_F16, HQ_BF16, HQ_F32 = 0, 1, 2
HQ_MOE_POS, HQ_MOE_H, HQ_MOE_D = 0, 1, 2
HQ_LAYOUT_PACKED, HQ_LAYOUT_BITPLANES = 0, 1
HQ_PATH_GEMV, HQ_PATH_TENSOR, HQ_PATH_GEMV32 = 0, 1, 2

_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t


class HqWeight(ctypes.Structure):
    _fields_ = [("bits", _i), ("M", _i), ("K", _i), ("zero", _i),
                ("qweight", _vp), ("scales", _vp), ("signs", _vp), ("zeros", _vp), ("layout", _i)]


class HqExpert(ctypes.Structure):
    _fields_ = [("bits", _i), ("zero", _i), ("q_gate", _vp), ("q_up", _vp), ("q_down", _vp),
                ("s_gate", _vp), ("s_up", _vp), ("s_down", _vp), ("signs_in", _vp), ("signs_mid", _vp)]


class HqReadout(ctypes.Structure):
    _fields_ = [("V", _i), ("K", _i), ("zero", _i), ("hi", _vp), ("lo", _vp), ("scales", _vp),
                ("signs", _vp)]


class HqKvCache(ctypes.Structure):
    _fields_ = [("head_dim", _i), ("n_kv_heads", _i), ("capacity", _i), ("k_codes", _vp), ("k_scale", _vp),
                ("k_min", _vp), ("v_codes", _vp), ("v_scale", _vp), ("v_min", _vp)]


class HqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libhq.so (built in-tree by bit_hadamard_rotated_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m bit_hadamard_rotated_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.hq_rotate.argtypes = [_vp, _i, _vp, _i, _i, _i, _vp, _vp]
        L.hq_rotate.restype = _i
        L.hq_linear_workspace_size.argtypes = [ctypes.POINTER(HqWeight), _i]
        L.hq_linear_workspace_size.restype = _sz
        L.hq_linear.argtypes = [ctypes.POINTER(HqWeight), _vp, _i, _vp, _vp, _sz, _vp]
        L.hq_linear.restype = _i
        L.hq_moe_workspace_size.argtypes = [_i, _i, _i, _i, _i]
        L.hq_moe_workspace_size.restype = _sz
        L.hq_moe_experts.argtypes = [_vp, _i, _i, _i, _vp, _i, _vp, _vp, _i, _vp, _vp, _vp,
                                     _vp, _sz, _vp]
        L.hq_moe_experts.restype = _i
        L.hq_check_status.argtypes = [_vp, _vp]
        L.hq_check_status.restype = _i
        L.hq_unpack_codes.argtypes = [_vp, _i, _sz, _vp, _vp]
        L.hq_unpack_codes.restype = _i
        L.hq_status_string.argtypes = [_i]
        L.hq_status_string.restype = ctypes.c_char_p
        L.hq_launch_count.argtypes = []
        L.hq_launch_count.restype = ctypes.c_uint64
        L.hq_linear_launches.argtypes = [ctypes.POINTER(HqWeight), _i]
        L.hq_linear_launches.restype = _i
        L.hq_linear_uses_tensor_cores.argtypes = [ctypes.POINTER(HqWeight), _i]
        L.hq_linear_uses_tensor_cores.restype = _i
        L.hq_linear_noalloc.argtypes = [ctypes.POINTER(HqWeight), _vp, _i, _vp, _vp]
        L.hq_linear_noalloc.restype = _i
        L.hq_linear_noalloc_check_status.argtypes = [_vp]
        L.hq_linear_noalloc_check_status.restype = _i
        L.hq_readout_workspace_size.argtypes = [ctypes.POINTER(HqReadout), _i]
        L.hq_readout_workspace_size.restype = _sz
        L.hq_readout_topk.argtypes = [ctypes.POINTER(HqReadout), _vp, _i, _i, ctypes.c_float, _vp, _vp,
                                      _vp, _sz, _vp]
        L.hq_readout_topk.restype = _i
        L.hq_split_nibbles.argtypes = [_vp, _i, _i, _vp, _vp, _vp]
        L.hq_to_bitplanes.argtypes = [_vp, _sz, _vp, _vp]
        L.hq_to_bitplanes.restype = _i
        L.hq_kv_append.argtypes = [ctypes.POINTER(HqKvCache), _vp, _vp, _i, _i, _vp]
        L.hq_kv_append.restype = _i
        L.hq_kv_attend_workspace_size.argtypes = [ctypes.POINTER(HqKvCache), _i, _i, _i]
        L.hq_kv_attend_workspace_size.restype = _sz
        L.hq_kv_attend.argtypes = [ctypes.POINTER(HqKvCache), _i, _vp, _i, _i, _vp, _vp, _sz, _vp]
        L.hq_kv_attend.restype = _i
        L.hq_kv_attend_launches.argtypes = []
        L.hq_kv_attend_launches.restype = _i
        L.hq_split_nibbles.restype = _i
        L.hq_quantize.argtypes = [_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp]
        L.hq_quantize.restype = _i
        L.hq_moe_workspace_offset.argtypes = [_i, _i, _i, _i, _i, _i]
        L.hq_moe_workspace_offset.restype = _sz
        L.hq_moe_launches.argtypes = []
        L.hq_moe_launches.restype = _i
        L.hq_set_test_fault.argtypes = [_i]
        L.hq_set_test_fault.restype = _i
        L.hq_set_tc_min_batch.argtypes = [_i]
        L.hq_set_tc_min_batch.restype = _i
        L.hq_set_gemv32_min_batch.argtypes = [_i]
        L.hq_set_gemv32_min_batch.restype = _i
        L.hq_linear_path.argtypes = [ctypes.POINTER(HqWeight), _i]
        L.hq_linear_path.restype = _i
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/hq.h declares."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hq_[a-z0-9_]+)\s*\(", src)))


def status_string(s: int) -> str:
    return lib().hq_status_string(int(s)).decode()


def check(status: int, what: str) -> None:
    if status != HQ_OK:
        raise HqError(status, what)
