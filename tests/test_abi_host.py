"""Host-only checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments on the host before launching
anything (these calls never reach the GPU, so they run on a CPU-only box)."""
import ctypes

import pytest

from bit_hadamard_rotated_b200 import _lib
from bit_hadamard_rotated_b200._lib import (HQ_ERR_INVALID_ARG, HQ_ERR_UNSUPPORTED,
                                            HQ_ERR_WORKSPACE, HQ_OK, HqWeight)

FAKE = 0x100000  # aligned, never dereferenced: every call below fails validation first


@pytest.fixture(scope="module")
def L():
    from bit_hadamard_rotated_b200 import build
    build.build()
    return _lib.lib()


def test_exports_every_declared_function(L):
    names = _lib.header_functions()
    assert {"hq_rotate", "hq_linear", "hq_moe_experts", "hq_unpack_codes",
            "hq_check_status", "hq_linear_workspace_size", "hq_moe_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for s in range(7):
        assert _lib.status_string(s).startswith("HQ_")


def W(**kw):
    d = dict(bits=4, M=64, K=4096, zero=8, qweight=FAKE, scales=FAKE, signs=None, zeros=None, layout=0)
    d.update(kw)
    return HqWeight(d["bits"], d["M"], d["K"], d["zero"], d["qweight"], d["scales"], d["signs"], d["zeros"],
                    d["layout"])


def lin(L, w, batch=1, x=FAKE, y=FAKE, ws=FAKE, ws_bytes=1 << 30):
    return L.hq_linear(None if w is None else ctypes.byref(w), x, batch, y, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,want", [
    (dict(bits=5), HQ_ERR_UNSUPPORTED), (dict(bits=0), HQ_ERR_INVALID_ARG),
    (dict(bits=9), HQ_ERR_INVALID_ARG), (dict(K=4096 + 128), HQ_ERR_UNSUPPORTED),
    (dict(K=64), HQ_ERR_UNSUPPORTED), (dict(K=65536), HQ_ERR_UNSUPPORTED),
    (dict(K=0), HQ_ERR_INVALID_ARG), (dict(M=0), HQ_ERR_INVALID_ARG),
    (dict(zero=16), HQ_ERR_INVALID_ARG), (dict(zero=-1), HQ_ERR_INVALID_ARG),
    (dict(qweight=FAKE + 8), HQ_ERR_INVALID_ARG), (dict(scales=FAKE + 2), HQ_ERR_INVALID_ARG),
    (dict(signs=FAKE + 1), HQ_ERR_INVALID_ARG), (dict(qweight=None), HQ_ERR_INVALID_ARG),
    (dict(layout=1), HQ_ERR_UNSUPPORTED), (dict(layout=2), HQ_ERR_INVALID_ARG),
    (dict(bits=2, zero=2, layout=-1), HQ_ERR_INVALID_ARG), (dict(zeros=FAKE + 4), HQ_ERR_INVALID_ARG),
])
def test_linear_rejects_bad_weight(L, kw, want):
    before = L.hq_launch_count()
    assert lin(L, W(**kw)) == want
    assert L.hq_launch_count() == before


def test_linear_rejects_bad_call_args(L):
    before = L.hq_launch_count()
    w = W()
    assert lin(L, None) == HQ_ERR_INVALID_ARG
    assert lin(L, w, batch=-1) == HQ_ERR_INVALID_ARG
    assert lin(L, w, batch=0) == HQ_OK                     # nothing to do, nothing launched
    assert lin(L, w, x=None) == HQ_ERR_INVALID_ARG
    assert lin(L, w, x=FAKE + 2) == HQ_ERR_INVALID_ARG
    assert lin(L, w, y=FAKE + 4) == HQ_ERR_INVALID_ARG
    assert lin(L, w, ws=None) == HQ_ERR_WORKSPACE
    assert lin(L, w, ws=FAKE + 16) == HQ_ERR_WORKSPACE     # needs 256-byte alignment
    need = L.hq_linear_workspace_size(ctypes.byref(w), 1)
    assert need > 0
    assert lin(L, w, ws_bytes=need - 1) == HQ_ERR_WORKSPACE
    assert L.hq_launch_count() == before


def test_workspace_size_queries(L):
    assert L.hq_linear_workspace_size(ctypes.byref(W(bits=7)), 1) == 0
    assert L.hq_linear_workspace_size(ctypes.byref(W()), -1) == 0
    # status word + one batch block of rotated activations (GEMV), or the
    # batch's activation images (tensor-core path): independent of M
    a = L.hq_linear_workspace_size(ctypes.byref(W(M=64)), 1)
    b = L.hq_linear_workspace_size(ctypes.byref(W(M=65536)), 1)
    assert 0 < a == b and a % 256 == 0
    # G x nb x 320 B of B fragments + G x 8 x 4 B of zero-point terms
    G = 4096 // 128
    assert a >= 256 + G * 1 * 320 + G * 32
    k2 = L.hq_linear_workspace_size(ctypes.byref(W(K=8192)), 1)
    assert k2 > a
    big = L.hq_linear_workspace_size(ctypes.byref(W(K=4096)), 64)
    assert big >= 256 + 64 * 4096 * 2          # tensor-core path: batch x K fp16


def test_rotate_rejects_bad_args(L):
    before = L.hq_launch_count()
    r = lambda **kw: L.hq_rotate(kw.get("x", FAKE), kw.get("xd", 0), kw.get("o", FAKE),
                                 kw.get("od", 2), kw.get("n", 1), kw.get("K", 1024),
                                 kw.get("s", None), None)
    assert r(K=100) == HQ_ERR_UNSUPPORTED
    assert r(K=16) == HQ_ERR_UNSUPPORTED
    assert r(K=65536) == HQ_ERR_UNSUPPORTED
    assert r(K=0) == HQ_ERR_INVALID_ARG
    assert r(n=-1) == HQ_ERR_INVALID_ARG
    assert r(n=0) == HQ_OK
    assert r(xd=7) == HQ_ERR_INVALID_ARG
    assert r(od=-1) == HQ_ERR_INVALID_ARG
    assert r(x=None) == HQ_ERR_INVALID_ARG
    assert r(x=FAKE + 2) == HQ_ERR_INVALID_ARG
    assert r(s=FAKE + 3) == HQ_ERR_INVALID_ARG
    assert L.hq_launch_count() == before


def test_unpack_rejects_bad_args(L):
    before = L.hq_launch_count()
    assert L.hq_unpack_codes(FAKE, 0, 10, FAKE, None) == HQ_ERR_INVALID_ARG
    assert L.hq_unpack_codes(FAKE, 9, 10, FAKE, None) == HQ_ERR_INVALID_ARG
    assert L.hq_unpack_codes(FAKE, 3, 0, FAKE, None) == HQ_OK
    assert L.hq_unpack_codes(FAKE + 2, 3, 10, FAKE, None) == HQ_ERR_INVALID_ARG
    assert L.hq_unpack_codes(None, 3, 10, FAKE, None) == HQ_ERR_INVALID_ARG
    assert L.hq_launch_count() == before


def moe_call(L, **kw):
    a = dict(ex=FAKE, E=8, hidden=256, inter=128, x=FAKE, T=4, ids=FAKE, w=FAKE, k=2,
             si=None, sm=None, y=FAKE, ws=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    return L.hq_moe_experts(a["ex"], a["E"], a["hidden"], a["inter"], a["x"], a["T"], a["ids"],
                            a["w"], a["k"], a["si"], a["sm"], a["y"], a["ws"], a["ws_bytes"], None)


def test_moe_rejects_bad_args(L):
    before = L.hq_launch_count()
    assert moe_call(L, E=0) == HQ_ERR_INVALID_ARG
    assert moe_call(L, k=0) == HQ_ERR_INVALID_ARG
    assert moe_call(L, k=33) == HQ_ERR_INVALID_ARG
    assert moe_call(L, T=-1) == HQ_ERR_INVALID_ARG
    assert moe_call(L, hidden=384) == HQ_ERR_UNSUPPORTED
    assert moe_call(L, inter=64) == HQ_ERR_UNSUPPORTED
    assert moe_call(L, T=0) == HQ_OK
    assert moe_call(L, x=None) == HQ_ERR_INVALID_ARG
    assert moe_call(L, x=FAKE + 8) == HQ_ERR_INVALID_ARG
    assert moe_call(L, ex=FAKE + 4) == HQ_ERR_INVALID_ARG
    assert moe_call(L, si=FAKE + 1) == HQ_ERR_INVALID_ARG
    assert moe_call(L, ws=None) == HQ_ERR_WORKSPACE
    need = L.hq_moe_workspace_size(8, 256, 128, 4, 2)
    assert need > 0 and need % 256 == 0
    assert moe_call(L, ws_bytes=need - 1) == HQ_ERR_WORKSPACE
    assert L.hq_moe_workspace_size(0, 256, 128, 4, 2) == 0
    assert L.hq_moe_launches() == 5
    assert L.hq_launch_count() == before


def test_tc_min_batch_override_and_automatic_default():
    from bit_hadamard_rotated_b200._lib import lib
    L = lib()
    old = L.hq_set_tc_min_batch(-1)  # negative: read only
    assert old == 0                 # automatic by default
    assert L.hq_set_tc_min_batch(7) == 0
    assert L.hq_set_tc_min_batch(-5) == 7
    assert L.hq_set_tc_min_batch(0) == 7
    assert L.hq_set_tc_min_batch(-1) == 0


def test_linear_path_choice():
    """The automatic GEMV / tensor-core switch (host only: nothing is launched)."""
    from bit_hadamard_rotated_b200._lib import lib
    L = lib()

    from bit_hadamard_rotated_b200._lib import HQ_PATH_GEMV, HQ_PATH_GEMV32, HQ_PATH_TENSOR

    def weight(bits, K, M=256):
        return HqWeight(bits, M, K, 1 << (bits - 1), FAKE, FAKE, None)

    def tc(bits, K, batch, M=256):
        return L.hq_linear_uses_tensor_cores(ctypes.byref(weight(bits, K, M)), batch)

    def path(bits, K, batch, M=256):
        return L.hq_linear_path(ctypes.byref(weight(bits, K, M)), batch)

    G, T, G32 = HQ_PATH_GEMV, HQ_PATH_TENSOR, HQ_PATH_GEMV32
    # the 32-row GEMV from batch 4 (8-bit), 5 (3/4-bit), 6 (2-bit; 9 above
    # 16384 rows) up to 16, the tensor cores beyond
    assert path(3, 8192, 4) == G and path(3, 8192, 5) == G32 and path(3, 8192, 16) == G32
    assert path(3, 8192, 17) == T and tc(3, 8192, 17) == 1 and tc(3, 8192, 5) == 0
    assert path(8, 4096, 3) == G and path(8, 4096, 4) == G32 and path(8, 16384, 5) == G32
    assert path(4, 4096, 4) == G and path(4, 4096, 5) == G32 and path(4, 4096, 9) == G32
    assert path(2, 8192, 5) == G and path(2, 8192, 6) == G32 and path(2, 8192, 64) == T
    assert path(2, 8192, 8, M=28672) == G and path(2, 8192, 9, M=28672) == G32
    assert path(4, 512, 64) == G and path(4, 512, 12) == G   # K < 1024: GEMV at every batch
    # where the 32-row GEMV does not apply (per-group zeros, K < 1024) the
    # tensor cores keep their own thresholds
    # at most 16 tiles of 32 rows per CTA: beyond 16 x 32 x SMs rows the tensor cores
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148
    assert path(2, 4096, 12, M=16 * 32 * sms) == G32 and path(2, 4096, 12, M=16 * 32 * sms + 1) == T
    assert path(4, 4096, 0) == -1 and path(5, 4096, 4) == -1 and tc(4, 4096, 0) == -1
    # launches: the rotation inside the 32-row GEMV when every batch row has a
    # CTA (8 tiles of 32 rows < 12 rows: a prep kernel first)
    assert L.hq_linear_launches(ctypes.byref(weight(2, 8192)), 12) == 2
    assert L.hq_linear_launches(ctypes.byref(weight(2, 8192, M=1024)), 12) == 1
    assert L.hq_linear_launches(ctypes.byref(weight(2, 16384, M=1024)), 12) == 2
    # overrides: an explicit tensor-core threshold wins; the 32-row GEMV from batch 1
    assert L.hq_set_gemv32_min_batch(-1) == 0
    old = L.hq_set_gemv32_min_batch(1)
    try:
        assert path(2, 8192, 1) == G32 and path(2, 4096, 16) == G32 and path(2, 4096, 17) == T
        prev = L.hq_set_tc_min_batch(9)
        try:
            assert path(2, 8192, 8) == G32 and path(2, 8192, 9) == T
        finally:
            L.hq_set_tc_min_batch(prev)
    finally:
        L.hq_set_gemv32_min_batch(old)
    assert L.hq_set_gemv32_min_batch(-1) == 0


def test_moe_workspace_offsets(L):
    """The stage intermediates lie inside the workspace, 256-byte aligned, in
    the order pos < h < d; a bad argument or part gives SIZE_MAX."""
    from bit_hadamard_rotated_b200._lib import HQ_MOE_D, HQ_MOE_H, HQ_MOE_POS
    E, H, I, T, k = 256, 2048, 512, 32, 8
    size = L.hq_moe_workspace_size(E, H, I, T, k)
    pos, h, d = (L.hq_moe_workspace_offset(E, H, I, T, k, p) for p in (HQ_MOE_POS, HQ_MOE_H, HQ_MOE_D))
    assert pos % 256 == 0 and h % 256 == 0 and d % 256 == 0
    assert pos + 4 * T * k <= h and h + 4 * T * k * I <= d and d + 4 * T * k * H <= size
    none = ctypes.c_size_t(-1).value
    assert L.hq_moe_workspace_offset(E, H + 1, I, T, k, HQ_MOE_H) == none
    assert L.hq_moe_workspace_offset(E, H, I, T, k, 7) == none


def test_kv_cache_rejects_bad_args(L):
    """hq_kv_append / hq_kv_attend validate the cache and the call on the host."""
    from bit_hadamard_rotated_b200._lib import HqKvCache

    def cache(d=128, n_kv=4, cap=1024, kc=FAKE, vs=FAKE):
        return HqKvCache(d, n_kv, cap, kc, FAKE, FAKE, FAKE, vs, FAKE)

    c = cache()
    ws = L.hq_kv_attend_workspace_size(ctypes.byref(c), 1000, 32, 16)
    # 1000 tokens = 8 steps of 128, one per chunk (37 chunks per kv head would
    # fill the SMs); a 256-byte status word, then per chunk 128 rows x
    # (128 + 4) floats, for 4 kv heads
    assert ws == 256 + 4 * 4 * 8 * 128 * 132
    assert L.hq_kv_attend_workspace_size(ctypes.byref(c), 1025, 32, 16) == 0     # past capacity
    assert L.hq_kv_attend_workspace_size(ctypes.byref(c), 1000, 32, 6) == 0      # heads not a multiple
    assert L.hq_kv_attend_workspace_size(ctypes.byref(cache(d=96)), 1000, 32, 16) == 0
    assert L.hq_kv_attend_launches() == 2
    # append: whole blocks inside the capacity, supported head_dim, aligned arrays
    assert L.hq_kv_append(ctypes.byref(cache(d=96)), FAKE, FAKE, 0, 32, None) == HQ_ERR_UNSUPPORTED
    assert L.hq_kv_append(ctypes.byref(c), FAKE, FAKE, 16, 32, None) == HQ_ERR_INVALID_ARG
    assert L.hq_kv_append(ctypes.byref(c), FAKE, FAKE, 0, 48, None) == HQ_ERR_INVALID_ARG
    assert L.hq_kv_append(ctypes.byref(c), FAKE, FAKE, 1024, 32, None) == HQ_ERR_INVALID_ARG
    assert L.hq_kv_append(ctypes.byref(cache(cap=1000)), FAKE, FAKE, 0, 32, None) == HQ_ERR_INVALID_ARG
    assert L.hq_kv_append(ctypes.byref(cache(kc=FAKE + 8)), FAKE, FAKE, 0, 32, None) == HQ_ERR_INVALID_ARG
    assert L.hq_kv_append(ctypes.byref(c), None, FAKE, 0, 32, None) == HQ_ERR_INVALID_ARG
    assert L.hq_kv_append(ctypes.byref(c), FAKE, FAKE, 0, 0, None) == HQ_OK          # nothing to do
    assert L.hq_kv_append(None, FAKE, FAKE, 0, 32, None) == HQ_ERR_INVALID_ARG
    # attend
    att = L.hq_kv_attend
    assert att(ctypes.byref(c), 1000, FAKE, 0, 16, FAKE, FAKE, 1 << 30, None) == HQ_OK  # n_q = 0
    assert att(ctypes.byref(c), 0, FAKE, 32, 16, FAKE, FAKE, 1 << 30, None) == HQ_ERR_INVALID_ARG
    assert att(ctypes.byref(c), 1025, FAKE, 32, 16, FAKE, FAKE, 1 << 30, None) == HQ_ERR_INVALID_ARG
    assert att(ctypes.byref(c), 1000, FAKE, 32, 15, FAKE, FAKE, 1 << 30, None) == HQ_ERR_INVALID_ARG
    assert att(ctypes.byref(c), 1000, FAKE + 2, 32, 16, FAKE, FAKE, 1 << 30, None) == HQ_ERR_INVALID_ARG
    assert att(ctypes.byref(c), 1000, FAKE, 32, 16, FAKE, FAKE, ws - 1, None) == HQ_ERR_WORKSPACE
    assert att(ctypes.byref(c), 1000, FAKE, 32, 16, FAKE, FAKE + 16, ws, None) == HQ_ERR_WORKSPACE
    assert att(ctypes.byref(c), 1000, FAKE, 1025, 16, FAKE, FAKE, 1 << 30, None) == HQ_ERR_UNSUPPORTED


def test_to_bitplanes_rejects_bad_args(L):
    before = L.hq_launch_count()
    assert L.hq_to_bitplanes(FAKE, 48, FAKE, None) == HQ_ERR_INVALID_ARG       # not whole 32-code spans
    assert L.hq_to_bitplanes(FAKE + 4, 64, FAKE, None) == HQ_ERR_INVALID_ARG   # misaligned
    assert L.hq_to_bitplanes(None, 64, FAKE, None) == HQ_ERR_INVALID_ARG
    assert L.hq_to_bitplanes(FAKE, 0, FAKE, None) == HQ_OK                      # nothing to do
    assert L.hq_launch_count() == before
    # the bit-plane layout is accepted for 2-bit weights (fails later, on the fake workspace size)
    assert lin(L, W(bits=2, zero=2, layout=1), ws_bytes=0) == HQ_ERR_WORKSPACE


def test_linear_workspace_grows_with_batch():
    """A workspace sized for a batch serves every smaller batch (RotatedLinear
    sizes one for its max_batch): hq_linear_workspace_size never shrinks as the
    batch grows, across the GEMV, 32-row GEMV and tensor-core paths."""
    from bit_hadamard_rotated_b200._lib import lib
    L = lib()
    for bits in (2, 3, 4, 8):
        for K in (128, 1024, 8192, 32768):
            for M in (16, 4096, 28672, 100000):
                w = HqWeight(bits, M, K, 1 << (bits - 1), FAKE, FAKE, None)
                sizes = [L.hq_linear_workspace_size(ctypes.byref(w), b) for b in range(1, 130)]
                assert all(s > 0 for s in sizes)
                assert all(b >= a for a, b in zip(sizes, sizes[1:])), (bits, K, M)
