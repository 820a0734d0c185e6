"""GPU parity of the tensor-core (tcgen05) path of hq_linear against the oracle.

hq_linear sends batches of at least the tensor-core threshold (9 by default)
with K >= 1024 to the tcgen05 GEMM.  These cases check it element by element
against the fp64 oracle with the same tolerance as the GEMV path,
|y - y_oracle| <= 2e-3 sum_k |w_k x'_k| + 1e-5, over ragged row counts (partial
128-row tiles), ragged batches (column blocks padded to 32), several column
blocks per call, several tiles per CTA, every code width, null signs and
non-default zero points.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_hadamard_rotated_b200 import synth

pytestmark = pytest.mark.gpu

REL, ABS = 2e-3, 1e-5


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_hadamard_rotated_b200 import build
    build.build()
    import bit_hadamard_rotated_b200._lib as L
    L.lib()
    # batches 9..16 (5..16 for 3/4/8-bit rows at K >= 8192) go to the 32-row
    # GEMV by default; this module checks the tensor-core GEMM at those sizes too
    from bit_hadamard_rotated_b200 import hq_set_gemv32_min_batch
    old = hq_set_gemv32_min_batch(1 << 20)
    yield torch.device("cuda:0")
    hq_set_gemv32_min_batch(old)


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def assert_within(y, want, bound, what=""):
    err = np.abs(y.astype(np.float64) - want)
    lim = REL * bound + ABS
    bad = err > lim
    if bad.any():
        i = np.unravel_index(np.argmax(err / lim), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {err.size} outside tolerance; worst at {i}: "
                             f"got {y[i]!r} want {want[i]!r} err {err[i]:.3e} lim {lim[i]:.3e}")


def weight(d):
    from bit_hadamard_rotated_b200 import make_weight
    q, s, g = dev(d["q"].view(np.int32)), dev(d["scales"]), dev(d["signs"])
    return q, s, g, make_weight(q, s, g, d["bits"], d["zero"])


def run(d, signs=True):
    from bit_hadamard_rotated_b200 import hq_launch_count, hq_linear
    from bit_hadamard_rotated_b200._lib import lib
    import ctypes
    q, s, g, w = weight(d)
    if not signs:
        g = None
        w.signs = None
    expect = int(lib().hq_linear_launches(ctypes.byref(w), d["N"]))
    x = dev(d["x"])
    torch.cuda.synchronize()
    n0 = hq_launch_count()
    y = hq_linear(q, s, g, x, d["bits"], d["zero"])
    torch.cuda.synchronize()
    return y.cpu().numpy(), hq_launch_count() - n0, expect


def tc_blocks(bits, K, N):
    """Expected tensor-core launches: the prep kernel plus one GEMM per batch block."""
    # mirror of the shared-memory plan: at least 4 ring slots of [128 code rows]
    # [x' image], two tile scale buffers, 320 B of barriers, 1 KiB alignment
    # pad; blocks shrink from 128 columns in steps of 32 until the plan fits
    G = K // 128
    per = 128
    while per >= 32:
        smem = 4 * (128 * 16 * bits + 256 * per) + 2 * 128 * G * 2 + 320 + 1024
        if smem <= 227 * 1024 - 1024:
            break
        per -= 32
    return 1 + (N + per - 1) // per


CASES = [
    # (M, K, N): ragged tiles, ragged batches, several blocks and tiles per CTA
    (128, 1024, 9), (1, 1024, 16), (129, 1024, 31), (300, 2048, 33), (77, 4096, 64),
    (256, 8192, 100), (200, 16384, 128), (130, 1024, 129), (64, 2048, 200),
    (20000, 1024, 24), (19100, 1024, 140),
]


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("M,K,N", CASES)
def test_tc_linear_parity(bits, M, K, N):
    d = synth.linear(M, K, bits, N, seed=11 * M + K + 3 * N + bits)
    y, launches, expect = run(d)
    assert launches == expect == tc_blocks(bits, K, N), (launches, expect)
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert_within(y, want, bound, what=f"tc b{bits} M{M} K{K} N{N}")


@pytest.mark.parametrize("bits,N", [(3, 5), (4, 6), (8, 8), (2, 8), (4, 4), (2, 5), (2, 12), (8, 16), (3, 17)])
def test_small_batches_at_large_k_either_path(bits, N):
    """The automatic switch at K = 8192 (300 rows): batches from 4 of 8-bit,
    5 of 3/4-bit and 6 of 2-bit codes take the 32-row GEMV up to batch 16, the
    tensor-core GEMM beyond, smaller batches the GEMV; all match the oracle."""
    import ctypes
    from bit_hadamard_rotated_b200 import hq_set_gemv32_min_batch
    from bit_hadamard_rotated_b200._lib import HQ_PATH_GEMV, HQ_PATH_GEMV32, HQ_PATH_TENSOR, lib
    M, K = 300, 8192
    d = synth.linear(M, K, bits, N, seed=31 + bits + N)
    _, _, _, w = weight(d)
    want_path = (HQ_PATH_TENSOR if N > 16 else
                 HQ_PATH_GEMV32 if N >= {2: 6, 3: 5, 4: 5, 8: 4}[bits] else HQ_PATH_GEMV)
    old = hq_set_gemv32_min_batch(0)
    try:
        assert lib().hq_linear_path(ctypes.byref(w), N) == want_path
        assert lib().hq_linear_uses_tensor_cores(ctypes.byref(w), N) == (1 if want_path == HQ_PATH_TENSOR else 0)
        y, launches, expect = run(d)
    finally:
        hq_set_gemv32_min_batch(old)
    assert launches == expect
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert_within(y, want, bound, what=f"b{bits} N{N} K{K}")


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_tc_nondefault_zero_null_signs_loguniform(bits):
    M, K, N = 200, 2048, 40
    d = synth.linear(M, K, bits, N, seed=99 + bits, scale_dist="loguniform", outlier_frac=0.01)
    d["zero"] = (1 << bits) - 1 if bits < 8 else 3
    y, _, _ = run(d, signs=False)
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], None, d["x"])
    assert_within(y, want, bound, what=f"tc zero/null-signs b{bits}")


def test_tc_matches_gemv_and_is_deterministic():
    from bit_hadamard_rotated_b200 import hq_linear, hq_set_tc_min_batch
    M, K, N, bits = 1000, 4096, 48, 3
    d = synth.linear(M, K, bits, N, seed=5)
    q, s, g, _ = weight(d)
    x = dev(d["x"])
    y1 = hq_linear(q, s, g, x, bits, d["zero"])
    y2 = hq_linear(q, s, g, x, bits, d["zero"])
    assert torch.equal(y1, y2)
    old = hq_set_tc_min_batch(1 << 20)
    try:
        yg = hq_linear(q, s, g, x, bits, d["zero"])
    finally:
        hq_set_tc_min_batch(old)
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert_within(y1.cpu().numpy(), want, bound, what="tc")
    assert_within(yg.cpu().numpy(), want, bound, what="gemv")


def test_tc_tiles_shared_between_ctas_deterministic():
    """More 128-row tiles than CTAs: CTAs own equal chunk ranges, so tiles are
    cut between two CTAs and finished by the second to arrive.  Repeat calls on
    one workspace are bit-identical and leave the tile counters (the 1 KiB after
    the status word) at zero."""
    from bit_hadamard_rotated_b200 import hq
    M, K, N, bits = 24000, 4096, 64, 2
    d = synth.linear(M, K, bits, N, seed=17)
    q, s, g, w = weight(d)
    x = dev(d["x"])
    ws = torch.zeros(hq.hq_linear_workspace_size(w, N), dtype=torch.uint8, device="cuda")
    y1 = hq.hq_linear(q, s, g, x, bits, d["zero"], workspace=ws)
    y2 = hq.hq_linear(q, s, g, x, bits, d["zero"], workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert int(ws[256:1280].count_nonzero()) == 0
    rows = np.r_[0:64, 12000:12300, M - 64:M]
    want, bound = oracle.linear(bits, len(rows), K, d["zero"], d["q"][rows], d["scales"][rows],
                                d["signs"], d["x"])
    assert_within(y1.cpu().numpy()[:, rows], want, bound, what="stream-K rows")


def test_tc_output_overwritten_and_status_clean():
    from bit_hadamard_rotated_b200 import RotatedLinear
    M, K, N, bits = 300, 1024, 20, 2
    d = synth.linear(M, K, bits, N, seed=8)
    q, s, g, _ = weight(d)
    lin = RotatedLinear(q, s, g, bits, d["zero"], max_batch=N)
    out = torch.full((N, M), float("nan"), device="cuda")
    lin(dev(d["x"]), out=out)
    lin.check_status()
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert_within(out.cpu().numpy(), want, bound, what="overwrite")


def test_tc_workspace_too_small_is_rejected():
    from bit_hadamard_rotated_b200 import HqError, hq_linear, hq_linear_workspace_size
    M, K, N, bits = 256, 2048, 64, 4
    d = synth.linear(M, K, bits, N, seed=3)
    q, s, g, w = weight(d)
    small = hq_linear_workspace_size(w, 8)
    big = hq_linear_workspace_size(w, N)
    assert big >= small + N * K * 2
    ws = torch.zeros(small, dtype=torch.uint8, device="cuda")
    with pytest.raises(HqError):
        hq_linear(q, s, g, dev(d["x"]), bits, d["zero"], workspace=ws)


@pytest.mark.parametrize("bits,M,K,N", [(3, 8192, 2048, 32), (2, 8192, 8192, 32), (8, 4096, 4096, 64),
                                        (4, 8192, 1024, 128)])
def test_tc_every_output_finite_over_repeated_calls(bits, M, K, N):
    """Many tiles, every call on a fresh zeroed workspace: each tile's scales must
    have landed before any warpgroup reads them (a stale scale shows as a
    non-finite or wrong row), on every call."""
    from bit_hadamard_rotated_b200 import hq_linear, hq_linear_workspace_size
    d = synth.linear(M, K, bits, N, seed=17 + bits)
    q, s, g, w = weight(d)
    x = dev(d["x"])
    rng = np.random.default_rng(M + K)
    rows = sorted(set(rng.choice(M, 12, replace=False).tolist()) | {0, M - 1})
    want = {}
    for m in rows:
        want[m] = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"],
                                m_begin=m, m_end=m + 1)
    for _ in range(4):
        ws = torch.zeros(hq_linear_workspace_size(w, N), dtype=torch.uint8, device="cuda")
        y = hq_linear(q, s, g, x, bits, d["zero"], workspace=ws).cpu().numpy()
        assert np.all(np.isfinite(y))
        for m in rows:
            assert_within(y[:, m], want[m][0][:, m], want[m][1][:, m], what=f"row {m}")
