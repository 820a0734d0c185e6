"""GPU parity of the 32-row GEMV (hq_linear's path for batches up to 16)
against the fp64 oracle, |y - y_oracle| <= 2e-3 sum_k |w_k x'_k| + 1e-5.

The kernel walks K in slices of 8 or 16 groups with two slice buffers, splits
each slice's (32-row tile, group) units between 16 warps in the same ranges,
and adds tiles split between warps in warp order at the end.  The cases cover
one and two 8-column blocks (batch 1..16, ragged), one slice (K = 1024) and
many (K = 32768), ragged row counts and uneven tiles per CTA, the largest row
count one launch takes (16 tiles per CTA), every code width, bit-plane codes,
null signs, non-default zero points and small activations.
"""
import ctypes

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
    return torch.device("cuda:0")


@pytest.fixture
def from_batch_1():
    """The 32-row GEMV for every batch up to 16 (one 8-column block below 9)."""
    from bit_hadamard_rotated_b200 import hq_set_gemv32_min_batch
    old = hq_set_gemv32_min_batch(1)
    yield
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


def run(d, signs=True, planes=False):
    """hq_linear on d through the C ABI; checks that the 32-row GEMV ran (path
    and launch count) and returns y."""
    from bit_hadamard_rotated_b200 import hq_launch_count, hq_linear, hq_to_bitplanes, make_weight
    from bit_hadamard_rotated_b200._lib import HQ_PATH_GEMV32, lib
    q = dev(d["q"].view(np.int32))
    if planes:
        q = hq_to_bitplanes(q)
    s, g = dev(d["scales"]), (dev(d["signs"]) if signs else None)
    w = make_weight(q, s, g, d["bits"], d["zero"], planes=planes)
    N = d["x"].shape[0]
    M, K = d["q"].shape[0], d["x"].shape[1]
    assert lib().hq_linear_path(ctypes.byref(w), N) == HQ_PATH_GEMV32
    # one launch when the rotation runs in the kernel (K <= 8192 and a CTA per
    # batch row), else the prep kernel first
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    fused = K <= 8192 and min(sms, (M + 31) // 32) >= N
    expect = 1 if fused else 2
    assert lib().hq_linear_launches(ctypes.byref(w), N) == expect
    x = dev(d["x"])
    torch.cuda.synchronize()
    n0 = hq_launch_count()
    y = hq_linear(q, s, g, x, d["bits"], d["zero"], planes=planes)
    torch.cuda.synchronize()
    assert hq_launch_count() - n0 == expect
    return y.cpu().numpy()


CASES = [
    # (M, K, N): one slice (K = 1024), ragged tiles and batches, uneven tiles per CTA
    (32, 1024, 9), (1, 1024, 16), (1000, 2048, 12), (4099, 4096, 16), (777, 8192, 10),
    (5000, 8192, 13), (300, 16384, 11), (9473, 1024, 15),
]


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("M,K,N", CASES)
def test_gemv32_parity(bits, M, K, N):
    d = synth.linear(M, K, bits, N, seed=7 * M + K + N + bits)
    y = run(d)
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"], threads=8)
    assert_within(y, want, bound, what=f"gemv32 b{bits} M{M} K{K} N{N}")


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("M,K,N", [(100, 1024, 1), (517, 4096, 3), (2048, 8192, 8), (33, 2048, 5)])
def test_gemv32_one_column_block(bits, M, K, N, from_batch_1):
    d = synth.linear(M, K, bits, N, seed=3 * M + K + N + bits, scale_dist="loguniform", outlier_frac=0.01)
    y = run(d)
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert_within(y, want, bound, what=f"gemv32 one block b{bits} M{M} K{K} N{N}")


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_gemv32_nondefault_zero_null_signs(bits):
    M, K, N = 700, 4096, 14
    d = synth.linear(M, K, bits, N, seed=90 + bits)
    d["zero"] = (1 << bits) - 1 if bits < 8 else 3
    y = run(d, signs=False)
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], None, d["x"])
    assert_within(y, want, bound, what=f"gemv32 zero/null signs b{bits}")


@pytest.mark.parametrize("N", [9, 16])
def test_gemv32_bit_planes(N):
    M, K = 1500, 8192
    d = synth.linear(M, K, 2, N, seed=123 + N)
    y = run(d, planes=True)
    want, bound = oracle.linear(2, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert_within(y, want, bound, what=f"gemv32 bit planes N{N}")


@pytest.mark.parametrize("scale", [2.0**-10, 2.0**-14])
def test_gemv32_small_activations(scale):
    M, K, N, bits = 400, 8192, 16, 3
    d = synth.linear(M, K, bits, N, seed=77)
    d["x"] = (d["x"].astype(np.float64) * scale).astype(np.float16)
    y = run(d)
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert_within(y, want, bound, what=f"gemv32 x*{scale}")


def test_gemv32_largest_launch_sampled_rows():
    """16 tiles of 32 rows for every CTA: the most one launch takes; one row
    more goes to the tensor-core GEMM."""
    from bit_hadamard_rotated_b200 import make_weight
    from bit_hadamard_rotated_b200._lib import HQ_PATH_TENSOR, lib
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    M, K, N, bits = 16 * 32 * sms, 1024, 16, 4
    d = synth.linear(M, K, bits, N, seed=5)
    y = run(d)
    rng = np.random.default_rng(1)
    rows = sorted(set(range(8)) | set(range(M - 40, M)) | set(rng.choice(M, 40, replace=False).tolist()))
    want, bound = oracle.linear(bits, len(rows), K, d["zero"], d["q"][rows], d["scales"][rows], d["signs"],
                                d["x"])
    assert_within(y[:, rows], want, bound, what="largest launch rows")
    w = make_weight(dev(d["q"][:1].view(np.int32)), dev(d["scales"][:1]), None, bits, d["zero"])
    w.M = M + 1
    assert lib().hq_linear_path(ctypes.byref(w), N) == HQ_PATH_TENSOR


def test_gemv32_deterministic_and_overwrites():
    from bit_hadamard_rotated_b200 import RotatedLinear
    M, K, N, bits = 3000, 8192, 16, 2
    d = synth.linear(M, K, bits, N, seed=9)
    lin = RotatedLinear(dev(d["q"].view(np.int32)), dev(d["scales"]), dev(d["signs"]), bits, d["zero"],
                        max_batch=N)
    assert lin.path(N) == "GEMV32"
    x = dev(d["x"])
    out = torch.full((N, M), float("nan"), device="cuda")
    lin(x, out=out)
    y1 = out.clone()
    lin(x, out=out)
    lin.check_status()
    assert torch.equal(y1, out)
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert_within(out.cpu().numpy(), want, bound, what="overwrite")


def test_gemv32_full_size_sampled_rows():
    """The dense MLP linear (28672 x 8192, 2-bit, log-uniform scales, outlier
    channels) at batch 16, sampled rows against the oracle."""
    M, K, bits, N = 28672, 8192, 2, 16
    d = synth.linear(M, K, bits, N, seed=1, scale_dist="loguniform", outlier_frac=0.01)
    y = run(d)
    rng = np.random.default_rng(M + N)
    rows = sorted(set(range(8)) | set(range(M - 8, M)) | set(rng.choice(M, 24, replace=False).tolist()))
    want, bound = oracle.linear(bits, len(rows), K, d["zero"], d["q"][rows], d["scales"][rows], d["signs"],
                                d["x"])
    assert_within(y[:, rows], want, bound, what="28672x8192 b2 N16")
    assert np.all(np.isfinite(y))
