"""GPU parity: libhq (through the C ABI) against the fp64 CPU oracle.

Tolerances:
  * unpack: bit-exact.
  * rotation, fp32 output: |d_i| <= (log2 K + 2) 2^-24 sum_j|x_j| / sqrt(K) + 1e-12
    (one fp32 rounding per butterfly stage of values bounded by sum|x|/sqrt(K)
    after scaling, plus the final scale); fp16/bf16 output adds one rounding
    of x' (2^-11 / 2^-8 relative, 2^-25 absolute for fp16 subnormals).
  * linear / MoE: |y - y_oracle| <= 2e-3 sum_k |w_k x'_k| + 1e-5 per element,
    with the sum taken by the oracle.
"""
import math

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


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def assert_within(y, want, bound, rel=REL, abs_=ABS, what=""):
    err = np.abs(y.astype(np.float64) - want)
    lim = rel * bound + abs_
    bad = err > lim
    if bad.any():
        i = np.unravel_index(np.argmax(err / lim), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {err.size} outside tolerance; worst at {i}: "
                             f"got {y[i]!r} want {want[i]!r} err {err[i]:.3e} lim {lim[i]:.3e}")


# ---------------------------------------------------------------- unpack (bit-exact)
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_unpack_codes_bit_exact(bits):
    from bit_hadamard_rotated_b200 import hq_unpack_codes
    rng = np.random.default_rng(bits)
    n = 32 * 40000 + (0 if bits in (1, 2, 4, 8) else 0)
    words = rng.integers(0, 2**32, size=n * bits // 32, dtype=np.uint64).astype(np.uint32)
    # pattern words at the front: all ones, alternating bits, single bits
    words[:3] = [0xFFFFFFFF, 0xAAAAAAAA, 0x55555555]
    got = hq_unpack_codes(dev(words.view(np.int32)), bits, n).cpu().numpy()
    assert np.array_equal(got, oracle.unpack(words, bits, n))


def test_unpack_ragged_tail_does_not_read_past_end():
    from bit_hadamard_rotated_b200 import hq_unpack_codes
    words = np.array([0x88FAC688, 0xC688FAC6], np.uint32)  # 64 bits -> 21 whole 3-bit codes
    got = hq_unpack_codes(dev(words.view(np.int32)), 3, 21).cpu().numpy()
    assert np.array_equal(got, oracle.unpack(words, 3, 21))


# ---------------------------------------------------------------- rotation
@pytest.mark.parametrize("K", [32, 64, 128, 512, 2048, 4096, 8192, 32768])
@pytest.mark.parametrize("in_dt,out_dt", [(torch.float16, torch.float32),
                                          (torch.float32, torch.float32),
                                          (torch.float16, torch.float16),
                                          (torch.bfloat16, torch.bfloat16)])
def test_rotate_parity(K, in_dt, out_dt):
    from bit_hadamard_rotated_b200 import hq_rotate
    rng = np.random.default_rng(K)
    rows = 5
    x = rng.standard_normal((rows, K)) * np.where(rng.random(K) < 0.01, 20.0, 1.0)
    s = synth.signs(rng, K)
    xt = torch.from_numpy(x).to(in_dt)
    x_used = xt.float().double().numpy()  # the exact input values the kernel sees
    got = hq_rotate(xt.cuda(), dev(s), out_dtype=out_dt).float().cpu().numpy()
    want = oracle.rotate(x_used, s)
    L = math.log2(K)
    bound = (L + 2) * 2.0**-24 * np.abs(x_used).sum(axis=1, keepdims=True) / math.sqrt(K)
    bound = bound + 1e-12
    if out_dt == torch.float16:
        bound = bound + 2.0**-11 * np.abs(want) + 2.0**-25
    if out_dt == torch.bfloat16:
        bound = bound + 2.0**-8 * np.abs(want) + 1e-38
    assert np.all(np.abs(got - want) <= bound), np.max(np.abs(got - want) / bound)


def test_rotate_null_signs_and_zero_rows():
    from bit_hadamard_rotated_b200 import hq_rotate
    K = 1024
    x = torch.zeros((3, K), dtype=torch.float16)
    x[0, 0] = 1.0
    x[1] = 1.0
    got = hq_rotate(x.cuda(), None).cpu().numpy()
    assert np.allclose(got[0], 1 / math.sqrt(K), atol=1e-7)
    assert abs(got[1, 0] - math.sqrt(K)) < 1e-4 and np.allclose(got[1, 1:], 0, atol=1e-5)
    assert np.array_equal(got[2], np.zeros(K, np.float32))
    empty = hq_rotate(torch.zeros((0, K), dtype=torch.float16).cuda())
    assert empty.shape == (0, K)


# ---------------------------------------------------------------- linear, small shapes (full check)
def run_linear(d, out=None):
    from bit_hadamard_rotated_b200 import hq_linear
    return hq_linear(dev(d["q"].view(np.int32)), dev(d["scales"]), dev(d["signs"]),
                     dev(d["x"]), d["bits"], d["zero"], out=out)


SMALL = [(16, 128, 1), (17, 256, 3), (33, 512, 8), (100, 1024, 5), (64, 4096, 2),
         (257, 2048, 7), (5, 128, 9), (40, 8192, 4), (16, 16384, 1), (48, 1024, 17),
         (1, 128, 1), (31, 256, 16)]


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("M,K,N", SMALL)
def test_linear_parity_small(bits, M, K, N):
    d = synth.linear(M, K, bits, N, seed=7 * M + K + N)
    y = run_linear(d).cpu().numpy()
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert_within(y, want, bound, what=f"b{bits} M{M} K{K} N{N}")


@pytest.mark.parametrize("bits", [2, 4])
def test_linear_outliers_and_loguniform_scales(bits):
    d = synth.linear(96, 8192, bits, 3, seed=3, scale_dist="loguniform", outlier_frac=0.01)
    y = run_linear(d).cpu().numpy()
    want, bound = oracle.linear(bits, 96, 8192, d["zero"], d["q"], d["scales"], d["signs"],
                                d["x"])
    assert_within(y, want, bound, what="outliers")


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_linear_nondefault_zero_and_null_signs(bits):
    d = synth.linear(40, 512, bits, 2, seed=11)
    d["zero"] = (1 << bits) - 1
    d["signs"] = None
    from bit_hadamard_rotated_b200 import hq_linear
    y = hq_linear(dev(d["q"].view(np.int32)), dev(d["scales"]), None, dev(d["x"]), bits,
                  d["zero"]).cpu().numpy()
    want, bound = oracle.linear(bits, 40, 512, d["zero"], d["q"], d["scales"], None, d["x"])
    assert_within(y, want, bound, what="zero/null signs")


def test_linear_special_codes():
    """All codes at the zero point give 0 (within the absolute floor, the tolerance's
    bound being 0); all at zero+1 give scale * sum x'."""
    bits, M, K, N = 4, 32, 1024, 3
    d = synth.linear(M, K, bits, N, seed=5)
    q0 = np.stack([oracle.pack(np.full(K, 8, np.uint8), bits)] * M)
    d0 = dict(d, q=q0)
    y0 = run_linear(d0).cpu().numpy()
    w0, b0 = oracle.linear(bits, M, K, 8, q0, d["scales"], d["signs"], d["x"])
    assert np.array_equal(w0, np.zeros((N, M))) and np.array_equal(b0, np.zeros((N, M)))
    assert_within(y0, w0, b0, what="zero codes")
    q1 = np.stack([oracle.pack(np.full(K, 9, np.uint8), bits)] * M)
    d1 = dict(d, q=q1)
    y1 = run_linear(d1).cpu().numpy()
    want, bound = oracle.linear(bits, M, K, 8, q1, d["scales"], d["signs"], d["x"])
    assert_within(y1, want, bound, what="constant codes")


def test_linear_batch_zero_and_determinism():
    from bit_hadamard_rotated_b200 import hq_linear
    d = synth.linear(256, 4096, 2, 4, seed=9)
    a = run_linear(d)
    b = run_linear(d)
    assert torch.equal(a, b)
    empty = hq_linear(dev(d["q"].view(np.int32)), dev(d["scales"]), dev(d["signs"]),
                      dev(d["x"][:0]), 2)
    assert empty.shape == (0, 256)


def test_linear_output_overwritten_not_accumulated():
    d = synth.linear(64, 1024, 3, 2, seed=12)
    out = torch.full((2, 64), 123.0, device="cuda")
    y = run_linear(d, out=out).cpu().numpy()
    want, bound = oracle.linear(3, 64, 1024, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert_within(y, want, bound, what="overwrite")


@pytest.mark.parametrize("bits,M,K,N", [(2, 2400, 1024, 1), (3, 4100, 512, 2), (8, 2376, 2048, 3),
                                         (4, 4739, 256, 8), (2, 2368, 4096, 1)])
def test_linear_uneven_tiles_per_cta_all_rows(bits, M, K, N):
    """Enough 16-row tiles that CTAs own different numbers of them, some tiles
    split between warps: every row is checked, and a repeat call on the same
    workspace is bit-identical."""
    from bit_hadamard_rotated_b200 import hq
    d = synth.linear(M, K, bits, N, seed=M + K)
    q, sc, sg, x = dev(d["q"].view(np.int32)), dev(d["scales"]), dev(d["signs"]), dev(d["x"])
    need = hq.hq_linear_workspace_size(hq.make_weight(q, sc, sg, bits, d["zero"]), N)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y1 = hq.hq_linear(q, sc, sg, x, bits, d["zero"], workspace=ws)
    y2 = hq.hq_linear(q, sc, sg, x, bits, d["zero"], workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert_within(y1.cpu().numpy(), want, bound, what=f"b{bits} M{M} K{K} N{N}")


def test_linear_workspace_shared_by_paths_and_batches():
    """One workspace serves GEMV calls of several batches and tensor-core calls
    in between (results match the oracle each time)."""
    from bit_hadamard_rotated_b200 import hq
    d = synth.linear(2400, 2048, 2, 64, seed=21)
    q, sc, sg = dev(d["q"].view(np.int32)), dev(d["scales"]), dev(d["signs"])
    w = hq.make_weight(q, sc, sg, 2, d["zero"])
    ws = torch.zeros(max(hq.hq_linear_workspace_size(w, n) for n in (1, 3, 64)), dtype=torch.uint8,
                     device="cuda")
    want, bound = oracle.linear(2, 2400, 2048, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    for n in (1, 64, 3, 1, 64, 2):
        y = hq.hq_linear(q, sc, sg, dev(d["x"][:n]), 2, d["zero"], workspace=ws).cpu().numpy()
        assert_within(y, want[:n], bound[:n], what=f"batch {n}")


def test_rotated_linear_prepared_launcher():
    """RotatedLinear.prepare: a launcher on fixed buffers gives the oracle's
    result on every call (also after the inputs change in place), and bad
    buffers are refused when it is made."""
    from bit_hadamard_rotated_b200 import RotatedLinear
    d = synth.linear(700, 1024, 3, 2, seed=23)
    lin = RotatedLinear(dev(d["q"].view(np.int32)), dev(d["scales"]), dev(d["signs"]), 3, d["zero"],
                        max_batch=2)
    x = torch.zeros((2, 1024), dtype=torch.float16, device="cuda")
    y = torch.full((2, 700), float("nan"), dtype=torch.float32, device="cuda")
    run = lin.prepare(x, y)
    want, bound = oracle.linear(3, 700, 1024, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    x.copy_(dev(d["x"]))
    for _ in range(2):
        run()
        assert_within(y.cpu().numpy(), want, bound, what="prepared launcher")
    x.mul_(-1)  # the launcher reads the buffer's current contents
    run()
    assert_within(y.cpu().numpy(), -want, bound, what="prepared launcher, negated input")
    with pytest.raises(ValueError):
        lin.prepare(x.float(), y)
    with pytest.raises(ValueError):
        lin.prepare(x, y[:, :699])
    with pytest.raises(ValueError):
        lin.prepare(torch.zeros((3, 1024), dtype=torch.float16, device="cuda"),
                    torch.zeros((3, 700), device="cuda"))


# ---------------------------------------------------------------- linear, full workload sizes (sampled rows)
def sample_rows(M, rng, n=24):
    rows = set(range(0, 8)) | set(range(M - 8, M)) | set(rng.choice(M, n, replace=False).tolist())
    return sorted(rows)


FULL = [
    # (M, K, bits, N, scale_dist, outlier_frac)
    (4096, 4096, 4, 1, "uniform", 0.0),
    (12288, 4096, 2, 1, "uniform", 0.0), (12288, 4096, 2, 8, "uniform", 0.0),
    (12288, 4096, 3, 1, "uniform", 0.0), (12288, 4096, 3, 4, "uniform", 0.0),
    (12288, 4096, 8, 1, "uniform", 0.0), (12288, 4096, 8, 2, "uniform", 0.0),
    (28672, 8192, 2, 1, "loguniform", 0.01), (28672, 8192, 2, 16, "loguniform", 0.01),
    (28672, 8192, 2, 64, "loguniform", 0.01),
    (8192, 8192, 3, 32, "uniform", 0.0), (8192, 8192, 8, 128, "uniform", 0.0),
]


# every (bits, batch) point of the bit-width-coverage workload, and the
# M = K = 8192 roofline sweep at batches 1, 8, 16, 64, 128 for every width
FULL += [(12288, 4096, b, n, "uniform", 0.0) for b in (2, 3, 8) for n in (1, 2, 4, 8)
         if (12288, 4096, b, n, "uniform", 0.0) not in FULL]
FULL += [(8192, 8192, b, n, "uniform", 0.0) for b in (2, 3, 4, 8) for n in (1, 8, 16, 64, 128)
         if (8192, 8192, b, n, "uniform", 0.0) not in FULL]


@pytest.mark.parametrize("M,K,bits,N,sd,of", FULL)
def test_linear_parity_full_size_sampled(M, K, bits, N, sd, of):
    d = synth.linear(M, K, bits, N, seed=1, scale_dist=sd, outlier_frac=of)
    y = run_linear(d).cpu().numpy()
    rng = np.random.default_rng(M + N)
    for m in sample_rows(M, rng):
        want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"],
                                    d["x"], m_begin=m, m_end=m + 1)
        assert_within(y[:, m], want[:, m], bound[:, m], what=f"row {m}")
    assert np.all(np.isfinite(y))


# ---------------------------------------------------------------- small activation scales
# The GEMV feeds the tensor cores x' * 2^-a in fp16 (a <= 8: the bit offset of
# a code's field inside its 16-bit half), so small activations reach fp16's
# subnormal range there first; the tensor-core path rounds x' itself to fp16.
# The same tolerance holds at any scale.
def _scaled(d, f):
    x = (d["x"].astype(np.float64) * f).astype(np.float16)
    return dict(d, x=x)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("N", [1, 2, 4, 16])
@pytest.mark.parametrize("scale", [2.0**-10, 2.0**-14])
def test_linear_small_activation_scales(bits, N, scale):
    M, K = 300, 4096
    d = _scaled(synth.linear(M, K, bits, N, seed=41 + bits + N), scale)
    assert np.any(np.abs(d["x"].astype(np.float64)) < 2.0**-14) or scale > 2.0**-14
    y = run_linear(d).cpu().numpy()
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert_within(y, want, bound, what=f"scale {scale} b{bits} N{N}")


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("N", [1, 3, 16])
@pytest.mark.parametrize("c", [1.0, 2.0**-12])
def test_linear_single_spike_null_signs(bits, N, c):
    """x = c e_j (a different j per row) with signs = NULL: x' = c H[:, j] / sqrt(K),
    every element +-c/sqrt(K), so y[n][m] = c sum_k w[m][k] H[k][j_n] / sqrt(K)."""
    from bit_hadamard_rotated_b200 import hq_linear
    M, K = 200, 8192
    d = synth.linear(M, K, bits, N, seed=51 + bits)
    x = np.zeros((N, K), np.float16)
    for n in range(N):
        x[n, (977 * n + 5) % K] = c
    y = hq_linear(dev(d["q"].view(np.int32)), dev(d["scales"]), None, dev(x), bits,
                  d["zero"]).cpu().numpy()
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], None, x)
    assert_within(y, want, bound, what=f"spike c={c} b{bits} N{N}")


# ---------------------------------------------------------------- the largest K
@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("N", [1, 2, 3, 9, 40])
def test_linear_k32768(bits, N):
    """K = 32768, the largest supported width: the GEMV (rotation in a prep
    kernel of 32 warps, batch blocks of 1 or 2 columns) and, from batch 5 or 9,
    the tensor-core GEMM with narrower column blocks."""
    M, K = 300, 32768
    d = synth.linear(M, K, bits, N, seed=61 + bits + N, scale_dist="loguniform", outlier_frac=0.01)
    y = run_linear(d).cpu().numpy()
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"], threads=8)
    assert_within(y, want, bound, what=f"K32768 b{bits} N{N}")


# ---------------------------------------------------------------- per-group zero points
@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("M,K,N", [(16, 128, 1), (37, 256, 3), (100, 1024, 2), (257, 2048, 1),
                                   (333, 4096, 5), (96, 8192, 8), (40, 16384, 2), (300, 4096, 19)])
def test_linear_per_group_zeros(bits, M, K, N):
    """Per-group zero points (uint8 [M][K/128], the GPTQ form): the small-batch
    kernel loads them beside the scales (a TMA box of 16 groups from K = 2048,
    the tile's span below) and starts each group's accumulator at its own
    row's zero-point term; batches past 8 run in blocks of 8 columns."""
    from bit_hadamard_rotated_b200 import hq_linear
    d = synth.linear(M, K, bits, N, seed=70 + M + K + bits)
    rng = np.random.default_rng(M + bits)
    zeros = rng.integers(0, 1 << bits, size=(M, K // 128)).astype(np.uint8)
    y = hq_linear(dev(d["q"].view(np.int32)), dev(d["scales"]), dev(d["signs"]), dev(d["x"]), bits,
                  zeros=dev(zeros)).cpu().numpy()
    want, bound = oracle.linear(bits, M, K, 0, d["q"], d["scales"], d["signs"], d["x"], zeros=zeros)
    assert_within(y, want, bound, what=f"zeros b{bits} M{M} K{K} N{N}")


def test_linear_per_group_zeros_full_size_sampled():
    from bit_hadamard_rotated_b200 import hq_linear
    M, K, bits, N = 28672, 8192, 2, 1
    d = synth.linear(M, K, bits, N, seed=5, scale_dist="loguniform", outlier_frac=0.01)
    zeros = np.random.default_rng(3).integers(0, 4, size=(M, K // 128)).astype(np.uint8)
    y = hq_linear(dev(d["q"].view(np.int32)), dev(d["scales"]), dev(d["signs"]), dev(d["x"]), bits,
                  zeros=dev(zeros)).cpu().numpy()
    rng = np.random.default_rng(7)
    for m in sample_rows(M, rng):
        want, bound = oracle.linear(bits, M, K, 0, d["q"], d["scales"], d["signs"], d["x"], m_begin=m,
                                    m_end=m + 1, zeros=zeros)
        assert_within(y[:, m], want[:, m], bound[:, m], what=f"row {m}")


# ---------------------------------------------------------------- 2-bit bit-plane storage
@pytest.mark.parametrize("M,K,N,pgz", [(16, 128, 1, False), (37, 256, 3, False), (100, 1024, 2, True),
                                       (333, 4096, 5, False), (96, 8192, 8, False), (200, 8192, 1, True),
                                       (40, 16384, 2, False), (300, 32768, 1, False), (300, 4096, 19, True)])
def test_linear_bit_planes(M, K, N, pgz):
    """2-bit codes kept as bit-planes (HQ_LAYOUT_BITPLANES): the small-batch
    kernel rebuilds each 32-code bundle's packed words in registers and reads
    the activations in the matching order; batches past 8 run in blocks of 8.
    Random words are valid plane words, so the synthetic q serves as is."""
    from bit_hadamard_rotated_b200 import hq_linear
    d = synth.linear(M, K, 2, N, seed=80 + M + K + N, scale_dist="loguniform", outlier_frac=0.01)
    zeros = np.random.default_rng(M).integers(0, 4, size=(M, K // 128)).astype(np.uint8) if pgz else None
    y = hq_linear(dev(d["q"].view(np.int32)), dev(d["scales"]), dev(d["signs"]), dev(d["x"]), 2,
                  zeros=None if zeros is None else dev(zeros), planes=True).cpu().numpy()
    want, bound = oracle.linear(2, M, K, 2, d["q"], d["scales"], d["signs"], d["x"], zeros=zeros, planes=True,
                                threads=4)
    assert_within(y, want, bound, what=f"planes M{M} K{K} N{N} pgz{pgz}")


def test_to_bitplanes_bit_exact_and_linear_full_size_sampled():
    """hq_to_bitplanes against the oracle's plane packer, then the 28672 x 8192
    layer in bit-plane form at batch 1 on sampled rows."""
    from bit_hadamard_rotated_b200 import hq_linear, hq_linear_noalloc, hq_to_bitplanes
    M, K, N = 28672, 8192, 1
    d = synth.linear(M, K, 2, N, seed=12, scale_dist="loguniform", outlier_frac=0.01)
    planes = hq_to_bitplanes(dev(d["q"].view(np.int32))).cpu().numpy().view(np.uint32)
    rng = np.random.default_rng(5)
    for m in rng.choice(M, 64, replace=False):
        assert np.array_equal(planes[m], oracle.pack_planes2(oracle.unpack(d["q"][m], 2, K))), m
    gp = dev(planes.view(np.int32))
    y = hq_linear(gp, dev(d["scales"]), dev(d["signs"]), dev(d["x"]), 2, planes=True).cpu().numpy()
    y2 = hq_linear_noalloc(gp, dev(d["scales"]), dev(d["signs"]), dev(d["x"]), 2, planes=True).cpu().numpy()
    # the planes hold d["q"]'s codes: the packed-stream oracle applies
    for m in sample_rows(M, rng):
        want, bound = oracle.linear(2, M, K, 2, d["q"], d["scales"], d["signs"], d["x"], m_begin=m, m_end=m + 1)
        assert_within(y[:, m], want[:, m], bound[:, m], what=f"row {m}")
        assert_within(y2[:, m], want[:, m], bound[:, m], what=f"noalloc row {m}")
