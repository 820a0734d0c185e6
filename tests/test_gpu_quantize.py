"""GPU parity of hq_quantize (the rotated round-to-nearest packer) against the
fp64 oracle, and the accuracy of the linear it feeds.

Codes and scales are integers decided in floating point; both sides decide in
fp64 (rotation, scale, r / scale, rint), with the same butterfly order for
K <= 16384, so codes and fp16 scales must match bit for bit.  At K = 32768 the
kernel takes the top butterfly stage first (two CTAs per row), so a code may
differ where r / scale lies within 1e-9 of a rounding tie, and a scale where
its fp16 rounding is within 1e-12 of a tie; nothing else may differ.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from bit_hadamard_rotated_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_hadamard_rotated_b200 import build
    build.build()


def weights(M, K, seed, dtype):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((M, K)) * 0.02
    W[:, rng.choice(K, max(1, K // 100), replace=False)] *= 20.0  # outlier input channels
    W[0, :] = 0.0                                                # a zero row
    Wt = torch.from_numpy(W).to(dtype)
    return Wt, Wt.double().numpy(), synth.signs(rng, K)


def codes_of(q, bits, K):
    return np.stack([oracle.unpack(row, bits, K) for row in q.view(np.uint32)])


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("M,K", [(37, 128), (64, 1024), (33, 4096), (9, 16384), (5, 32768)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_quantize_parity(bits, M, K, dtype):
    from bit_hadamard_rotated_b200 import hq_quantize
    Wt, Wd, s = weights(M, K, 100 * bits + K % 97 + M, dtype)
    q, sc = hq_quantize(Wt.cuda(), bits, torch.from_numpy(s).cuda())
    q, sc = q.cpu().numpy(), sc.cpu().numpy()
    qo, sco, r = oracle.quantize(Wd, bits, s, want_rotated=True)
    got_s, want_s = sc.view(np.uint16), sco.view(np.uint16)
    got_c, want_c = codes_of(q, bits, K), codes_of(qo, bits, K)
    if K <= 16384:
        assert np.array_equal(got_s, want_s)
        assert np.array_equal(q.view(np.uint32), qo)
        return
    # K = 32768: only near-ties may differ
    qmax = (1 << bits) - 1
    pre = np.minimum(2 * np.abs(r).reshape(M, K // 128, 128).max(axis=2) / qmax, 65504.0)
    bad_s = got_s != want_s
    if bad_s.any():
        lo = sco.astype(np.float64)[bad_s]
        hi = sc.astype(np.float64)[bad_s]
        mid = (lo + hi) / 2
        assert np.all(np.abs(pre[bad_s] - mid) <= 1e-12 * mid), "scale differs away from a tie"
    scale = np.repeat(sc.astype(np.float64), 128, axis=1)
    bad_c = got_c != want_c
    if bad_c.any():
        with np.errstate(divide="ignore", invalid="ignore"):
            t = r / scale
        dist = np.abs(np.abs(t - np.floor(t)) - 0.5)
        ok = (dist[bad_c] < 1e-9) | np.repeat(bad_s, 128, axis=1)[bad_c]
        assert np.all(ok), "code differs away from a rounding tie"
        assert np.all(np.abs(got_c[bad_c].astype(int) - want_c[bad_c].astype(int)) <= 1)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("M,K,N", [(600, 4096, 1), (300, 8192, 16), (256, 2048, 64)])
def test_quantized_linear_approximates_dense_product(bits, M, K, N):
    """hq_quantize then hq_linear: y is W x (numpy, fp64) within the
    quantisation bound sum_g scale_g / 2 (1 + 2^(b-10)) sum_{k in g} |x'_k|
    (the rotation cancels: W x = W_rot x') plus the linear's own tolerance,
    2e-3 sum_k |w_k x'_k| + 1e-5 (w the dequantised rotated weights)."""
    from bit_hadamard_rotated_b200 import hq_linear, hq_quantize
    Wt, Wd, s = weights(M, K, 7 * bits + N, torch.float32)
    st = torch.from_numpy(s).cuda()
    q, sc = hq_quantize(Wt.cuda(), bits, st)
    rng = np.random.default_rng(bits)
    x = rng.standard_normal((N, K)).astype(np.float16)
    y = hq_linear(q, sc, st, torch.from_numpy(x).cuda(), bits).cpu().numpy().astype(np.float64)
    xd = x.astype(np.float64)
    want = xd @ Wd.T
    xr = oracle.rotate(xd, s)
    ax = np.abs(xr).reshape(N, K // 128, 128).sum(axis=2)
    scf = sc.cpu().numpy().astype(np.float64)
    qbound = (ax @ (scf.T / 2)) * (1 + 2.0**(bits - 10))
    _, lin_bound = oracle.linear(bits, M, K, 1 << (bits - 1), q.cpu().numpy().view(np.uint32),
                                 sc.cpu().numpy(), s, x)
    lim = qbound * (1 + 1e-9) + 2e-3 * lin_bound + 1e-5
    err = np.abs(y - want)
    assert np.all(err <= lim), float(np.max(err / lim))
    # the 8-bit grid is fine enough that the product is close in relative terms too
    if bits == 8:
        assert np.max(err) <= 0.05 * np.max(np.abs(want))
