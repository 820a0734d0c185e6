"""hq_linear_noalloc: the workspace-free variant of hq_linear, for callers
that cannot allocate device memory (its scratch lives in a fixed device array
inside the library).  Called through the C ABI, it must give the same results
as hq_linear within the linear's tolerance, on two calls in a row (the second
call reuses the scratch the first one left behind).  Collected last, so a run
that stops at the first failure has already run every other test."""
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


@pytest.mark.parametrize("M,K,bits,N", [(4096, 4096, 4, 1), (1000, 1024, 3, 3), (12288, 4096, 2, 8),
                                         (257, 8192, 8, 2),
                                         # batches past one block of 8 columns: the blocks run
                                         # in turn through the one scratch region, at offsets
                                         # n0*K of x and n0*M of y; K = 16384 rotates in a
                                         # separate kernel for every block
                                         (257, 4096, 2, 11), (1000, 4096, 3, 17),
                                         (257, 16384, 4, 20), (333, 2048, 8, 9),
                                         (130, 32768, 2, 3), (130, 32768, 8, 2)])
def test_noalloc_matches_hq_linear_twice(M, K, bits, N):
    from bit_hadamard_rotated_b200 import _lib, hq_linear, make_weight
    d = synth.linear(M, K, bits, N, seed=M + K + bits)
    q = torch.from_numpy(d["q"].view(np.int32)).cuda()
    sc = torch.from_numpy(d["scales"]).cuda()
    s = torch.from_numpy(d["signs"]).cuda()
    x = torch.from_numpy(d["x"]).cuda()
    ref = hq_linear(q, sc, s, x, bits, d["zero"]).cpu().numpy()
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"],
                                threads=8)
    w = make_weight(q, sc, s, bits, d["zero"])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        y = torch.full((N, M), float("nan"), dtype=torch.float32, device="cuda")
        st = _lib.lib().hq_linear_noalloc(ctypes.byref(w), ctypes.c_void_p(x.data_ptr()), N,
                                          ctypes.c_void_p(y.data_ptr()), stream)
        assert st == 0, _lib.status_string(st)
        got = y.cpu().numpy()
        lim = REL * bound + ABS
        assert np.all(np.abs(got - ref) <= lim), (call, float(np.max(np.abs(got - ref) / lim)))
        assert np.all(np.abs(got - want) <= lim), (call, float(np.max(np.abs(got - want) / lim)))
        st = _lib.lib().hq_linear_noalloc_check_status(stream)
        assert st == 0, _lib.status_string(st)


def test_noalloc_rejects_what_hq_linear_rejects():
    """No size limit of its own: unsupported shapes fail with hq_linear's status,
    before anything is launched."""
    from bit_hadamard_rotated_b200 import _lib
    from bit_hadamard_rotated_b200._lib import HQ_ERR_UNSUPPORTED, HqWeight
    L = _lib.lib()
    before = L.hq_launch_count()
    for K, want in ((65536, HQ_ERR_UNSUPPORTED), (96, HQ_ERR_UNSUPPORTED)):
        w = HqWeight(4, 64, K, 8, 0x100000, 0x100000, None)
        st = L.hq_linear_noalloc(ctypes.byref(w), 0x100000, 1, 0x100000, None)
        assert st == want
    assert L.hq_launch_count() == before
