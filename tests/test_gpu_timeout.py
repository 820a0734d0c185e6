"""The device error path: a bounded wait that runs out.

hq_set_test_fault makes the next GEMV launch leave one shared-memory copy of
CTA 0's last warp unrequested (the shapes give that warp several chunks); that warp's wait gives up after about a second,
the kernel records HQ_ERR_TIMEOUT in the status word and returns (no trap, no
hang), the copies that were requested are drained, and the context stays
usable: the next call on a zeroed workspace matches the oracle again."""
import ctypes

import numpy as np
import pytest
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


def test_gemv_wait_runs_out_and_is_reported():
    from bit_hadamard_rotated_b200 import HqError, hq, hq_check_status, hq_linear
    from bit_hadamard_rotated_b200._lib import HQ_ERR_TIMEOUT, lib
    M, K, bits = 16384, 4096, 4
    d = synth.linear(M, K, bits, 1, seed=91)
    q, sc, s, x = (torch.from_numpy(np.ascontiguousarray(v)).cuda()
                   for v in (d["q"].view(np.int32), d["scales"], d["signs"], d["x"]))
    w = hq.make_weight(q, sc, s, bits, d["zero"])
    ws = torch.zeros(hq.hq_linear_workspace_size(w, 1), dtype=torch.uint8, device="cuda")
    L = lib()
    assert L.hq_set_test_fault(1) == 0
    hq_linear(q, sc, s, x, bits, d["zero"], workspace=ws)
    with pytest.raises(HqError) as ei:
        hq_check_status(ws)
    assert ei.value.status == HQ_ERR_TIMEOUT
    assert L.hq_set_test_fault(-1) == 0  # used up by that one launch
    ws.zero_()
    y = hq_linear(q, sc, s, x, bits, d["zero"], workspace=ws).cpu().numpy()
    hq_check_status(ws)
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"], threads=8)
    assert np.all(np.abs(y - want) <= 2e-3 * bound + 1e-5)


def test_noalloc_wait_runs_out_and_is_reported():
    from bit_hadamard_rotated_b200 import HqError, hq_linear_noalloc, hq_linear_noalloc_check_status
    from bit_hadamard_rotated_b200._lib import HQ_ERR_TIMEOUT, lib
    M, K, bits = 16384, 4096, 2
    d = synth.linear(M, K, bits, 1, seed=92)
    q, sc, s, x = (torch.from_numpy(np.ascontiguousarray(v)).cuda()
                   for v in (d["q"].view(np.int32), d["scales"], d["signs"], d["x"]))
    lib().hq_set_test_fault(1)
    hq_linear_noalloc(q, sc, s, x, bits, d["zero"])
    with pytest.raises(HqError) as ei:
        hq_linear_noalloc_check_status()
    assert ei.value.status == HQ_ERR_TIMEOUT
    y = hq_linear_noalloc(q, sc, s, x, bits, d["zero"]).cpu().numpy()
    hq_linear_noalloc_check_status()
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"], threads=8)
    assert np.all(np.abs(y - want) <= 2e-3 * bound + 1e-5)


def test_gemv32_gate_wait_runs_out_and_is_reported():
    """The 32-row GEMV with its rotation inside: CTA 0 withholds its rotated
    row, every CTA's wait at the gate gives up, the status says so, and the
    next call on a zeroed workspace matches the oracle."""
    from bit_hadamard_rotated_b200 import HqError, hq, hq_check_status, hq_linear
    from bit_hadamard_rotated_b200._lib import HQ_ERR_TIMEOUT, HQ_PATH_GEMV32, lib
    M, K, bits, N = 4096, 4096, 2, 12
    d = synth.linear(M, K, bits, N, seed=93)
    q, sc, s, x = (torch.from_numpy(np.ascontiguousarray(v)).cuda()
                   for v in (d["q"].view(np.int32), d["scales"], d["signs"], d["x"]))
    w = hq.make_weight(q, sc, s, bits, d["zero"])
    L = lib()
    assert L.hq_linear_path(ctypes.byref(w), N) == HQ_PATH_GEMV32 and L.hq_linear_launches(ctypes.byref(w), N) == 1
    ws = torch.zeros(hq.hq_linear_workspace_size(w, N), dtype=torch.uint8, device="cuda")
    assert L.hq_set_test_fault(1) == 0
    hq_linear(q, sc, s, x, bits, d["zero"], workspace=ws)
    with pytest.raises(HqError) as ei:
        hq_check_status(ws)
    assert ei.value.status == HQ_ERR_TIMEOUT
    assert L.hq_set_test_fault(-1) == 0
    ws.zero_()
    y = hq_linear(q, sc, s, x, bits, d["zero"], workspace=ws).cpu().numpy()
    hq_check_status(ws)
    want, bound = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"], threads=8)
    assert np.all(np.abs(y - want) <= 2e-3 * bound + 1e-5)
