"""GPU parity of the nibble-split screened readout (hq_readout_topk) and of
hq_split_nibbles against the fp64 oracle.

The returned ids are integers decided by floating point: the oracle's exact
top-k is unique except where two exact logits lie within the linear's
tolerance of each other, so the check is: every GPU logit within 2e-3 of its
row's sum_k |w_k x'_k| (+1e-5) of the oracle's exact logit of the same row,
the GPU ids in non-increasing exact order up to that tolerance, and the GPU's
set equal to the oracle's except for rows whose exact logit is within the
tolerance of the topk-th value."""
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


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def merged_q8(r, rows):
    """8-bit packed codes 16 hi + lo of the given rows (oracle unpack/pack)."""
    out = []
    for m in rows:
        c = 16 * oracle.unpack(r["hi"][m], 4, r["K"]).astype(np.int64) + oracle.unpack(r["lo"][m], 4, r["K"])
        out.append(oracle.pack(c.astype(np.uint8), 8))
    return np.stack(out)


def run(r, topk, beta=6.0):
    from bit_hadamard_rotated_b200 import ScreenedReadout
    ro = ScreenedReadout(dev(r["hi"].view(np.int32)), dev(r["lo"].view(np.int32)), dev(r["scales"]),
                         dev(r["signs"]), r["zero"], max_batch=r["N"])
    ids, out = ro.topk(dev(r["x"]), topk, beta)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), out.cpu().numpy()


def check(r, topk, ids, out, beta=6.0):
    oid, oval, _, yall, _ = oracle.readout(r["hi"], r["lo"], r["scales"], r["signs"], r["V"], r["K"], r["zero"],
                                           r["x"], topk, beta=beta, want_all=True)
    for n in range(r["N"]):
        rows = ids[n].tolist()
        assert len(set(rows)) == topk and min(rows) >= 0 and max(rows) < r["V"]
        q8 = merged_q8(r, rows)
        # per-row tolerance base sum_k |w x'| of the GPU's rows (oracle linear on the merged codes)
        _, bnd = oracle.linear(8, len(rows), r["K"], r["zero"], q8, r["scales"][rows], r["signs"],
                               r["x"][n:n + 1])
        lim = 2e-3 * bnd[0] + 1e-5
        exact = yall[n, rows]
        assert np.all(np.abs(out[n] - exact) <= lim), float(np.max(np.abs(out[n] - exact) / lim))
        assert np.all(np.diff(exact) <= 2 * lim[1:] + 2 * lim[:-1])
        kth = oval[n, -1]
        tol = float(np.max(lim)) * 2
        want = set(oid[n].tolist())
        got = set(rows)
        for m in want ^ got:
            assert abs(yall[n, m] - kth) <= tol, ("set differs away from a near-tie", m)


@pytest.mark.parametrize("V,K,N,topk", [(3000, 256, 1, 1), (3000, 256, 3, 8), (5000, 2048, 2, 64),
                                        (20000, 1024, 8, 5), (777, 128, 1, 256)])
def test_readout_small(V, K, N, topk):
    r = synth.readout(V=V, K=K, N=N, seed=V + K + N)
    ids, out = run(r, topk)
    check(r, topk, ids, out)


def test_readout_full_vocabulary():
    """The lm_head of the 157,184-token vocabulary over hidden 2048, batch 1, top-8."""
    r = synth.readout(N=1, seed=1)
    ids, out = run(r, 8)
    check(r, 8, ids, out)


def test_readout_every_row_a_candidate():
    """beta so large that every row is refined: the final selection then runs
    over the whole vocabulary's exact logits."""
    r = synth.readout(V=40000, K=256, N=2, seed=4)
    ids, out = run(r, 16, beta=1e6)
    check(r, 16, ids, out, beta=1e6)


def test_readout_repeat_calls_reuse_workspace():
    """Counters left at zero: a second call on the same workspace gives the same result."""
    from bit_hadamard_rotated_b200 import ScreenedReadout
    r = synth.readout(V=6000, K=512, N=2, seed=5)
    ro = ScreenedReadout(dev(r["hi"].view(np.int32)), dev(r["lo"].view(np.int32)), dev(r["scales"]),
                         dev(r["signs"]), r["zero"], max_batch=2)
    a = [t.cpu().numpy() for t in ro.topk(dev(r["x"]), 10)]
    b = [t.cpu().numpy() for t in ro.topk(dev(r["x"]), 10)]
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    check(r, 10, a[0], a[1])


def test_split_nibbles_bit_exact():
    from bit_hadamard_rotated_b200 import hq_split_nibbles
    rng = np.random.default_rng(3)
    rows, K = 300, 1024
    q8 = rng.integers(0, 2**32, size=(rows, K // 4), dtype=np.uint64).astype(np.uint32)
    hi, lo = hq_split_nibbles(dev(q8.view(np.int32)), K)
    hi, lo = hi.cpu().numpy().view(np.uint32), lo.cpu().numpy().view(np.uint32)
    for m in range(0, rows, 37):
        c = oracle.unpack(q8[m], 8, K)
        assert np.array_equal(oracle.unpack(hi[m], 4, K), c >> 4)
        assert np.array_equal(oracle.unpack(lo[m], 4, K), c & 15)
