"""GPU parity of hq_moe_experts (through the C ABI) against the fp64 oracle.

Tolerance (end to end, two chained contractions): |y - y_oracle| <=
4e-3 * sum_j |topk_w[t][j]| sum_k |w_down x h'_k| + 1e-5, the oracle's bound;
each single contraction is held to 2e-3 (the stage-wise checks below: h
against the oracle's h, and d against the oracle's down projection of the
GPU's own h), and the chain doubles it.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from bit_hadamard_rotated_b200 import synth

pytestmark = pytest.mark.gpu

REL, ABS = 4e-3, 1e-5


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_hadamard_rotated_b200 import build
    build.build()
    import bit_hadamard_rotated_b200._lib as L
    L.lib()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def device_experts(experts):
    out = []
    for e in experts:
        d = dict(bits=e["bits"], zero=e["zero"])
        for n in ("q_gate", "q_up", "q_down"):
            d[n] = dev(e[n].view(np.int32))
        for n in ("s_gate", "s_up", "s_down"):
            d[n] = dev(e[n])
        for n in ("signs_in", "signs_mid"):
            if e.get(n) is not None:
                d[n] = dev(e[n])
        out.append(d)
    return out


def run_moe(m, ids=None, w=None, experts=None, ws=None):
    from bit_hadamard_rotated_b200 import expert_table, hq_moe_experts
    dexp = device_experts(m["experts"] if experts is None else experts)
    table = expert_table(dexp, "cuda")
    ids = m["topk_ids"] if ids is None else ids
    w = m["topk_w"] if w is None else w
    y = hq_moe_experts(table, len(dexp), m["hidden"], m["inter"], dev(m["x"]), dev(ids.astype(np.int32)),
                       dev(w.astype(np.float32)), dev(m["s_in"]), dev(m["s_mid"]), workspace=ws)
    torch.cuda.synchronize()
    return y.cpu().numpy(), dexp


def check(y, want, bound, what=""):
    err = np.abs(y.astype(np.float64) - want)
    lim = REL * bound + ABS
    bad = err > lim
    assert not bad.any(), (what, int(bad.sum()), float(np.max(err / lim)))


def oracle_moe(m, ids=None, w=None, experts=None, threads=8):
    return oracle.moe(m["experts"] if experts is None else experts, m["hidden"], m["inter"], m["x"],
                      m["topk_ids"] if ids is None else ids, m["topk_w"] if w is None else w,
                      m["s_in"], m["s_mid"], threads=threads)


def test_moe_full_layer():
    m = synth.moe(seed=0)
    y, _ = run_moe(m)
    want, bound, _ = oracle_moe(m)
    check(y, want, bound, "full")
    assert np.all(np.isfinite(y))


@pytest.mark.parametrize("seed,k,probs", [(1, 2, (0.4, 0.3, 0.3)), (2, 3, (0.0, 1.0, 0.0)),
                                          (3, 1, (0.0, 0.0, 1.0)), (4, 4, (1.0, 0.0, 0.0))])
def test_moe_small_mixed_widths(seed, k, probs):
    m = synth.moe(seed=seed, E=6, hidden=256, inter=128, T=5, k=k, probs=probs)
    y, _ = run_moe(m)
    want, bound, _ = oracle_moe(m)
    check(y, want, bound, f"small seed {seed}")


def test_moe_with_8bit_experts_and_other_shapes():
    m = synth.moe(seed=5, E=7, hidden=512, inter=256, T=9, k=3, probs=(0.25, 0.25, 0.5),
                  bits_choices=(2, 8, 4))
    y, _ = run_moe(m)
    want, bound, _ = oracle_moe(m)
    check(y, want, bound, "8-bit mix")


@pytest.mark.parametrize("hidden,inter", [(8192, 256), (256, 8192), (4096, 1024), (16384, 128),
                                          (32768, 128), (128, 32768)])
def test_moe_wide_shapes(hidden, inter):
    """Widths whose activation fragments do not fit beside the copy rings in
    shared memory (read from global memory instead), and ones that just fit."""
    m = synth.moe(seed=11, E=5, hidden=hidden, inter=inter, T=11, k=2, probs=(0.4, 0.3, 0.3),
                  bits_choices=(2, 3, 4))
    y, _ = run_moe(m)
    want, bound, _ = oracle_moe(m)
    check(y, want, bound, f"hidden {hidden} inter {inter}")


def test_moe_expert_with_many_tokens():
    """All 20 tokens choose expert 2 (three column blocks of <= 8 tokens)."""
    m = synth.moe(seed=6, E=4, hidden=256, inter=128, T=20, k=2)
    ids = np.tile(np.array([[2, 1]], np.int32), (20, 1))
    w = np.tile(np.array([[0.75, 0.25]], np.float32), (20, 1))
    y, _ = run_moe(m, ids=ids, w=w)
    want, bound, _ = oracle_moe(m, ids=ids, w=w)
    check(y, want, bound, "many tokens")


def test_moe_top1_is_single_chain_and_deterministic():
    m = synth.moe(seed=7, E=8, hidden=1024, inter=256, T=6, k=1)
    w1 = np.ones((6, 1), np.float32)
    y1, _ = run_moe(m, w=w1)
    y2, _ = run_moe(m, w=w1)
    assert np.array_equal(y1, y2)
    want, bound, _ = oracle_moe(m, w=w1)
    check(y1, want, bound, "top1")


def test_moe_bad_ids_and_descriptors_are_skipped_and_reported():
    from bit_hadamard_rotated_b200 import HqError, expert_table, hq_check_status, hq_moe_experts, \
        hq_moe_workspace_size
    m = synth.moe(seed=8, E=5, hidden=256, inter=128, T=4, k=2)
    ids = m["topk_ids"].copy()
    w = m["topk_w"].copy()
    ids[0, 1] = 5          # out of range
    ids[2, 0] = -1         # negative
    bad = [dict(e) for e in m["experts"]]
    bad[3] = dict(bad[3], bits=5)  # unsupported width: its pairs are skipped
    ids[1, 0] = 3
    dexp = device_experts(bad)
    table = expert_table(dexp, "cuda")
    ws = torch.zeros(hq_moe_workspace_size(5, 256, 128, 4, 2), dtype=torch.uint8, device="cuda")
    y = hq_moe_experts(table, 5, 256, 128, dev(m["x"]), dev(ids), dev(w), dev(m["s_in"]),
                       dev(m["s_mid"]), workspace=ws).cpu().numpy()
    with pytest.raises(HqError) as ei:
        hq_check_status(ws)
    assert ei.value.status == 5  # HQ_ERR_DATA
    hq_check_status(ws)  # cleared by the read
    # oracle: skipped pairs contribute nothing
    ids_o = ids.copy()
    w_o = w.copy()
    skip = (ids_o < 0) | (ids_o >= 5) | (ids_o == 3)
    ids_o[skip] = 0
    w_o[skip] = 0.0
    want, bound, _ = oracle_moe(m, ids=ids_o, w=w_o, experts=m["experts"])
    check(y, want, bound, "bad ids")


@pytest.mark.parametrize("E", [200, 1500])
def test_moe_many_experts_untouched_bad_descriptor(E):
    """Routing over many experts.  With hidden 128 (64-thread routing block)
    the 200-entry table is checked whole before the dependent-launch wait,
    the 1500-entry one only where the pairs name it; either way a bad
    descriptor that no pair names reports nothing and changes nothing.  Expert
    e's descriptor points at expert e % 5's tensors."""
    from bit_hadamard_rotated_b200 import expert_table, hq_check_status, hq_moe_experts, \
        hq_moe_workspace_size
    T, k = 7, 3
    m = synth.moe(seed=12, E=5, hidden=128, inter=128, T=T, k=k)
    base = device_experts(m["experts"])
    bad_e = E // 2
    descs = [base[e % 5] for e in range(E)]
    descs[bad_e] = dict(base[bad_e % 5], bits=5)
    rng = np.random.default_rng(E)
    choices = np.array([e for e in range(E) if e != bad_e])
    ids = np.stack([rng.choice(choices, k, replace=False) for _ in range(T)]).astype(np.int32)
    w = m["topk_w"].astype(np.float32)
    ws = torch.zeros(hq_moe_workspace_size(E, 128, 128, T, k), dtype=torch.uint8, device="cuda")
    y = hq_moe_experts(expert_table(descs, "cuda"), E, 128, 128, dev(m["x"]), dev(ids), dev(w),
                       dev(m["s_in"]), dev(m["s_mid"]), workspace=ws).cpu().numpy()
    hq_check_status(ws)  # nothing recorded
    want, bound, _ = oracle_moe(m, ids=ids % 5, w=w)
    check(y, want, bound, f"E={E}")


def test_moe_zero_tokens():
    from bit_hadamard_rotated_b200 import expert_table, hq_moe_experts
    m = synth.moe(seed=9, E=3, hidden=256, inter=128, T=2, k=1)
    dexp = device_experts(m["experts"])
    table = expert_table(dexp, "cuda")
    y = hq_moe_experts(table, 3, 256, 128, dev(m["x"][:0]), dev(m["topk_ids"][:0]),
                       dev(m["topk_w"][:0]), dev(m["s_in"]), dev(m["s_mid"]))
    assert y.shape == (0, 256)


# ---------------------------------------------------------------- stage by stage
def _stages(ws, m, E):
    """pos [T*k], h [rows][inter], d [rows][hidden] as the call left them in its workspace."""
    from bit_hadamard_rotated_b200 import _lib
    L = _lib.lib()
    T, k, H, I = m["T"], m["k"], m["hidden"], m["inter"]
    raw = ws.cpu().numpy()

    def part(which, count, dtype):
        off = L.hq_moe_workspace_offset(E, H, I, T, k, which)
        assert off % 256 == 0
        return raw[off:off + count * np.dtype(dtype).itemsize].view(dtype)

    rows = T * k
    return (part(_lib.HQ_MOE_POS, rows, np.int32), part(_lib.HQ_MOE_H, rows * I, np.float32).reshape(rows, I),
            part(_lib.HQ_MOE_D, rows * H, np.float32).reshape(rows, H))


def _check_stages(m, ws):
    E, T, k, H, I = len(m["experts"]), m["T"], m["k"], m["hidden"], m["inter"]
    pos, h_gpu, d_gpu = _stages(ws, m, E)
    _, _, h_want = oracle.moe(m["experts"], H, I, m["x"], m["topk_ids"], m["topk_w"], m["s_in"],
                              m["s_mid"], want_h=True, threads=8)
    assert sorted(pos.tolist()) == list(range(T * k))  # every pair valid, rows a permutation
    xr = oracle.rotate(m["x"], m["s_in"])
    rel = 2e-3
    for t in range(T):
        for j in range(k):
            e = m["experts"][int(m["topk_ids"][t, j])]
            r = int(pos[t * k + j])
            # gate/up + SwiGLU: h = silu(g) u with g, u each within 2e-3 of their own
            # L1 bases Bg, Bu; to first order |dh| <= max|silu'| |u| dg + |silu(g)| du
            # (max silu' = 1.0998), plus the product of the two errors
            xt = xr[t:t + 1] if e.get("signs_in") is None else oracle.rotate(m["x"][t:t + 1], e["signs_in"])
            g, bg = oracle.dequant_dot(e["bits"], I, H, e["zero"], e["q_gate"], e["s_gate"], xt)
            u, bu = oracle.dequant_dot(e["bits"], I, H, e["zero"], e["q_up"], e["s_up"], xt)
            g, bg, u, bu = g[0], bg[0], u[0], bu[0]
            silu = g / (1.0 + np.exp(-g))
            lim = rel * (1.1 * np.abs(u) * bg + np.abs(silu) * bu) + 1.1 * rel * rel * bg * bu + 1e-5
            err = np.abs(h_gpu[r].astype(np.float64) - h_want[t * k + j])
            assert np.all(err <= lim), ("h", t, j, float(np.max(err / lim)))
            # down, fed the GPU's own h: d = W_down H diag(s_mid) h_gpu / sqrt(inter)
            hr = oracle.rotate(h_gpu[r].astype(np.float64),
                               m["s_mid"] if e.get("signs_mid") is None else e["signs_mid"])
            dw, db = oracle.dequant_dot(e["bits"], H, I, e["zero"], e["q_down"], e["s_down"], hr[None, :])
            err = np.abs(d_gpu[r].astype(np.float64) - dw[0])
            lim = rel * db[0] + 1e-5
            assert np.all(err <= lim), ("d", t, j, float(np.max(err / lim)))


@pytest.mark.parametrize("which", ["full", "mixed-small", "mixed-8bit", "wide"])
def test_moe_stagewise(which):
    from bit_hadamard_rotated_b200 import hq_moe_workspace_size
    if which == "full":
        m = synth.moe(seed=0)
    elif which == "mixed-small":
        m = synth.moe(seed=1, E=6, hidden=256, inter=128, T=5, k=2, probs=(0.4, 0.3, 0.3))
    elif which == "mixed-8bit":
        m = synth.moe(seed=5, E=7, hidden=512, inter=256, T=9, k=3, probs=(0.25, 0.25, 0.5),
                      bits_choices=(2, 8, 4))
    else:
        m = synth.moe(seed=11, E=5, hidden=8192, inter=256, T=11, k=2, probs=(0.4, 0.3, 0.3))
    E = len(m["experts"])
    ws = torch.zeros(hq_moe_workspace_size(E, m["hidden"], m["inter"], m["T"], m["k"]),
                     dtype=torch.uint8, device="cuda")
    y, _ = run_moe(m, ws=ws)
    _check_stages(m, ws)
    want, bound, _ = oracle_moe(m)
    check(y, want, bound, which)


# ---------------------------------------------------------------- per-expert rotation signs
@pytest.mark.parametrize("hidden,inter,T,k", [(2048, 512, 32, 8), (256, 128, 9, 3), (8192, 256, 5, 2)])
def test_moe_per_expert_signs(hidden, inter, T, k):
    """Experts with their own rotation signs beside experts on the shared
    vectors: x rotated again per pair with the expert's signs_in, h with its
    signs_mid; stage-wise and end-to-end parity as above."""
    from bit_hadamard_rotated_b200 import hq_moe_workspace_size
    E = 16 if hidden == 2048 else 6
    m = synth.moe(seed=13 + hidden, E=E, hidden=hidden, inter=inter, T=T, k=k)
    rng = np.random.default_rng(hidden)
    for i, e in enumerate(m["experts"]):
        if i % 3 != 2:
            e["signs_in"] = synth.signs(rng, hidden)
        if i % 2 == 1:
            e["signs_mid"] = synth.signs(rng, inter)
    ws = torch.zeros(hq_moe_workspace_size(E, hidden, inter, T, k), dtype=torch.uint8, device="cuda")
    y, _ = run_moe(m, ws=ws)
    _check_stages(m, ws)
    want, bound, _ = oracle_moe(m)
    check(y, want, bound, "per-expert signs")
