"""Pins for the fp64 CPU oracle against facts that do not come from the oracle itself.

Each test checks one oracle function against something fixed independently of
its code: a brute-force dense Hadamard matrix built from its definition
H[i][j] = (-1)^popcount(i & j), scipy's Sylvester construction, exact algebraic
identities (H.H^T = K.I, orthogonality, involution), hand-derived fixtures in
tests/golden/, numpy's own bit unpacking, numpy's fp16 decoding, closed forms,
and an explicit dense W_eff = dequant(Q).H.diag(s)/sqrt(K) product built with
numpy/scipy.  A dropped term, a wrong sign or index, or a transposed operand
anywhere in the oracle fails at least one of them.
"""
import os

import numpy as np
import pytest
import scipy.linalg

import oracle
from bit_hadamard_rotated_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers (independent of the oracle)
def dense_hadamard(K):
    i = np.arange(K)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0)


def np_unpack(words, bits, n):
    """Codes from the little-endian bit stream via numpy.unpackbits."""
    stream = np.unpackbits(np.ascontiguousarray(words, dtype="<u4").view(np.uint8), bitorder="little")
    stream = stream[: bits * n].reshape(n, bits).astype(np.int64)
    return (stream << np.arange(bits)).sum(axis=1)


def np_pack(codes, bits):
    """Little-endian bit stream of the codes via numpy.packbits."""
    c = np.asarray(codes, dtype=np.int64)
    stream = ((c[:, None] >> np.arange(bits)) & 1).astype(np.uint8).reshape(-1)
    return np.packbits(stream, bitorder="little").view("<u4").astype(np.uint32)


def sign_vec(signs, K):
    return np.ones(K) if signs is None else np.where(np.asarray(signs) < 0, -1.0, 1.0)


def dense_weff(q, scales, bits, zero, M, K, signs):
    """Explicit effective weight W_eff = dequant(Q) . H_K . diag(s) / sqrt(K)."""
    codes = np.stack([np_unpack(q[m], bits, K) for m in range(M)])
    sc = np.repeat(np.asarray(scales, dtype=np.float16).astype(np.float64), 128, axis=1)
    Wq = sc * (codes - zero)
    H = scipy.linalg.hadamard(K).astype(np.float64)
    return Wq, Wq @ H @ np.diag(sign_vec(signs, K)) / np.sqrt(K)


# ---------------------------------------------------------------- fp16 decode
def test_f16_decode_every_pattern():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(int(p)) for p in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros too
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


# ---------------------------------------------------------------- FWHT
@pytest.mark.parametrize("K", [2, 4, 8, 16, 32, 64, 128, 256])
def test_fwht_equals_bruteforce_dense(K):
    rng = np.random.default_rng(K)
    v = rng.integers(-1000, 1000, size=K).astype(np.float64)
    assert np.array_equal(oracle.fwht(v), dense_hadamard(K) @ v)


@pytest.mark.parametrize("K", [512, 2048, 4096])
def test_fwht_equals_scipy_sylvester(K):
    rng = np.random.default_rng(K)
    v = rng.integers(-1000, 1000, size=K).astype(np.float64)
    assert np.array_equal(oracle.fwht(v), scipy.linalg.hadamard(K) @ v)


def test_hadamard_hht_is_k_identity():
    K = 64
    H = np.stack([oracle.fwht(np.eye(K)[i]) for i in range(K)], axis=1)
    assert np.array_equal(H @ H.T, K * np.eye(K))
    assert np.array_equal(H, H.T)


@pytest.mark.parametrize("K", [128, 512, 2048, 8192])
def test_rotation_preserves_norm_and_inverts(K):
    rng = np.random.default_rng(7 + K)
    x = rng.standard_normal(K)
    s = synth.signs(rng, K)
    xr = oracle.rotate(x, s)
    assert abs(np.linalg.norm(xr) - np.linalg.norm(x)) <= 1e-13 * np.linalg.norm(x)
    # inverse: diag(s) H x' / sqrt(K) == x
    back = sign_vec(s, K) * oracle.fwht(xr) / np.sqrt(K)
    assert np.max(np.abs(back - x)) <= 1e-12


@pytest.mark.parametrize("K", [128, 4096])
def test_rotation_closed_forms(K):
    e0 = np.zeros(K)
    e0[0] = 1.0
    assert np.allclose(oracle.rotate(e0), np.full(K, 1 / np.sqrt(K)), rtol=0, atol=1e-15)
    one = np.ones(K)
    want = np.zeros(K)
    want[0] = np.sqrt(K)
    assert np.allclose(oracle.rotate(one), want, rtol=0, atol=1e-12)


def test_rotation_hand_fixtures():
    for line in open(os.path.join(GOLDEN, "hadamard_small.txt")):
        if line.startswith("#") or not line.strip():
            continue
        K, s, x, want = [f.split() for f in line.split("|")]
        K = int(K[0])
        s = np.array([int(v) for v in s], np.int8)
        x = np.array([float(v) for v in x])
        got = oracle.rotate(x, s) * np.sqrt(K)
        assert np.allclose(got, [float(v) for v in want], rtol=0, atol=1e-12), line


def test_rotation_sign_convention_and_null_signs():
    K = 256
    rng = np.random.default_rng(3)
    x = rng.standard_normal(K)
    s_pos = np.ones(K, np.int8)
    s_mixed = np.array(rng.integers(-3, 4, size=K), np.int8)  # 0 counts as +1, any negative as -1
    assert np.array_equal(oracle.rotate(x, None), oracle.rotate(x, s_pos))
    H = scipy.linalg.hadamard(K)
    want = H @ (np.where(s_mixed < 0, -1.0, 1.0) * x) / np.sqrt(K)
    assert np.allclose(oracle.rotate(x, s_mixed), want, rtol=0, atol=1e-12)


def test_rotation_of_fp16_input_reads_fp16_bits():
    K = 512
    rng = np.random.default_rng(11)
    x16 = rng.standard_normal((3, K)).astype(np.float16)
    s = synth.signs(rng, K)
    got = oracle.rotate(x16, s)
    H = scipy.linalg.hadamard(K)
    want = (H @ (sign_vec(s, K)[:, None] * x16.astype(np.float64).T)).T / np.sqrt(K)
    assert np.allclose(got, want, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- packing
def test_unpack_hand_fixtures():
    n = 0
    for line in open(os.path.join(GOLDEN, "unpack_patterns.txt")):
        if line.startswith("#") or not line.strip():
            continue
        bits, words, codes = [f.split() for f in line.split("|")]
        bits = int(bits[0])
        words = np.array([int(w, 16) for w in words], np.uint32)
        codes = np.array([int(c) for c in codes])
        assert np.array_equal(oracle.unpack(words, bits, codes.size), codes), line
        assert np.array_equal(oracle.pack(codes, bits), words), line
        n += 1
    assert n >= 8


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_unpack_matches_numpy_unpackbits(bits):
    rng = np.random.default_rng(100 + bits)
    n = 32 * 97
    words = rng.integers(0, 2**32, size=n * bits // 32, dtype=np.uint64).astype(np.uint32)
    assert np.array_equal(oracle.unpack(words, bits, n), np_unpack(words, bits, n))


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_pack_unpack_round_trip(bits):
    rng = np.random.default_rng(200 + bits)
    codes = rng.integers(0, 1 << bits, size=4096).astype(np.uint8)
    words = oracle.pack(codes, bits)
    assert words.size == 4096 * bits // 32
    assert np.array_equal(oracle.unpack(words, bits, codes.size), codes)
    assert np.array_equal(np_unpack(words, bits, codes.size), codes)


def test_three_bit_straddling_codes_single_bits():
    """A single set stream bit p in a 3-bit triplet lands in code p//3 as 1 << (p%3)."""
    for p in range(96):
        words = np.zeros(3, np.uint32)
        words[p // 32] = np.uint32(1 << (p % 32))
        codes = oracle.unpack(words, 3, 32)
        want = np.zeros(32, np.int64)
        want[p // 3] = 1 << (p % 3)
        assert np.array_equal(codes, want), p


def test_bit_planes_match_numpy_and_round_trip():
    """2-bit codes in the bit-plane layout: code 32 s + i = bit i of word 2s
    plus twice bit i of word 2s + 1 (numpy's unpackbits, little bit order),
    single-bit fixtures, and the round trip."""
    rng = np.random.default_rng(17)
    words = rng.integers(0, 2**32, size=2 * 40, dtype=np.uint64).astype(np.uint32)
    bits = np.unpackbits(words.view(np.uint8), bitorder="little").reshape(-1, 32)   # [word][bit]
    want = (bits[0::2] + 2 * bits[1::2]).reshape(-1)
    got = oracle.unpack_planes2(words, 40 * 32)
    assert np.array_equal(got, want)
    assert np.array_equal(oracle.pack_planes2(got), words)
    one = np.zeros(4, np.uint32)
    one[3] = np.uint32(1 << 5)                     # plane 1 of span 1, bit 5: code 37 = 2
    c = oracle.unpack_planes2(one, 64)
    assert c[37] == 2 and c.sum() == 2
    one[2] = np.uint32(1 << 5)                     # plane 0 too: code 37 = 3
    assert oracle.unpack_planes2(one, 64)[37] == 3


def test_linear_bit_planes_equals_packed_linear():
    """The linear over bit-plane words equals the linear over the same codes in
    the packed 2-bit stream (codes rebuilt through numpy's unpackbits)."""
    d = synth.linear(24, 256, 2, 2, seed=9)
    rng = np.random.default_rng(4)
    planes = rng.integers(0, 2**32, size=(24, 256 // 16), dtype=np.uint64).astype(np.uint32)
    bits = np.unpackbits(planes.view(np.uint8), axis=1, bitorder="little").reshape(24, -1, 2, 32)
    codes = (bits[:, :, 0] + 2 * bits[:, :, 1]).reshape(24, 256).astype(np.uint8)
    packed = np.stack([np_pack(codes[m], 2) for m in range(24)])
    y_p, b_p = oracle.linear(2, 24, 256, 2, planes, d["scales"], d["signs"], d["x"], planes=True)
    y_q, b_q = oracle.linear(2, 24, 256, 2, packed, d["scales"], d["signs"], d["x"])
    assert np.array_equal(y_p, y_q) and np.array_equal(b_p, b_q)


# ---------------------------------------------------------------- dequant + dot
def _mk(bits, M, K, N, seed, signs=True):
    d = synth.linear(M, K, bits, N, seed=seed)
    if not signs:
        d["signs"] = None
    return d


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_zero_codes_give_exact_zero(bits):
    M, K, N = 8, 256, 2
    d = _mk(bits, M, K, N, 1)
    z = 1 << (bits - 1)
    q = np.stack([oracle.pack(np.full(K, z, np.uint8), bits) for _ in range(M)])
    y, b = oracle.linear(bits, M, K, z, q, d["scales"], d["signs"], d["x"])
    assert np.array_equal(y, np.zeros((N, M)))
    assert np.array_equal(b, np.zeros((N, M)))


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_constant_codes_closed_form(bits):
    """q = z+1 everywhere and one constant scale c: y_m = c . sum_k x'_k."""
    M, K, N = 4, 512, 3
    d = _mk(bits, M, K, N, 2)
    z = 1 << (bits - 1)
    c = np.float16(0.0117)
    q = np.stack([oracle.pack(np.full(K, z + 1, np.uint8), bits) for _ in range(M)])
    sc = np.full((M, K // 128), c, np.float16)
    y, _ = oracle.linear(bits, M, K, z, q, sc, d["signs"], d["x"])
    H = scipy.linalg.hadamard(K)
    xr = (H @ (sign_vec(d["signs"], K)[:, None] * d["x"].astype(np.float64).T)).T / np.sqrt(K)
    want = float(c) * xr.sum(axis=1)
    assert np.allclose(y, np.repeat(want[:, None], M, axis=1), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("bits", [2, 4])
def test_unit_input_gives_row_sums(bits):
    """s = 1 and x = e0: x' = 1/sqrt(K) everywhere, so y_m = sum_k w_mk / sqrt(K)."""
    M, K = 16, 256
    d = _mk(bits, M, K, 1, 3)
    x = np.zeros((1, K), np.float16)
    x[0, 0] = 1.0
    y, _ = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], None, x)
    Wq, _ = dense_weff(d["q"], d["scales"], bits, d["zero"], M, K, None)
    assert np.allclose(y[0], Wq.sum(axis=1) / np.sqrt(K), rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("bits,M,K,N", [(2, 64, 512, 3), (3, 40, 256, 2), (4, 33, 512, 4),
                                         (8, 17, 128, 5), (3, 8, 512, 1)])
def test_linear_equals_explicit_dense_weff(bits, M, K, N):
    d = _mk(bits, M, K, N, 10 + bits)
    y, b = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    Wq, Weff = dense_weff(d["q"], d["scales"], bits, d["zero"], M, K, d["signs"])
    xd = d["x"].astype(np.float64)
    want = xd @ Weff.T
    assert np.allclose(y, want, rtol=1e-12, atol=1e-12)
    # the tolerance base: sum_k |w_k x'_k| with x' rotated explicitly
    H = scipy.linalg.hadamard(K)
    xr = (H @ (sign_vec(d["signs"], K)[:, None] * xd.T)).T / np.sqrt(K)
    want_b = np.abs(Wq[None, :, :] * xr[:, None, :]).sum(axis=2)
    assert np.allclose(b, want_b, rtol=1e-12, atol=1e-12)
    assert np.all(np.abs(y) <= b * (1 + 1e-12))


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_linear_per_group_zeros_equals_dense(bits):
    """Per-group zero points (the GPTQ form, one uint8 per row and group):
    the oracle's linear equals x' . (scale (q - z[m][k/128]))^T built densely
    with numpy, and a constant zeros array equals the scalar zero."""
    M, K, N = 20, 512, 3
    d = _mk(bits, M, K, N, 40 + bits)
    rng = np.random.default_rng(bits)
    zeros = rng.integers(0, 1 << bits, size=(M, K // 128)).astype(np.uint8)
    y, b = oracle.linear(bits, M, K, 0, d["q"], d["scales"], d["signs"], d["x"], zeros=zeros)
    codes = np.stack([np_unpack(d["q"][m], bits, K) for m in range(M)])
    sc = np.repeat(np.asarray(d["scales"], dtype=np.float16).astype(np.float64), 128, axis=1)
    Wq = sc * (codes - np.repeat(zeros.astype(np.int64), 128, axis=1))
    H = scipy.linalg.hadamard(K).astype(np.float64)
    xr = (H @ (sign_vec(d["signs"], K)[:, None] * d["x"].astype(np.float64).T)).T / np.sqrt(K)
    assert np.allclose(y, xr @ Wq.T, rtol=1e-12, atol=1e-12)
    assert np.allclose(b, np.abs(Wq[None] * xr[:, None, :]).sum(axis=2), rtol=1e-12, atol=1e-12)
    zc = np.full((M, K // 128), d["zero"], np.uint8)
    y2, b2 = oracle.linear(bits, M, K, 0, d["q"], d["scales"], d["signs"], d["x"], zeros=zc)
    y3, b3 = oracle.linear(bits, M, K, d["zero"], d["q"], d["scales"], d["signs"], d["x"])
    assert np.array_equal(y2, y3) and np.array_equal(b2, b3)


def test_linear_row_ranges_compose():
    d = _mk(4, 50, 256, 2, 21)
    y_all, b_all = oracle.linear(4, 50, 256, 8, d["q"], d["scales"], d["signs"], d["x"])
    y_t, b_t = oracle.linear(4, 50, 256, 8, d["q"], d["scales"], d["signs"], d["x"], threads=3)
    assert np.array_equal(y_all, y_t) and np.array_equal(b_all, b_t)


# ---------------------------------------------------------------- MoE composition
def _small_moe(seed, E=6, hidden=256, inter=128, T=5, k=2, probs=(0.4, 0.3, 0.3)):
    return synth.moe(seed=seed, E=E, hidden=hidden, inter=inter, T=T, k=k, probs=probs)


def _dense_expert_chain(e, x_row, s_in, s_mid, hidden, inter):
    s_in = e.get("signs_in", s_in) if e.get("signs_in") is not None else s_in
    s_mid = e.get("signs_mid", s_mid) if e.get("signs_mid") is not None else s_mid
    _, Wg = dense_weff(e["q_gate"], e["s_gate"], e["bits"], e["zero"], inter, hidden, s_in)
    _, Wu = dense_weff(e["q_up"], e["s_up"], e["bits"], e["zero"], inter, hidden, s_in)
    _, Wd = dense_weff(e["q_down"], e["s_down"], e["bits"], e["zero"], hidden, inter, s_mid)
    g = Wg @ x_row
    u = Wu @ x_row
    h = g * u / (1.0 + np.exp(-g))
    return Wd @ h, h


def test_moe_top1_equals_dense_chain():
    m = _small_moe(31, k=1)
    T = m["T"]
    ids = m["topk_ids"]
    w1 = np.ones((T, 1), np.float32)
    y, b, h = oracle.moe(m["experts"], m["hidden"], m["inter"], m["x"], ids, w1, m["s_in"],
                         m["s_mid"], want_h=True)
    for t in range(T):
        e = m["experts"][int(ids[t, 0])]
        want, hw = _dense_expert_chain(e, m["x"][t].astype(np.float64), m["s_in"], m["s_mid"],
                                       m["hidden"], m["inter"])
        assert np.allclose(y[t], want, rtol=1e-11, atol=1e-12)
        assert np.allclose(h[t], hw, rtol=1e-11, atol=1e-12)
        assert np.all(np.abs(y[t]) <= b[t] * (1 + 1e-12))


def test_moe_weighted_combine_order_and_weights():
    m = _small_moe(32, k=3)
    y, _, _ = oracle.moe(m["experts"], m["hidden"], m["inter"], m["x"], m["topk_ids"], m["topk_w"],
                         m["s_in"], m["s_mid"])
    for t in range(m["T"]):
        want = np.zeros(m["hidden"])
        for j in range(m["k"]):
            e = m["experts"][int(m["topk_ids"][t, j])]
            d, _ = _dense_expert_chain(e, m["x"][t].astype(np.float64), m["s_in"], m["s_mid"],
                                       m["hidden"], m["inter"])
            want += float(m["topk_w"][t, j]) * d
        assert np.allclose(y[t], want, rtol=1e-11, atol=1e-12)


def test_moe_identical_experts_reduce_to_one():
    m = _small_moe(33, k=4, E=5)
    same = [m["experts"][0]] * m["E"]
    y, _, _ = oracle.moe(same, m["hidden"], m["inter"], m["x"], m["topk_ids"], m["topk_w"],
                         m["s_in"], m["s_mid"])
    for t in range(m["T"]):
        want, _ = _dense_expert_chain(same[0], m["x"][t].astype(np.float64), m["s_in"], m["s_mid"],
                                      m["hidden"], m["inter"])
        assert np.allclose(y[t], want, rtol=1e-6, atol=1e-9)  # weights sum to 1 in fp32


def test_moe_bound_base_for_several_slots():
    """The MoE tolerance base, bound_t[i] = sum_j |topk_w[t][j]| sum_k |Wq_down[i][k] h'_k|,
    rebuilt from dense numpy chains at k = 3 and 8 with some negative routing
    weights (so a dropped |.| or a dropped weight changes it), to 1e-12."""
    for seed, k in ((34, 3), (35, 8)):
        m = _small_moe(seed, k=k, E=9)
        w = m["topk_w"].copy()
        w[:, 1] *= -1.0
        y, b, _ = oracle.moe(m["experts"], m["hidden"], m["inter"], m["x"], m["topk_ids"], w,
                             m["s_in"], m["s_mid"])
        H = scipy.linalg.hadamard(m["inter"]).astype(np.float64)
        for t in range(m["T"]):
            want = np.zeros(m["hidden"])
            want_y = np.zeros(m["hidden"])
            for j in range(k):
                e = m["experts"][int(m["topk_ids"][t, j])]
                d, h = _dense_expert_chain(e, m["x"][t].astype(np.float64), m["s_in"], m["s_mid"],
                                           m["hidden"], m["inter"])
                hr = H @ (sign_vec(m["s_mid"], m["inter"]) * h) / np.sqrt(m["inter"])
                Wq, _ = dense_weff(e["q_down"], e["s_down"], e["bits"], e["zero"], m["hidden"],
                                   m["inter"], m["s_mid"])
                want += abs(float(w[t, j])) * np.abs(Wq * hr[None, :]).sum(axis=1)
                want_y += float(w[t, j]) * d
            assert np.allclose(b[t], want, rtol=1e-12, atol=1e-14)
            assert np.allclose(y[t], want_y, rtol=1e-11, atol=1e-12)
            assert np.all(np.abs(y[t]) <= b[t] * (1 + 1e-12))


def test_moe_per_expert_signs_equals_dense_chain():
    """Experts with their own rotation signs (some with signs_in, some with
    signs_mid, some with both, the rest on the shared vectors): every token's
    output equals the weighted sum of dense chains built with each expert's
    signs."""
    m = _small_moe(36, k=3, E=6)
    rng = np.random.default_rng(36)
    for i, e in enumerate(m["experts"]):
        if i % 3 != 2:
            e["signs_in"] = synth.signs(rng, m["hidden"])
        if i % 2 == 1:
            e["signs_mid"] = synth.signs(rng, m["inter"])
    y, b, _ = oracle.moe(m["experts"], m["hidden"], m["inter"], m["x"], m["topk_ids"], m["topk_w"],
                         m["s_in"], m["s_mid"])
    for t in range(m["T"]):
        want = np.zeros(m["hidden"])
        for j in range(m["k"]):
            e = m["experts"][int(m["topk_ids"][t, j])]
            d, _ = _dense_expert_chain(e, m["x"][t].astype(np.float64), m["s_in"], m["s_mid"],
                                       m["hidden"], m["inter"])
            want += float(m["topk_w"][t, j]) * d
        assert np.allclose(y[t], want, rtol=1e-11, atol=1e-12)
        assert np.all(np.abs(y[t]) <= b[t] * (1 + 1e-12))


# ---------------------------------------------------------------- nibble-split screened readout
def _merged_codes(r):
    hi = np.stack([np_unpack(r["hi"][m], 4, r["K"]) for m in range(r["V"])])
    lo = np.stack([np_unpack(r["lo"][m], 4, r["K"]) for m in range(r["V"])])
    return hi, lo


@pytest.mark.parametrize("topk", [1, 5])
def test_readout_exact_topk_and_screen_decomposition(topk):
    """The oracle's readout: exact logits equal a dense numpy product of the
    merged 8-bit codes (16 hi + lo); the screen e plus the low-nibble
    remainder sum scale (lo - 7.5) x' (numpy) is the exact logit; the returned
    ids are the topk of the exact logits (numpy's stable descending order), all
    of them candidates."""
    r = synth.readout(V=300, K=256, N=2, seed=topk)
    ids, out, cand, ya, ea = oracle.readout(r["hi"], r["lo"], r["scales"], r["signs"], r["V"], r["K"],
                                            r["zero"], r["x"], topk, want_all=True)
    hi, lo = _merged_codes(r)
    sc = np.repeat(r["scales"].astype(np.float64), 128, axis=1)
    W = sc * (16 * hi + lo - r["zero"])
    H = scipy.linalg.hadamard(r["K"]).astype(np.float64)
    xr = (H @ (sign_vec(r["signs"], r["K"])[:, None] * r["x"].astype(np.float64).T)).T / np.sqrt(r["K"])
    assert np.allclose(ya, xr @ W.T, rtol=1e-12, atol=1e-12)
    rem = xr @ (sc * (lo - 7.5)).T
    assert np.allclose(ea + rem, ya, rtol=1e-11, atol=1e-11)
    for n in range(2):
        order = np.argsort(-ya[n], kind="stable")[:topk]
        assert ids[n].tolist() == order.tolist()
        assert np.allclose(out[n], ya[n, order], rtol=0, atol=0)
        assert np.all(cand[n, order] == 1)


def test_readout_screen_band():
    """beta = 0: the candidates are exactly the rows whose screen reaches the
    topk-th largest screen (numpy); a huge beta keeps every row."""
    r = synth.readout(V=400, K=256, N=1, seed=9)
    _, _, cand, _, ea = oracle.readout(r["hi"], r["lo"], r["scales"], r["signs"], r["V"], r["K"], r["zero"],
                                       r["x"], 7, beta=0.0, want_all=True)
    tau = np.sort(ea[0])[::-1][6]
    assert np.array_equal(cand[0].astype(bool), ea[0] >= tau)
    _, _, cand2, _, _ = oracle.readout(r["hi"], r["lo"], r["scales"], r["signs"], r["V"], r["K"], r["zero"],
                                       r["x"], 7, beta=1e9)
    assert np.all(cand2 == 1)


# ---------------------------------------------------------------- int4 KV cache
def test_kv_quant_group_nearest_code_and_range():
    """Each 4-bit code of a group is a nearest point of the grid mn + scale c
    (brute force over the 16 codes, in float64 of the float32 decision), the
    scale is float16((float32 max - float32 min) / 15) and mn float16(min)
    (numpy's float32 and float16 roundings)."""
    r = synth.kv(T=64, n_kv=2, d=32, n_q=1, n_heads=2, seed=3)
    cache = oracle.kv_quantize(r["k"], r["v"])
    for h in range(2):
        for b in range(2):
            for c in range(32):
                x = r["k"][32 * b:32 * b + 32, h, c].astype(np.float32)
                s = np.float16((x.max() - x.min()) / np.float32(15))
                assert cache["ks"][h, b, c] == s and cache["km"][h, b, c] == np.float16(x.min())
                grid = np.float64(cache["km"][h, b, c]) + np.float64(s) * np.arange(16)
                codes = cache["kc"][h, b, c]
                err = np.abs(x[:, None].astype(np.float64) - grid[None, :])
                assert np.all(err[np.arange(32), codes] <= err.min(axis=1) + 1e-6 * np.abs(grid).max())
        for t in range(64):
            x = r["v"][t, h].astype(np.float32)
            s = np.float16((x.max() - x.min()) / np.float32(15))
            assert cache["vs"][h, t] == s and cache["vm"][h, t] == np.float16(x.min())
            assert cache["vc"][h, t].max() <= 15


def test_kv_attend_equals_dense_softmax_attention():
    """The oracle's attention over the int4 cache equals a dense numpy softmax
    attention over the dequantised keys and values (grouped heads)."""
    r = synth.kv(T=96, n_kv=2, d=32, n_q=3, n_heads=4, seed=5)
    cache = oracle.kv_quantize(r["k"], r["v"])
    out, base = oracle.kv_attend(cache, 96, r["q"])
    K = (cache["ks"].astype(np.float64)[..., None] * cache["kc"] + cache["km"].astype(np.float64)[..., None])
    K = K.transpose(0, 1, 3, 2).reshape(2, 96, 32)                       # [h][t][c]
    V = cache["vs"].astype(np.float64)[..., None] * cache["vc"] + cache["vm"].astype(np.float64)[..., None]
    q = r["q"].astype(np.float64)
    for i in range(3):
        for j in range(4):
            h = j // 2
            s = K[h] @ q[i, j] / np.sqrt(32)
            p = np.exp(s - s.max())
            p /= p.sum()
            assert np.allclose(out[i, j], p @ V[h], rtol=1e-12, atol=1e-12)
            assert np.allclose(base[i, j], p @ np.abs(V[h]), rtol=1e-12, atol=1e-12)
    # a prefix of T = 75 tokens (not a whole number of blocks): only tokens
    # 0..74 enter the softmax
    out3, _ = oracle.kv_attend(cache, 75, r["q"])
    for i in range(3):
        for j in range(4):
            h = j // 2
            s = K[h, :75] @ q[i, j] / np.sqrt(32)
            p = np.exp(s - s.max())
            p /= p.sum()
            assert np.allclose(out3[i, j], p @ V[h, :75], rtol=1e-12, atol=1e-12)
    # equal keys: uniform weights, the output is the values' mean
    c2 = dict(cache, kc=np.zeros_like(cache["kc"]), km=np.zeros_like(cache["km"]))
    out2, _ = oracle.kv_attend(c2, 96, r["q"])
    assert np.allclose(out2[0, 0], V[0].mean(axis=0), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- routing inputs
def test_routing_weights_and_ties():
    rng = np.random.default_rng(5)
    _, ids, w = synth.routing(rng, 32, 256, 8)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-6)
    assert np.all(np.diff(w, axis=1) <= 0)          # descending logits -> descending weights
    for t in range(32):
        assert len(set(ids[t].tolist())) == 8
    # ties: equal logits keep the lower index first
    logits = np.zeros((1, 16), np.float32)
    order = np.argsort(-logits, axis=1, kind="stable")[:, :4]
    assert order.tolist() == [[0, 1, 2, 3]]


# ---------------------------------------------------------------- rotated round-to-nearest quantiser
def test_f64_to_f16_matches_numpy():
    """The oracle's double -> binary16 rounding against numpy's (ties to even),
    over normals, subnormals, exact ties and the overflow edge."""
    rng = np.random.default_rng(3)
    v = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.uniform(-9, 5, 20000),
        (np.arange(1, 3000) + 0.5) * 2.0**-24,           # subnormal ties
        1.0 + (np.arange(0, 2048) + 0.5) * 2.0**-10,     # normal ties at [1, 3)
        [0.0, -0.0, 65504.0, 65519.99, 2.0**-14, 2.0**-14 - 2.0**-25, 2.0**-25, -2.0**-25],
    ])
    with np.errstate(over="ignore"):
        want = v.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f64_to_f16(x) for x in v], np.uint16)
    assert np.array_equal(got, want)


def _rand_weights(M, K, seed, outliers=True):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((M, K)) * 0.02
    if outliers:
        W[:, rng.choice(K, max(1, K // 100), replace=False)] *= 20.0
    return W.astype(np.float32).astype(np.float64), synth.signs(rng, K)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_quantize_rotation_grid_and_packing(bits):
    """hqo_quantize against what fixes it independently: the rotated row equals
    W diag(s) H / sqrt(K) built with scipy; every code is a nearest point of
    its group's grid scale (q - 2^(b-1)), q in [0, 2^b - 1] (brute force over
    all codes); the group's largest |r| lands on the top code if positive, on
    code 0 if negative (code 1 only when the fp16 scale rounded up, which
    moves -2^(b-1) scale past it); the grid spans that largest |r| to within
    the fp16 rounding of the scale; the words unpack (numpy) to those codes."""
    M, K = 24, 512
    W, s = _rand_weights(M, K, 70 + bits)
    q, sc, r = oracle.quantize(W, bits, s, want_rotated=True)
    H = scipy.linalg.hadamard(K).astype(np.float64)
    assert np.allclose(r, W @ np.diag(sign_vec(s, K)) @ H / np.sqrt(K), rtol=1e-12, atol=1e-15)
    z, qmax = 1 << (bits - 1), (1 << bits) - 1
    codes = np.stack([np_unpack(q[m], bits, K) for m in range(M)])
    scale = np.repeat(sc.astype(np.float64), 128, axis=1)
    err = np.abs(r - scale * (codes - z))
    grid = scale[..., None] * (np.arange(qmax + 1)[None, None, :] - z)
    best = np.min(np.abs(r[..., None] - grid), axis=2)
    assert np.all(err <= best * (1 + 1e-12) + 1e-300)
    for m in range(M):
        for g in range(K // 128):
            seg = r[m, 128 * g:128 * g + 128]
            i = int(np.argmax(np.abs(seg)))
            a = abs(seg[i])
            c = codes[m, 128 * g + i]
            span = float(sc[m, g]) * qmax / 2
            assert abs(span - a) <= 2.0**-11 * max(span, a)
            if seg[i] > 0:
                assert c == qmax
            else:
                assert c == 0 or (c == 1 and span > a)
    assert np.all(err <= scale / 2 * (1 + 2.0**(bits - 10)))


def test_quantize_zero_rows_and_tiny_groups():
    """A zero row quantises to scale 0 and the zero-point code; a group whose
    scale underflows fp16 does the same; the rest of the row is unaffected."""
    K, bits = 256, 4
    W = np.zeros((2, K))
    W[1, :] = 1e-3
    W[1, 0] += 1.0
    q, sc, r = oracle.quantize(W, bits, None, want_rotated=True)
    assert np.all(sc[0] == 0) and np.all(np_unpack(q[0], bits, K) == 8)
    assert np.all(sc[1] > 0)
    W2 = np.full((1, K), 1e-12)
    q2, sc2, _ = oracle.quantize(W2, bits, None)
    assert np.all(sc2 == 0) and np.all(np_unpack(q2[0], bits, K) == 8)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_quantize_then_linear_approximates_dense_product(bits):
    """y = dequant(quantize(W)) x' with the oracle's own linear is W x (numpy,
    dense) up to the quantisation bound sum_g scale_g / 2 (1 + 2^(b-10))
    sum_{k in g} |x'_k|: the rotation cancels (W x = W_rot x') and every
    rotated weight is within half a grid step."""
    M, K, N = 40, 1024, 3
    W, s = _rand_weights(M, K, 80 + bits)
    q, sc, _ = oracle.quantize(W, bits, s)
    rng = np.random.default_rng(9)
    x = rng.standard_normal((N, K)).astype(np.float16)
    y, _ = oracle.linear(bits, M, K, 1 << (bits - 1), q, sc, s, x)
    xd = x.astype(np.float64)
    want = xd @ W.T
    H = scipy.linalg.hadamard(K).astype(np.float64)
    xr = (H @ (sign_vec(s, K)[:, None] * xd.T)).T / np.sqrt(K)
    ax = np.abs(xr).reshape(N, K // 128, 128).sum(axis=2)          # [N][G]
    bound = (ax @ (sc.astype(np.float64).T / 2)) * (1 + 2.0**(bits - 10))  # [N][M]
    assert np.all(np.abs(y - want) <= bound * (1 + 1e-9) + 1e-12)
    # and the bound is not vacuous: the error is a sizeable part of it somewhere
    assert np.max(np.abs(y - want) / bound) > 0.05
