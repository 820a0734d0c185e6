"""GPU parity of the int4 KV cache (hq_kv_append, hq_kv_attend) against the
fp64 oracle.

Codes, scales and minima are decided in IEEE single precision on both sides,
so they must match bit for bit.  The attention output is floating point; its
bound follows from the kernel's arithmetic, row by row:
  - a score is sum_c q_c s_c n_tc + sum_c q_c m_c with every product exact in
    the tensor cores (s = s_hi + s_lo, both halves times the code exact in
    fp16; q and m fp16) and 3d products summed in fp32, so
    |ds_t| <= g_d S with g_d = (3d + 4) 2^-24 and
    S = max_t sum_c |q_c| (|k_tc| + 2 |m_c|) / sqrt(d) (|s n| <= |k| + |m|);
  - a score error moves the softmax weights by p_t (ds_t - sum p ds), so the
    output moves by at most 2 g_d S sum_t p_t |v_t| = 2 g_d S base;
  - exp is the hardware 2^x (about 2^-22 relative), p v_scale enters as fp16
    hi + lo (2^-22) and the weighted values are summed in fp32 over at most
    T + 64 terms (inside a chunk, then across chunks): g_T = (T + 64) 2^-24
    relative to base.
  tol = (2 g_d S + g_T + 2^-20) base + 1e-6.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_hadamard_rotated_b200 import HqError, KVCache, hq_launch_count, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_hadamard_rotated_b200 import build
    build.build()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_codes(c: KVCache, T: int):
    """The GPU cache's first T tokens in the oracle's layout: kc [n_kv][T/32][d][32],
    vc [n_kv][T][d] (one code per byte), scales and minima as fp16."""
    nb = (T + 31) // 32
    kb = c.k_codes[:, :nb].cpu().numpy()                       # [h][b][tok][d/2]
    k = np.stack([kb & 15, kb >> 4], axis=-1).reshape(*kb.shape[:3], -1)   # [h][b][tok][d]
    vb = c.v_codes[:, :nb].cpu().numpy()                       # [h][b][d][16]
    v = np.stack([vb & 15, vb >> 4], axis=-1).reshape(*vb.shape[:3], 32)   # [h][b][d][tok]
    v = v.transpose(0, 1, 3, 2).reshape(c.n_kv_heads, nb * 32, c.head_dim)[:, :T]
    return dict(kc=k.transpose(0, 1, 3, 2), ks=c.k_scale[:, :nb].cpu().numpy(),
                km=c.k_min[:, :nb].cpu().numpy(), vc=v, vs=c.v_scale[:, :T].cpu().numpy(),
                vm=c.v_min[:, :T].cpu().numpy())


def assert_same_cache(g, o, T):
    nb = T // 32
    assert np.array_equal(g["kc"][:, :nb], o["kc"][:, :nb])
    assert np.array_equal(g["ks"][:, :nb].view(np.uint16), o["ks"][:, :nb].view(np.uint16))
    assert np.array_equal(g["km"][:, :nb].view(np.uint16), o["km"][:, :nb].view(np.uint16))
    assert np.array_equal(g["vc"][:, :T], o["vc"][:, :T])
    assert np.array_equal(g["vs"][:, :T].view(np.uint16), o["vs"][:, :T].view(np.uint16))
    assert np.array_equal(g["vm"][:, :T].view(np.uint16), o["vm"][:, :T].view(np.uint16))


def tolerance(cache, T, q, base):
    """The bound of the module docstring for every output element."""
    n_kv, _, d, _ = cache["kc"].shape
    nb = (T + 31) // 32
    km = np.abs(cache["km"][:, :nb].astype(np.float64))[..., None]
    K = (cache["ks"][:, :nb].astype(np.float64)[..., None] * cache["kc"][:, :nb]
         + cache["km"][:, :nb].astype(np.float64)[..., None])
    K = np.abs(K) + 2 * km                                                    # |k| + 2 |m|
    K = K.transpose(0, 1, 3, 2).reshape(n_kv, nb * 32, d)[:, :T]              # [h][t][c]
    n_q, n_heads, _ = q.shape
    G = n_heads // n_kv
    qa = np.abs(q.astype(np.float64))
    g_d = (3 * d + 4) * 2.0**-24
    g_T = (T + 64) * 2.0**-24
    tol = np.empty_like(base)
    for j in range(n_heads):
        S = (qa[:, j] @ K[j // G].T).max(axis=1) / np.sqrt(d)                  # [n_q]
        tol[:, j] = (2 * g_d * S[:, None] + g_T + 2.0**-20) * base[:, j] + 1e-6
    return tol


def check_attention(c, ocache, T, q, rows=None):
    out = c.attend(dev(q), T).cpu().numpy().astype(np.float64)
    qs = q if rows is None else q[rows]
    ref, base = oracle.kv_attend(ocache, T, qs)
    got = out if rows is None else out[rows]
    tol = tolerance(ocache, T, qs, base)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got))
    bad = err > tol
    assert not bad.any(), f"{bad.sum()} outside; worst err/tol {np.max(err / tol):.3g}"
    return float(np.max(err / tol))


def fill(c: KVCache, r, parts):
    """Append r's keys and values in the given [pos, pos + n) pieces."""
    for p0, n in parts:
        c.append(dev(r["k"][p0:p0 + n]), dev(r["v"][p0:p0 + n]), p0)


@pytest.mark.parametrize("d", [64, 128])
def test_append_bit_exact(d):
    r = synth.kv(T=256, n_kv=3, d=d, n_q=1, n_heads=3, seed=11)
    # degenerate groups: a key channel constant over block 1, a constant value
    # token, and one large-magnitude block
    r["k"][32:64, 0, 5] = np.float16(1.5)
    r["v"][7, 1, :] = np.float16(-2.0)
    r["k"][128:160, 2] *= np.float16(300)
    r["v"][200, 0] *= np.float16(500)
    c = KVCache(3, d, 320, "cuda")
    fill(c, r, [(0, 160), (160, 96)])
    torch.cuda.synchronize()
    o = oracle.kv_quantize(r["k"], r["v"])
    g = gpu_codes(c, 256)
    assert_same_cache(g, o, 256)
    assert np.all(g["kc"][0, 1, 5] == 0) and np.all(g["vc"][1, 7] == 0)
    # an append leaves other positions alone
    assert int(c.k_scale[:, 8:].abs().sum()) == 0 and int(c.v_scale[:, 256:].abs().sum()) == 0


@pytest.mark.parametrize("T_app,T,n_kv,d,n_q,n_heads", [
    (256, 256, 2, 128, 4, 8),       # 4 rows per kv head
    (256, 200, 2, 128, 1, 2),       # ragged context, one query
    (1024, 1000, 4, 64, 32, 16),    # 128 rows per kv head, d = 64
    (2048, 2048, 1, 128, 32, 8),    # 256 rows: two row groups
    (96, 33, 3, 128, 5, 3),         # G = 1, one token into the second block
    (32, 1, 1, 64, 1, 1),           # a single cached token
    (4096, 4096, 2, 128, 3, 14),    # odd row count (21 rows per kv head)
])
def test_attend_parity(T_app, T, n_kv, d, n_q, n_heads):
    r = synth.kv(T=T_app, n_kv=n_kv, d=d, n_q=n_q, n_heads=n_heads, seed=T_app + d + n_q)
    c = KVCache(n_kv, d, T_app, "cuda")
    fill(c, r, [(0, T_app)])
    o = oracle.kv_quantize(r["k"], r["v"])
    assert_same_cache(gpu_codes(c, T_app), o, T_app)
    n0 = hq_launch_count()
    check_attention(c, o, T, r["q"])
    assert hq_launch_count() - n0 == 2
    c.check_status()


def test_attend_large_scores():
    """Sharp softmax: queries x16 make scores of several hundred, so one token
    per row dominates and exp underflows for most others."""
    r = synth.kv(T=512, n_kv=2, d=128, n_q=4, n_heads=4, seed=7)
    r["q"] = (r["q"].astype(np.float32) * 16).astype(np.float16)
    c = KVCache(2, 128, 512, "cuda")
    fill(c, r, [(0, 512)])
    check_attention(c, oracle.kv_quantize(r["k"], r["v"]), 512, r["q"])


def test_attend_full_size_sampled():
    """The 32K-token, 4 kv-head, 32-query-token layer: the whole cache bit for
    bit, the attention of query tokens 0 and 31 (all 16 heads) against the
    oracle."""
    r = synth.kv(seed=0)
    c = KVCache(r["n_kv"], r["d"], r["T"], "cuda")
    fill(c, r, [(0, r["T"])])
    o = oracle.kv_quantize(r["k"], r["v"])
    assert_same_cache(gpu_codes(c, r["T"]), o, r["T"])
    check_attention(c, o, r["T"], r["q"], rows=[0, 31])


def test_attend_reuses_workspace_and_rejects_bad_args():
    r = synth.kv(T=128, n_kv=2, d=64, n_q=2, n_heads=4, seed=2)
    c = KVCache(2, 64, 128, "cuda")
    fill(c, r, [(0, 128)])
    o = oracle.kv_quantize(r["k"], r["v"])
    a = c.attend(dev(r["q"]), 128).cpu().numpy()
    b = c.attend(dev(r["q"]), 128).cpu().numpy()
    assert np.array_equal(a, b)                       # deterministic, workspace reused
    check_attention(c, o, 128, r["q"])
    with pytest.raises(HqError):
        c.append(dev(r["k"][:16]), dev(r["v"][:16]), 0)          # not whole blocks
    with pytest.raises(HqError):
        c.append(dev(r["k"][:32]), dev(r["v"][:32]), 128)        # past capacity
    with pytest.raises(HqError):
        c.attend(dev(r["q"]), 129)                                # more tokens than capacity
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(HqError):
        c.attend(dev(r["q"]), 128, workspace=small)
    n0 = hq_launch_count()
    out = c.attend(dev(r["q"][:0]), 128)
    assert out.shape == (0, 4, 64) and hq_launch_count() == n0
