"""Pins of the oracle against facts that do not come from the oracle itself:
format tables fixed by the OCP specs (golden fixtures) and by torch's float8
conversion, exact rational arithmetic, brute-force sorting, textbook/numpy
routines for the special cases, and invariants of the method."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    for line in open(os.path.join(GOLD, name), encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, *v = line.split()
        out[k] = [float(x) for x in v]
    return out


# ---------------------------------------------------------------- formats

def test_e4m3_table_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_e4m3_golden_constants():
    g = _golden("e2m1_e4m3_formats.txt")
    vals = [oracle.e4m3_value(c) for c in range(0x7F)]
    assert max(vals) == g["e4m3_max"][0]
    assert min(v for v in vals if v > 0) == g["e4m3_min_subnormal"][0]
    assert oracle.e4m3_value(0x08) == g["e4m3_min_normal"][0]


def test_e2m1_golden_values():
    g = _golden("e2m1_e4m3_formats.txt")
    assert [oracle.e2m1_value(i) for i in range(8)] == g["e2m1_magnitudes"]
    assert [oracle.e2m1_value(8 + i) for i in range(8)] == [-v for v in g["e2m1_magnitudes"]]
    assert math.copysign(1.0, oracle.e2m1_value(8)) == -1.0


def test_e4m3_encode_matches_torch_rne():
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.uniform(0, 448, 20000), np.exp(rng.uniform(math.log(2.0**-12), math.log(448.0), 20000)),
        [0.0, 2.0**-10, 2.0**-10 * 1.0000001, 2.0**-10 * 0.9999999, 2.0**-9, 3 * 2.0**-10, 448.0, 440.0, 432.0],
    ]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(x)) for x in v], np.uint8)
    assert np.array_equal(ref, got)


def test_e4m3_encode_saturates():
    for v in [448.0, 449.0, 463.9, 464.0, 500.0, 1e6, 1e30]:
        assert oracle.e4m3_encode(v) == 0x7E


# ---------------------------------------------------------------- quantiser

E2M1 = [Fraction(x) for x in ("0", "1/2", "1", "3/2", "2", "3", "4", "6")]


def _rne_index(q: Fraction) -> int:
    """round-to-nearest-even of an exact non-negative quotient on the E2M1 grid, saturating"""
    best, bd = 0, None
    for i, v in enumerate(E2M1):
        d = abs(q - v)
        if bd is None or d < bd or (d == bd and i % 2 == 0):
            best, bd = i, d
    return best


def _pos_scales():
    return [c for c in range(1, 0x7F) if oracle.e4m3_value(c) > 0]


def _unpack(codes, d):
    lo = codes & 15
    hi = codes >> 4
    return np.stack([lo, hi], -1).reshape(codes.shape[0], d)


def test_quantize_boundaries_exact_rational():
    """For every positive E4M3 scale s, inputs at s*m and one ulp either side
    of every rounding midpoint m; the expected code is RNE of the exact
    quotient x/s, computed with Fractions."""
    mids = [Fraction(1, 4), Fraction(3, 4), Fraction(5, 4), Fraction(7, 4), Fraction(5, 2), Fraction(7, 2),
            Fraction(5), Fraction(6)]
    rows, expect, scale_codes = [], [], []
    for sc in _pos_scales():
        s = Fraction(oracle.e4m3_value(sc))
        vals = []
        for m in mids:
            x = np.float32(float(s * m))
            assert Fraction(float(x)) == s * m  # exact in fp32
            vals += [x, np.nextafter(x, np.float32(np.inf)), np.nextafter(x, np.float32(0))]
        vals = vals[:30]
        vals = [v for v in vals if Fraction(float(v)) <= 6 * s]
        while len(vals) < 31:
            vals.append(np.float32(0))
        row = np.array([np.float32(float(6 * s))] + vals, np.float32)  # amax = 6s -> scale s exactly
        sign = np.where(np.arange(32) % 3 == 1, -1, 1).astype(np.float32)
        row = row * sign
        rows.append(row)
        scale_codes.append(sc)
        exp = []
        for x in row:
            idx = _rne_index(Fraction(abs(float(x))) / s)
            exp.append((8 if np.signbit(x) else 0) | idx)
        expect.append(exp)
    x = np.stack(rows)
    codes, scales, bad = oracle.quantize_fp4(x)
    assert bad == 0
    assert np.array_equal(scales[:, 0], np.array(scale_codes, np.uint8))
    assert np.array_equal(_unpack(codes, 32), np.array(expect, np.uint8))


def test_quantize_scale_rule_exact():
    """scale = RNE_E4M3(amax / 6 in fp32), checked against torch's float8 RNE cast of the fp32 quotient"""
    rng = np.random.default_rng(1)
    amax = np.exp(rng.uniform(math.log(1e-4), math.log(2000.0), 3000)).astype(np.float32)
    x = np.zeros((len(amax), 32), np.float32)
    x[:, 5] = amax
    x[:, 7] = -amax * np.float32(0.5)
    _, scales, _ = oracle.quantize_fp4(x)
    q = (torch.from_numpy(amax) / 6.0)
    ref = q.clamp(max=448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(scales[:, 0], ref)


def test_quantize_zero_and_negative_zero():
    x = np.zeros((2, 64), np.float32)
    x[1] = -0.0
    codes, scales, bad = oracle.quantize_fp4(x)
    assert bad == 0 and np.all(scales == 0)
    assert np.all(codes[0] == 0) and np.all(codes[1] == 0x88)
    # tiny values: amax/6 <= 2^-10 -> scale 0 -> magnitude 0, sign kept
    x = np.full((1, 32), -1e-4, np.float32)
    codes, scales, _ = oracle.quantize_fp4(x)
    assert scales[0, 0] == 0 and np.all(codes == 0x88)


def test_quantize_nonfinite_reported():
    x = np.zeros((3, 64), np.float32)
    x[0, 3] = np.inf
    x[2, 40] = np.nan
    _, _, bad = oracle.quantize_fp4(x)
    assert bad == 2


def test_quantize_error_bound_and_roundtrip():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((500, 128)) * np.exp(rng.uniform(-6, 6, (500, 1)))).astype(np.float32)
    codes, scales, _ = oracle.quantize_fp4(x)
    xt = oracle.dequant_fp4(codes, scales)
    s = np.repeat(np.array([[oracle.e4m3_value(c) for c in r] for r in scales]), 32, 1)
    ax = np.abs(x.astype(np.float64))
    within = ax <= 6 * s
    spacing = np.where(ax < 2 * s, 0.5, np.where(ax < 4 * s, 1.0, 2.0)) * s
    assert np.all(np.abs(x - xt)[within] <= spacing[within] / 2 * (1 + 1e-12))
    # groups whose largest code is 6 re-quantise to identical bytes
    c2, s2, _ = oracle.quantize_fp4(xt.astype(np.float32))
    mag = _unpack(codes, 128) & 7
    has6 = (mag.reshape(500, 4, 32) == 7).any(-1)
    same_c = (_unpack(c2, 128) == _unpack(codes, 128)).reshape(500, 4, 32).all(-1)
    same_s = s2 == scales
    assert np.all(same_c[has6]) and np.all(same_s[has6])
    assert has6.mean() > 0.5


# ---------------------------------------------------------------- scores

def _rand_fp4(rng, n, d, scale=1.0):
    x = (rng.standard_normal((n, d)) * scale).astype(np.float32)
    c, s, _ = oracle.quantize_fp4(x)
    return c, s


def test_scores_one_hot_closed_form():
    rng = np.random.default_rng(3)
    kc, ks = _rand_fp4(rng, 300, 64)
    kd = oracle.dequant_fp4(kc, ks)
    for c in [0, 17, 63]:
        q = np.zeros((1, 64))
        q[0, c] = 1.0
        s = oracle.index_scores(q, np.array([1.0]), kc, ks)
        assert np.array_equal(s, np.maximum(kd[:, c], 0.0))


def test_scores_all_positive_textbook():
    rng = np.random.default_rng(4)
    x = np.abs(rng.standard_normal((200, 128))).astype(np.float32)
    kc, ks, _ = oracle.quantize_fp4(x)
    kd = oracle.dequant_fp4(kc, ks)
    q = np.abs(rng.standard_normal((8, 128)))
    w = rng.uniform(0, 1, 8)
    s = oracle.index_scores(q, w, kc, ks)
    ref = kd @ (w[:, None] * q).sum(0)
    np.testing.assert_allclose(s, ref, rtol=1e-12)


def test_scores_relu_per_head():
    """mixed-sign dot products: each head's negative part is dropped, then weighted"""
    rng = np.random.default_rng(5)
    kc, ks = _rand_fp4(rng, 100, 64)
    kd = oracle.dequant_fp4(kc, ks)
    q = rng.standard_normal((4, 64))
    w = np.array([0.5, 1.0, 0.25, 2.0])
    s = oracle.index_scores(q, w, kc, ks)
    ref = (np.maximum(kd @ q.T, 0.0) * w[None, :]).sum(1)
    np.testing.assert_allclose(s, ref, rtol=1e-12)
    assert np.all(s >= 0)


# ---------------------------------------------------------------- selection

def test_topk_bruteforce_with_ties():
    rng = np.random.default_rng(6)
    for n in [1, 2, 7, 50, 333]:
        for k in [1, 3, 64, 400]:
            sc = rng.integers(0, 5, n).astype(np.float64)  # many exact ties
            ids = rng.permutation(10 * n)[:n].astype(np.int64)
            got = oracle.topk(sc, ids, k)
            order = sorted(range(n), key=lambda i: (-sc[i], ids[i]))[:k]
            assert np.array_equal(got, np.sort(ids[order]))


def test_block_scores_partial_block():
    rng = np.random.default_rng(7)
    s = rng.standard_normal(37)
    for p in [0, 6, 7, 8, 15, 36]:
        bs = oracle.block_scores(s, p)
        pad = np.full(((p + 8) // 8) * 8, -np.inf)
        pad[: p + 1] = s[: p + 1]
        assert np.array_equal(bs, pad.reshape(-1, 8).max(1))


def _tiny_case(seed, L, d=64, H=4, zero_blocks=()):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((L, d)).astype(np.float32)
    for j in zero_blocks:
        x[8 * j: 8 * j + 8] = 0
    kc, ks, _ = oracle.quantize_fp4(x)
    q = oracle.dequant_fp4(*oracle.quantize_fp4(rng.standard_normal((H, d)).astype(np.float32))[:2])
    w = rng.uniform(0, 1, H)
    return q, w, kc, ks


@pytest.mark.parametrize("L,P,K", [(8, 1, 4), (9, 1, 16), (64, 3, 10), (1000, 20, 64), (1000, 200, 64),
                                   (4096, 64, 256)])
def test_full_select_bruteforce_and_invariants(L, P, K):
    q, w, kc, ks = _tiny_case(L, L, zero_blocks=(0, 3) if L > 32 else ())
    p = L - 1
    r = oracle.full_select(q, w, kc, ks, p, P, K)
    s = oracle.index_scores(q, w, kc[: p + 1], ks[: p + 1])
    # pool by brute force: blocks sorted by (max desc, id asc)
    nb = (p + 8) // 8
    bmax = [max(s[8 * j: min(8 * j + 8, p + 1)]) for j in range(nb)]
    pool = sorted(sorted(range(nb), key=lambda j: (-bmax[j], j))[:P])
    assert list(r.pool) == pool
    cand = [t for j in pool for t in range(8 * j, min(8 * j + 8, p + 1))]
    idx = sorted(sorted(cand, key=lambda t: (-s[t], t))[:K])
    assert list(r.idx) == idx
    assert set(r.idx) <= set(cand)
    if K <= P:  # the pool's top-K is the global top-K
        glob = sorted(sorted(range(p + 1), key=lambda t: (-s[t], t))[:K])
        assert list(r.idx) == glob


@pytest.mark.parametrize("L", [8, 100, 2000])
def test_reindex_with_full_query_equals_full(L):
    """with a pool covering the whole context, Reindex with the Full layer's
    (q, w) selects exactly what the Full layer selects"""
    q, w, kc, ks = _tiny_case(100 + L, L)
    p = L - 1
    K = 32
    full = oracle.full_select(q, w, kc, ks, p, P=(L + 7) // 8, K=K)
    assert len(full.pool) == (L + 7) // 8
    idx, _, _ = oracle.reindex_select(q, w, kc, ks, p, full.pool, K)
    assert np.array_equal(idx, full.idx)


def test_select_ties_lower_ids_and_zero_scores():
    # all-zero keys: every score is 0, ties resolve to the lowest ids
    kc = np.zeros((64, 32), np.uint8)
    ks = np.zeros((64, 2), np.uint8)
    q = np.ones((2, 64))
    r = oracle.full_select(q, np.ones(2), kc, ks, 63, P=3, K=5)
    assert list(r.pool) == [0, 1, 2]
    assert list(r.idx) == [0, 1, 2, 3, 4]


def test_k_larger_than_visible():
    q, w, kc, ks = _tiny_case(9, 20)
    r = oracle.full_select(q, w, kc, ks, 12, P=8, K=64)
    assert list(r.idx) == list(range(13))


# ---------------------------------------------------------------- attention

def _softmax_attend_numpy(q, v, scale, mask=None):
    z = scale * q @ v.T
    if mask is not None:
        z = np.where(mask[None, :], z, -np.inf)
    z = z - z.max(1, keepdims=True)
    e = np.exp(z)
    return (e / e.sum(1, keepdims=True)) @ v


def test_attention_equals_dense_masked():
    rng = np.random.default_rng(8)
    L, D, H = 300, 128, 16
    v = oracle.dequant_fp4(*oracle.quantize_fp4(rng.standard_normal((L, D)).astype(np.float32))[:2])
    q = rng.standard_normal((H, D))
    S = np.sort(rng.choice(L, 77, replace=False))
    mask = np.zeros(L, bool)
    mask[S] = True
    out, _ = oracle.attend(q, v[S], 1 / math.sqrt(D))
    ref = _softmax_attend_numpy(q, v, 1 / math.sqrt(D), mask)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_attention_single_row_and_zero_query():
    rng = np.random.default_rng(9)
    v = rng.standard_normal((10, 64))
    q = rng.standard_normal((4, 64))
    out, lse = oracle.attend(q, v[3:4], 0.125)
    assert np.array_equal(out, np.repeat(v[3:4], 4, 0))
    np.testing.assert_allclose(lse, 0.125 * q @ v[3], rtol=1e-14)
    out, lse = oracle.attend(np.zeros((2, 64)), v, 0.125)
    np.testing.assert_allclose(out, np.repeat(v.mean(0, keepdims=True), 2, 0), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, math.log(10.0), rtol=1e-14)


def test_attention_lse_split_merge_invariance():
    rng = np.random.default_rng(10)
    v = rng.standard_normal((100, 32))
    q = rng.standard_normal((3, 32)) * 3
    full, lse = oracle.attend(q, v, 0.3)
    for cut in [1, 37, 99]:
        o1, l1 = oracle.attend(q, v[:cut], 0.3)
        o2, l2 = oracle.attend(q, v[cut:], 0.3)
        m = np.maximum(l1, l2)
        a1, a2 = np.exp(l1 - m), np.exp(l2 - m)
        merged = (a1[:, None] * o1 + a2[:, None] * o2) / (a1 + a2)[:, None]
        np.testing.assert_allclose(merged, full, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(m + np.log(a1 + a2), lse, rtol=1e-13)


def test_swa_merge_is_one_softmax_over_concatenation():
    rng = np.random.default_rng(11)
    kv = rng.standard_normal((50, 64))
    sw = rng.standard_normal((20, 64))
    q = rng.standard_normal((4, 64))
    out, _ = oracle.attend_rows(q, kv, sw, 0.2)
    ref = _softmax_attend_numpy(q, np.concatenate([kv, sw]), 0.2)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-13)


def test_structural_constants_of_configs():
    from synth.workloads import BLOCK, CONFIGS
    g = _golden("hierarchical_indexer.txt")
    assert BLOCK == g["block_positions"][0]
    assert g["pool_blocks"][0] * g["block_positions"][0] == g["pool_positions"][0]
    for i in (2, 3, 4, 5):
        c = CONFIGS[i]
        assert c.P == g["pool_blocks"][0] and c.K == g["final_topk"][0]
    assert CONFIGS[5].window == g["swa_window"][0]
    for i in (3, 4, 5):
        c = CONFIGS[i]
        assert 1 + c.n_reindex + c.n_reuse == g["decoder_layers"][0]
