"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test checks the oracle against a fact the pages or the mathematics fix: a worked example
(tests/golden), an explicit matrix built independently, a closed form, an invariant, a library
routine (numpy's IEEE binary16), brute force on tiny inputs, or a statistical property.
"""
import math
import os
from decimal import Decimal, getcontext
from itertools import combinations

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sylvester(d):
    """Natural-order Hadamard matrix by the Kronecker recursion H_2n = [[H, H], [H, -H]]."""
    H = np.ones((1, 1), dtype=np.int64)
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def read_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------------------------- rotation
def test_splitmix64_published_outputs():
    want = [int(x, 16) for x in read_golden("splitmix64_seed0.txt")]
    got = [int(x) for x in oracle.splitmix64(0, 3)]
    assert got == want


def test_signs_are_top_bits_and_involutive():
    d = 128
    D = oracle.signs(7, d)
    outs = oracle.splitmix64(7, d)
    want = np.where((outs >> np.uint64(63)) == 1, -1.0, 1.0).astype(np.float32)
    assert np.array_equal(D, want)
    assert np.all(D * D == 1.0)
    # not degenerate: both signs occur
    assert 16 < int((D < 0).sum()) < 112


@pytest.mark.parametrize("d", [32, 64, 128])
def test_fwht_equals_explicit_sylvester_matrix(d):
    rng = np.random.default_rng(d)
    H = sylvester(d)
    assert np.array_equal(H @ H.T, d * np.eye(d, dtype=np.int64))  # H H^T = d I exactly
    for _ in range(20):
        x = rng.standard_normal(d).astype(np.float32)
        y = oracle.fwht(x)
        ref = H.astype(np.float64) @ x.astype(np.float64)
        assert np.max(np.abs(y - ref)) <= 1e-5 * np.linalg.norm(x) * math.sqrt(d)
        # FWHT o FWHT = d * id ; norm grows by sqrt(d)
        assert np.allclose(oracle.fwht(y), d * x, rtol=0, atol=1e-4 * d * np.abs(x).max())
        assert abs(np.dot(y.astype(np.float64), y) - d * np.dot(x.astype(np.float64), x)) <= 1e-5 * d * np.dot(x, x)


def test_rotation_HD_is_scaled_orthogonal():
    d = 128
    H = sylvester(d)
    D = oracle.signs(3, d).astype(np.int64)
    R = H * D[None, :]  # H diag(D)
    assert np.array_equal(R.T @ R, d * np.eye(d, dtype=np.int64))


# ---------------------------------------------------------------------------------- key sketch
def test_bitmap_layout_matches_page_worked_example():
    lines = read_golden("bitmap_h1ibkv.txt")
    plus = [int(t) for t in lines[0].split(":")[1].split()]
    want_bytes = bytes(int(t, 16) for t in lines[1].split(":")[1].split())
    d = 32
    rng = np.random.default_rng(1)
    s = -np.ones(d)
    s[plus] = 1.0
    y = s * (0.5 + rng.random(d))  # rotated key with these signs
    D = oracle.signs(11, d)
    # k = (H D)^-1 y = D H y / d
    k = (D.astype(np.float64) * (sylvester(d) @ y) / d).astype(np.float32)
    enc = oracle.encode(k[None, :], np.zeros((1, d), np.float32), D)
    got = enc["bits"][0].astype("<u4").tobytes()
    assert got == want_bytes
    # decode with the page's rule: bit (idx % 8) of byte (idx / 8); 1 -> +1.0, 0 -> -1.0
    dec = [1.0 if (got[i // 8] >> (i % 8)) & 1 else -1.0 for i in range(d)]
    assert dec == list(s)


def test_key_bits_norm_cinv_against_fp64_matrix():
    d = 128
    rng = np.random.default_rng(5)
    D = oracle.signs(0, d)
    R = sylvester(d) * D.astype(np.float64)[None, :]
    K = rng.standard_normal((200, d)).astype(np.float32)
    K[:, 7] *= 10.0
    enc = oracle.encode(K, np.zeros_like(K), D)
    for t in range(K.shape[0]):
        y = R @ K[t].astype(np.float64)
        bits = np.array([(enc["bits"][t, i // 32] >> (i % 32)) & 1 for i in range(d)])
        sure = np.abs(y) > 1e-4 * np.linalg.norm(y)
        assert np.array_equal(bits[sure], (y[sure] >= 0).astype(bits.dtype))
        n = np.linalg.norm(K[t].astype(np.float64))
        assert abs(enc["norm"][t] - n) <= 1e-6 * n
        cinv = d * n / np.abs(y).sum()
        assert abs(enc["cinv"][t] - cinv) <= 1e-5 * cinv


def test_correction_mean_is_sqrt_2_over_pi_for_gaussian_keys():
    # C = sum|y| / (d ||k||) with y = HDk; for k ~ N(0, I): C -> sqrt(2/pi).
    d = 128
    rng = np.random.default_rng(9)
    K = rng.standard_normal((4000, d)).astype(np.float32)
    enc = oracle.encode(K, np.zeros_like(K), oracle.signs(1, d))
    C = 1.0 / enc["cinv"].astype(np.float64)
    assert abs(C.mean() - math.sqrt(2 / math.pi)) < 0.005


def _flat_key(d, seed):
    """A key whose rotated image has all |y_i| equal (= 1): k = D H s / d for a sign vector s."""
    rng = np.random.default_rng(seed)
    s = rng.choice([-1.0, 1.0], size=d)
    D = oracle.signs(seed, d)
    k = (D.astype(np.float64) * (sylvester(d) @ s) / d).astype(np.float32)
    return k, s, D


def test_flat_key_closed_form_C_is_one_and_estimate_is_exact():
    d = 128
    k, s, D = _flat_key(d, 21)
    enc = oracle.encode(k[None, :], np.zeros((1, d), np.float32), D)
    assert enc["norm"][0] == 1.0 and enc["cinv"][0] == 1.0  # ||k|| = 1, C = 1 exactly
    rng = np.random.default_rng(2)
    for _ in range(10):
        q = rng.standard_normal(d).astype(np.float32)
        qp = oracle.query_prep(q, D)
        # with the exact rotated query, N*cinv*sum(2b-1) z / d equals q.k
        b = np.array([(enc["bits"][0, i // 32] >> (i % 32)) & 1 for i in range(d)], dtype=np.float64)
        est_exact = enc["norm"][0] * enc["cinv"][0] * np.dot(2 * b - 1, qp["z"].astype(np.float64)) / d
        qk = float(np.dot(q.astype(np.float64), k.astype(np.float64)))
        assert abs(est_exact - qk) <= 1e-5 * (1 + abs(qk))
        # with the 4-bit query the integer pipeline is within delta/2 of q.k (here N*cinv = 1)
        A, Bc = oracle.score_ints(enc["bits"], qp["planes"])
        s_logit = oracle.logit(A[0], Bc[0], qp["Sq"], qp["vl"], qp["delta"], enc["norm"][0], enc["cinv"][0], 1.0, d)
        assert abs(s_logit - qk) <= qp["delta"] / 2 * (1 + 1e-5) + 1e-5


def test_estimator_equals_rabitq_form_with_orthonormal_P():
    # RaBitQ: <q,k> ~ ||k|| <xbar, Pq> / <xbar, P k/||k||>, xbar = sign(Pk)/sqrt(d), P orthonormal.
    d = 128
    rng = np.random.default_rng(4)
    for seed in range(5):
        D = oracle.signs(seed, d)
        P = sylvester(d) * D.astype(np.float64)[None, :] / math.sqrt(d)
        k = rng.standard_normal(d).astype(np.float32)
        q = rng.standard_normal(d).astype(np.float32)
        kk, qq = k.astype(np.float64), q.astype(np.float64)
        xbar = np.where(P @ kk >= 0, 1.0, -1.0) / math.sqrt(d)
        rabitq = np.linalg.norm(kk) * np.dot(xbar, P @ qq) / np.dot(xbar, P @ kk / np.linalg.norm(kk))
        enc = oracle.encode(k[None, :], np.zeros((1, d), np.float32), D)
        z = oracle.query_prep(q, D)["z"].astype(np.float64)
        b = np.array([(enc["bits"][0, i // 32] >> (i % 32)) & 1 for i in range(d)], dtype=np.float64)
        ours = float(enc["norm"][0]) * float(enc["cinv"][0]) * np.dot(2 * b - 1, z) / d
        assert abs(ours - rabitq) <= 1e-4 * (1 + abs(rabitq))


def test_rabitq_form_is_unbiased_under_haar_rotation():
    # The estimator form the oracle implements is unbiased over Haar-random rotations.
    d = 128
    rng = np.random.default_rng(12)
    k = rng.standard_normal(d)
    q = rng.standard_normal(d)
    ests = []
    for _ in range(3000):
        Q, Rm = np.linalg.qr(rng.standard_normal((d, d)))
        P = Q * np.sign(np.diag(Rm))[None, :]
        pk = P @ k
        xbar = np.where(pk >= 0, 1.0, -1.0) / math.sqrt(d)
        ests.append(np.linalg.norm(k) * np.dot(xbar, P @ q) / np.dot(xbar, pk / np.linalg.norm(k)))
    ests = np.array(ests)
    assert abs(ests.mean() - np.dot(q, k)) <= 4 * ests.std() / math.sqrt(len(ests))


def test_oracle_estimator_nearly_unbiased_over_rotation_seeds():
    # The oracle's own pipeline (H D rotation, 1-bit key, 4-bit query, integer scoring),
    # averaged over rotation seeds, for fixed Gaussian q and k.
    d = 128
    rng = np.random.default_rng(13)
    k = rng.standard_normal(d).astype(np.float32)
    q = rng.standard_normal(d).astype(np.float32)
    qk = float(np.dot(q.astype(np.float64), k.astype(np.float64)))
    ests = []
    for seed in range(1500):
        D = oracle.signs(seed, d)
        enc = oracle.encode(k[None, :], np.zeros((1, d), np.float32), D)
        qp = oracle.query_prep(q, D)
        A, Bc = oracle.score_ints(enc["bits"], qp["planes"])
        ests.append(oracle.logit(A[0], Bc[0], qp["Sq"], qp["vl"], qp["delta"], enc["norm"][0], enc["cinv"][0], 1.0, d))
    ests = np.array(ests)
    sem = ests.std() / math.sqrt(len(ests))
    bias = ests.mean() - qk
    # statistical error plus a small allowance for the deterministic 4-bit query rounding
    assert abs(bias) <= 4 * sem + 0.02 * abs(qk) + 0.05, (bias, sem, qk)


# ---------------------------------------------------------------------------------- values
def test_half_decoder_matches_ieee_binary16_for_all_finite_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = bits.view(np.float16).astype(np.float64)
    for b in range(0, 65536, 1):
        if not np.isfinite(want[b]):
            continue
        if b % 97 and b not in (0, 1, 0x3ff, 0x400, 0x7bff, 0x8001, 0xfbff):
            continue  # a spread sample; the decoder is a closed form
        assert oracle.half_to_double(b) == want[b]


def _groups(enc_sm, t, g):
    w = int(enc_sm[t, g])
    scale = np.uint16(w & 0xFFFF).view(np.float16).astype(np.float64)
    mn = np.uint16(w >> 16).view(np.float16).astype(np.float64)
    return scale, mn


def test_value_quant_bounds_rounding_and_minimal_scale():
    d = 128
    rng = np.random.default_rng(6)
    V = rng.standard_normal((300, d)).astype(np.float32) * rng.uniform(0.01, 30, size=(300, 1)).astype(np.float32)
    enc = oracle.encode(np.ones_like(V), V, oracle.signs(0, d))
    assert enc["flags"] == 0
    vhat = oracle.dequant(enc["codes"], enc["sm"])
    for t in range(V.shape[0]):
        for g in range(d // 32):
            scale, mn = _groups(enc["sm"], t, g)
            x = V[t, 32 * g:32 * g + 32].astype(np.float64)
            # min is the largest binary16 <= min(x)   (numpy's IEEE binary16 as the library check)
            assert mn <= x.min()
            up = np.nextafter(np.float16(mn), np.float16(np.inf)).astype(np.float64)
            assert up > x.min()
            # scale is the smallest binary16 with 15*scale >= max(x) - min
            assert 15 * scale >= x.max() - mn
            if scale > 0:
                dn = np.nextafter(np.float16(scale), np.float16(0)).astype(np.float64)
                assert 15 * dn < x.max() - mn
            err = np.abs(vhat[t, 32 * g:32 * g + 32] - x)
            assert np.all(err <= scale / 2 * (1 + 1e-6) + 1e-12)
    codes = np.array([[(enc["codes"][t, c // 8] >> (4 * (c % 8))) & 15 for c in range(d)] for t in range(3)])
    assert codes.min() == 0 and codes.max() == 15


def test_value_quant_brute_force_codes_small():
    # every code equals the nearest grid point index (ties up), found by brute force over 0..15
    d = 32
    rng = np.random.default_rng(8)
    V = rng.standard_normal((50, d)).astype(np.float32)
    enc = oracle.encode(np.ones_like(V), V, oracle.signs(0, d))
    for t in range(50):
        scale, mn = _groups(enc["sm"], t, 0)
        for c in range(d):
            code = (enc["codes"][t, c // 8] >> (4 * (c % 8))) & 15
            grid = mn + scale * np.arange(16)
            dist = np.abs(grid - V[t, c])
            best = np.flatnonzero(dist <= dist.min() + 1e-6 * scale)
            assert code in best


def test_value_quant_special_cases():
    d = 32
    V = np.full((1, d), 0.5, np.float32)  # constant, representable
    enc = oracle.encode(np.ones_like(V), V, oracle.signs(0, d))
    assert np.all(oracle.dequant(enc["codes"], enc["sm"]) == 0.5)
    # min + 15*scale spans at most 65504 * 16; beyond that (or below -65504) saturation is flagged
    for big in (1e7, -1e6):
        V = np.full((1, d), big, np.float32)
        assert oracle.encode(np.ones_like(V), V, oracle.signs(0, d))["flags"] & 2
    V = np.full((1, d), 1e6, np.float32)  # representable: 65504 + 15 * scale covers it
    enc = oracle.encode(np.ones_like(V), V, oracle.signs(0, d))
    assert enc["flags"] == 0
    assert np.all(np.abs(oracle.dequant(enc["codes"], enc["sm"]) - 1e6) <= 65504 / 2)
    V = np.zeros((1, d), np.float32)
    V[0, 3] = np.inf
    assert oracle.encode(np.ones_like(V), V, oracle.signs(0, d))["flags"] & 1


# ---------------------------------------------------------------------------------- query
def test_query_quantization_bounds_and_planes():
    d = 128
    rng = np.random.default_rng(10)
    D = oracle.signs(0, d)
    for _ in range(50):
        q = rng.standard_normal(d).astype(np.float32) * rng.uniform(0.1, 10)
        qp = oracle.query_prep(q, D)
        z = qp["z"].astype(np.float64)
        assert np.allclose(z, sylvester(d) @ (D.astype(np.float64) * q), atol=1e-4 * np.abs(z).max())
        c = qp["codes"].astype(np.int64)
        assert c.min() == 0 and c.max() == 15
        assert c[np.argmin(z)] == 0 and c[np.argmax(z)] == 15
        zt = float(qp["vl"]) + float(qp["delta"]) * c
        assert np.all(np.abs(zt - z) <= float(qp["delta"]) / 2 * (1 + 1e-5) + 1e-6)
        rec = np.zeros(d, np.int64)
        for j in range(4):
            for i in range(d):
                rec[i] |= ((int(qp["planes"][j, i // 32]) >> (i % 32)) & 1) << j
        assert np.array_equal(rec, c)
        assert qp["Sq"] == c.sum()


def test_query_flat_gives_zero_codes():
    d = 128
    D = oracle.signs(0, d)
    q = np.zeros(d, np.float32)
    qp = oracle.query_prep(q, D)
    assert qp["delta"] == 0 and np.all(qp["codes"] == 0) and qp["Sq"] == 0


def test_popcount_integers_equal_direct_sums():
    d = 128
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 2**32, size=(100, 4), dtype=np.uint64).astype(np.uint32)
    codes = rng.integers(0, 16, size=d)
    planes = np.zeros((4, 4), np.uint32)
    for j in range(4):
        for i in range(d):
            if (codes[i] >> j) & 1:
                planes[j, i // 32] |= np.uint32(1 << (i % 32))
    A, Bc = oracle.score_ints(bits, planes)
    for t in range(100):
        b = np.array([(int(bits[t, i // 32]) >> (i % 32)) & 1 for i in range(d)])
        assert A[t] == int(np.dot(b, codes))
        assert Bc[t] == int(b.sum())


# ---------------------------------------------------------------------------------- attention
def _enc_random(L, d, seed, scale_v=1.0):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = (rng.standard_normal((L, d)) * scale_v).astype(np.float32)
    D = oracle.signs(seed, d)
    return oracle.encode(K, V, D), D, K, V


def test_attend_special_cases():
    d = 128
    enc, D, K, V = _enc_random(1, d, 1)
    q = np.random.default_rng(0).standard_normal(d).astype(np.float32)
    vhat = oracle.dequant(enc["codes"], enc["sm"])
    assert np.allclose(oracle.attend(enc, q, D, 0.1), vhat[0], rtol=0, atol=1e-12)  # L = 1
    # identical keys -> equal logits -> mean of the dequantised values
    enc2, D2, K2, V2 = _enc_random(40, d, 2)
    Ksame = np.repeat(K2[:1], 40, axis=0)
    enc3 = oracle.encode(Ksame, V2, D2)
    vh3 = oracle.dequant(enc3["codes"], enc3["sm"])
    assert np.allclose(oracle.attend(enc3, q, D2, 0.1), vh3.mean(axis=0), rtol=0, atol=1e-12)
    # one key far along q dominates -> its value
    Kd = K2.copy()
    Kd[17] = 200.0 * q / np.linalg.norm(q)
    enc4 = oracle.encode(Kd, V2, D2)
    vh4 = oracle.dequant(enc4["codes"], enc4["sm"])
    assert np.allclose(oracle.attend(enc4, q, D2, 1.0), vh4[17], rtol=0, atol=1e-9)
    # empty cache -> zeros
    empty = {k: v[:0] for k, v in enc.items() if k != "flags"}
    assert np.all(oracle.attend(empty, q, D, 0.1) == 0)


def test_attend_matches_direct_softmax_of_its_logits():
    d = 128
    enc, D, K, V = _enc_random(300, d, 4)
    q = np.random.default_rng(1).standard_normal(d).astype(np.float32)
    qp = oracle.query_prep(q, D)
    s = oracle.logits(enc, qp, 1 / math.sqrt(d)).astype(np.float64)
    w = np.exp(s - s.max())
    ref = (w[:, None] * oracle.dequant(enc["codes"], enc["sm"])).sum(0) / w.sum()
    assert np.allclose(oracle.attend(enc, q, D, 1 / math.sqrt(d)), ref, rtol=1e-12, atol=1e-12)


def test_estimator_error_scales_as_inverse_sqrt_d():
    # RaBitQ's error bound is O(1/sqrt(d)) in ||q|| ||k|| (the pages print no constant, so only
    # the scaling is pinned): the normalised error at d = 32 is about twice that at d = 128.
    rng = np.random.default_rng(17)
    norm_err = {}
    for d in (32, 128):
        errs = []
        for seed in range(40):
            K = rng.standard_normal((64, d)).astype(np.float32)
            q = rng.standard_normal(d).astype(np.float32)
            D = oracle.signs(1000 + seed, d)
            qp = oracle.query_prep(q, D)
            s = oracle.logits(oracle.encode(K, np.zeros_like(K), D), qp, 1.0).astype(np.float64)
            ex = K.astype(np.float64) @ q.astype(np.float64)
            errs.append((s - ex) / (np.linalg.norm(q) * np.linalg.norm(K, axis=1)))
        norm_err[d] = np.std(np.concatenate(errs))
    ratio = norm_err[32] / norm_err[128]
    assert 1.6 < ratio < 2.5, ratio
    assert norm_err[128] < 1.0 / math.sqrt(128)


# ---------------------------------------------------------------------------------- Top-p
def test_exp2_coefficients_are_correctly_rounded():
    getcontext().prec = 60
    ln2 = Decimal(2).ln()
    for k in range(8):
        exact = ln2 ** k / math.factorial(k)
        # correctly rounded fp32: the nearest of the fp32 neighbours of the fp64 approximation
        f = np.float32(float(exact))
        cands = [np.nextafter(f, np.float32(-1)), f, np.nextafter(f, np.float32(2))]
        best = min(cands, key=lambda c: abs(Decimal(float(c)) - exact))
        assert np.float32(oracle.exp2_coef(k)) == best


def test_topp_weight_tracks_exp():
    rng = np.random.default_rng(0)
    for _ in range(3000):
        m = float(np.float32(rng.uniform(-5, 5)))
        s = float(np.float32(m - rng.exponential(6)))
        u = oracle.topp_weight(s, m)
        t = float(np.float32(np.float32(np.float32(s) - np.float32(m)) * np.float32(1.4426950408889634)))
        if t < -40:
            assert u == 0
            continue
        ref = 2.0 ** 32 * 2.0 ** t
        assert abs(u - ref) <= 1e-6 * ref + 1.0
    assert oracle.topp_weight(1.5, 1.5) == 2 ** 32


def _mass(s, idx):
    return sum(oracle.topp_weight(s[i], s.max()) for i in idx)


def test_topp_brute_force_minimal_sets_small():
    rng = np.random.default_rng(1)
    for trial in range(120):
        L = int(rng.integers(1, 11))
        s = (rng.standard_normal(L) * rng.uniform(0.1, 4)).astype(np.float32)
        if trial % 5 == 0 and L > 2:
            s[1] = s[0]  # ties
        p = float(np.float32(rng.uniform(0.05, 1.0)))
        sel = oracle.topp_select(s, p)
        u = [oracle.topp_weight(x, s.max()) for x in s]
        U = sum(u)
        T = min(U, max(1, math.ceil(np.float64(p) * np.float64(U))))
        n = len(sel)
        assert sum(u[i] for i in sel) >= T
        # minimal cardinality: no subset of size n - 1 reaches T
        if n > 1:
            assert all(sum(u[i] for i in c) < T for c in combinations(range(L), n - 1))
        # the set is the prefix of the order (s desc, index asc)
        order = sorted(range(L), key=lambda i: (-float(s[i]), i))
        assert sorted(order[:n]) == list(sel)
        assert list(sel) == sorted(sel)


def test_topp_invariants_and_special_cases():
    rng = np.random.default_rng(2)
    s = rng.standard_normal(500).astype(np.float32) * 3
    for p in (0.1, 0.5, 0.9, 0.99):
        sel = oracle.topp_select(s, p)
        u = {i: oracle.topp_weight(s[i], s.max()) for i in range(len(s))}
        U = sum(u.values())
        T = math.ceil(np.float64(np.float32(p)) * np.float64(U))
        order = sorted(range(len(s)), key=lambda i: (-float(s[i]), i))
        last = order[len(sel) - 1]
        assert sum(u[i] for i in sel) >= T > sum(u[i] for i in sel) - u[last]
        # real-valued softmax mass of the set reaches p
        w = np.exp(s.astype(np.float64) - s.max())
        assert w[sel].sum() / w.sum() >= p - 1e-6
    # p = 1 takes every token with non-zero weight
    s2 = np.array([0.0, -1.0, -100.0, -2.0], np.float32)
    assert list(oracle.topp_select(s2, 1.0)) == [0, 1, 3]
    # one dominant token
    s3 = np.zeros(100, np.float32)
    s3[42] = 50.0
    assert list(oracle.topp_select(s3, 0.9)) == [42]
    with pytest.raises(ValueError):
        oracle.topp_select(s3, 0.0)
    with pytest.raises(ValueError):
        oracle.topp_select(s3, 1.5)


def test_attend_topp_matches_softmax_over_selected():
    d = 128
    enc, D, K, V = _enc_random(200, d, 9)
    q = np.random.default_rng(5).standard_normal(d).astype(np.float32)
    sc = 1 / math.sqrt(d)
    sel, out = oracle.attend_topp(enc, q, D, sc, 0.7)
    s = oracle.logits(enc, oracle.query_prep(q, D), sc).astype(np.float64)
    assert np.array_equal(sel, oracle.topp_select(s.astype(np.float32), 0.7))
    w = np.exp(s[sel] - s[sel].max())
    ref = (w[:, None] * oracle.dequant(enc["codes"][sel], enc["sm"][sel])).sum(0) / w.sum()
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
    # p = 1 with every weight non-zero equals full attention
    sel1, out1 = oracle.attend_topp(enc, q, D, sc, 1.0)
    if len(sel1) == 200:
        assert np.allclose(out1, oracle.attend(enc, q, D, sc), rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ exact attention over a selected set
# RaBitQCache (abstract / core idea): the proxy scores pick the tokens, attention over them uses the
# exact keys and values.  Pinned by closed forms, invariants and a worked two-token example.
def _exact_inputs(L=40, d=128, seed=3):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(d).astype(np.float32), rng.standard_normal((L, d)).astype(np.float32),
            rng.standard_normal((L, d)).astype(np.float32))


def test_exact_selected_single_token_and_empty():
    q, K, V = _exact_inputs()
    for t in (0, 17, 39):
        assert np.array_equal(oracle.attend_exact_selected(q, K, V, [t], 0.3), V[t].astype(np.float64))
    assert np.count_nonzero(oracle.attend_exact_selected(q, K, V, [], 0.3)) == 0
    with pytest.raises(ValueError):
        oracle.attend_exact_selected(q, K, V, [40], 0.3)
    with pytest.raises(ValueError):
        oracle.attend_exact_selected(q, K, V, [-1], 0.3)


def test_exact_selected_equal_logits_give_the_mean():
    q, K, V = _exact_inputs()
    sel = [2, 5, 11, 30]
    out = oracle.attend_exact_selected(np.zeros_like(q), K, V, sel, 0.3)  # q = 0: every logit is 0
    ref = V[sel].astype(np.float64).sum(0) / len(sel)
    assert np.allclose(out, ref, rtol=1e-13, atol=1e-15)


def test_exact_selected_two_token_worked_example():
    # q = e_0, k_a = 0, k_b = c e_0 with scale * c = ln 3 (up to the fp32 rounding of c): weights 1/4, 3/4
    d, scale = 128, 0.5
    q = np.zeros(d, np.float32)
    q[0] = 1.0
    K = np.zeros((2, d), np.float32)
    K[1, 0] = np.float32(2.0 * math.log(3.0))
    V = np.zeros((2, d), np.float32)
    V[0, :] = 4.0
    V[1, :] = -8.0
    out = oracle.attend_exact_selected(q, K, V, [0, 1], scale)
    assert np.allclose(out, 0.25 * 4.0 + 0.75 * -8.0, rtol=1e-6)  # = -5


def test_exact_selected_invariants():
    q, K, V = _exact_inputs(seed=8)
    sel = [1, 4, 9, 16, 25, 36]
    out = oracle.attend_exact_selected(q, K, V, sel, 0.2)
    # the order of the selected list does not matter
    assert np.allclose(oracle.attend_exact_selected(q, K, V, sel[::-1], 0.2), out, rtol=1e-13, atol=1e-15)
    # a convex combination of the selected values
    assert np.all(out <= V[sel].max(0) + 1e-12) and np.all(out >= V[sel].min(0) - 1e-12)
    # adding a constant vector to every value adds it to the output; scaling the values scales it
    c = np.linspace(-3, 3, 128).astype(np.float32)
    assert np.allclose(oracle.attend_exact_selected(q, K, V + c, sel, 0.2), out + c, rtol=1e-6, atol=1e-6)
    assert np.allclose(oracle.attend_exact_selected(q, K, 2 * V, sel, 0.2), 2 * out, rtol=1e-13, atol=1e-15)
    # tokens outside the set do not matter
    V2 = V.copy()
    V2[0] = 1e6
    K2 = K.copy()
    K2[0] = 1e3
    assert np.array_equal(oracle.attend_exact_selected(q, K2, V2, sel, 0.2), out)
    # a dominant logit takes the whole mass
    K3 = K.copy()
    K3[9] = 50.0 * q / np.linalg.norm(q)
    out3 = oracle.attend_exact_selected(q, K3, V, sel, 1.0)
    assert np.allclose(out3, V[9], rtol=1e-9, atol=1e-9)


# ------------------------------------------------------------------ Top-k budget and the kept window
# RaBitQCache abstract (adaptive Top-p vs a fixed Top-k budget) and the H1IB-KV article's high-precision
# layer, read as an always-kept first `sink` / last `recent` window.
def _key_order(s):
    """(s desc, index asc) order by numpy's lexsort (a library sort, independent of the oracle)."""
    return np.lexsort((np.arange(len(s)), -s.astype(np.float64)))


def test_select_topk_is_the_first_k_in_key_order():
    rng = np.random.default_rng(12)
    for L in (1, 7, 40, 300):
        s = np.round(rng.standard_normal(L) * 3, 1).astype(np.float32)  # many equal logits
        order = _key_order(s)
        for k in (0, 1, 5, L, L + 3):
            sel = oracle.select(s, oracle.SELECT_TOPK, k=k)
            assert np.array_equal(sel, np.sort(order[:min(k, L)]))


def test_select_window_is_always_kept_and_budget_applies_to_the_rest():
    rng = np.random.default_rng(13)
    L = 200
    s = rng.standard_normal(L).astype(np.float32)
    s[3] = 50.0  # a dominant token inside the sink
    for sink, recent in ((0, 0), (4, 0), (0, 16), (4, 16), (150, 60)):
        win = [t for t in range(L) if t < sink or t >= L - recent]
        rest = np.array([t for t in range(L) if t not in win], np.int64)
        order = rest[_key_order(s[rest])] if rest.size else rest
        for k in (0, 3, 10):
            sel = oracle.select(s, oracle.SELECT_TOPK, k=k, sink=sink, recent=recent)
            assert np.array_equal(sel, np.sort(np.concatenate([win, order[:k]]).astype(np.int64)))
        for p in (0.3, 0.9, 1.0):
            sel = oracle.select(s, oracle.SELECT_TOPP, p=p, sink=sink, recent=recent)
            assert set(win) <= set(sel.tolist())
            m = s.max()
            u = np.array([oracle.topp_weight(x, m) for x in s], dtype=object)
            T = min(max(int(math.ceil(float(np.float32(p)) * float(sum(u)))), 1), int(sum(u)))
            extra = [t for t in sel.tolist() if t not in win]
            mass = sum(u[t] for t in sel.tolist())
            if extra:
                # the extra tokens are a prefix of the key order, and the shortest one reaching T
                assert extra == sorted(order[:len(extra)].tolist())
                last = order[len(extra) - 1]
                assert mass >= T and mass - u[last] < T
            else:
                assert sum(u[t] for t in win) >= T or len(rest) == 0
    # with no window, Top-p equals the plain Top-p selection
    assert np.array_equal(oracle.select(s, oracle.SELECT_TOPP, p=0.7), oracle.topp_select(s, 0.7))
    # a window covering everything keeps everything
    assert np.array_equal(oracle.select(s, oracle.SELECT_TOPK, k=0, sink=120, recent=120), np.arange(L))
    with pytest.raises(ValueError):
        oracle.select(s, 2)
    with pytest.raises(ValueError):
        oracle.select(s, oracle.SELECT_TOPK, k=-1)
    with pytest.raises(ValueError):
        oracle.select(s, oracle.SELECT_TOPP, p=0.0)


# ------------------------------------------------------------------ stronger rotation (several H D rounds)
def test_rotation_rounds_signs_continue_one_stream():
    d = 128
    s3 = oracle.signs(7, d, rounds=3)
    assert s3.shape == (3 * d,) and set(np.unique(s3)) <= {-1.0, 1.0}
    assert np.array_equal(s3[:d], oracle.signs(7, d))  # round 0 is the single-round rotation
    draws = oracle.splitmix64(7, 3 * d)  # round r = the next d draws of the same stream
    assert np.array_equal(s3, np.where(draws >> np.uint64(63), -1.0, 1.0).astype(np.float32))
    assert np.array_equal(oracle.signs(7, d, rounds=2), s3[:2 * d])


def test_three_round_key_sketch_against_fp64_matrix():
    d = 128
    rng = np.random.default_rng(21)
    S = oracle.signs(3, d, rounds=3).reshape(3, d).astype(np.float64)
    H = sylvester(d).astype(np.float64)
    R = np.eye(d)
    for r in range(3):
        R = H @ np.diag(S[r]) @ R  # y = H D_3 H D_2 H D_1 k
    assert np.allclose(R.T @ R, d ** 3 * np.eye(d))  # orthogonal up to the scale d^3
    K = rng.standard_normal((150, d)).astype(np.float32)
    enc = oracle.encode(K, np.zeros_like(K), S.reshape(-1).astype(np.float32))
    for t in range(K.shape[0]):
        y = R @ K[t].astype(np.float64)
        bits = np.array([(enc["bits"][t, i // 32] >> (i % 32)) & 1 for i in range(d)])
        sure = np.abs(y) > 1e-4 * np.linalg.norm(y)
        assert np.array_equal(bits[sure], (y[sure] >= 0).astype(bits.dtype))
        n = np.linalg.norm(K[t].astype(np.float64))
        cinv = d * n / np.abs(y).sum()  # the same definition for any number of rounds
        assert abs(enc["cinv"][t] - cinv) <= 1e-5 * cinv


def test_three_round_estimator_nearly_unbiased_and_scale_free():
    d = 128
    rng = np.random.default_rng(13)
    k = rng.standard_normal(d).astype(np.float32)
    q = rng.standard_normal(d).astype(np.float32)
    qk = float(np.dot(q.astype(np.float64), k.astype(np.float64)))
    ests = []
    for seed in range(1000):
        D = oracle.signs(seed, d, rounds=3)
        enc = oracle.encode(k[None, :], np.zeros((1, d), np.float32), D)
        qp = oracle.query_prep(q, D)
        A, Bc = oracle.score_ints(enc["bits"], qp["planes"])
        ests.append(oracle.logit(A[0], Bc[0], qp["Sq"], qp["vl"], qp["delta"], enc["norm"][0], enc["cinv"][0], 1.0, d))
    ests = np.array(ests)
    sem = ests.std() / math.sqrt(len(ests))
    assert abs(ests.mean() - qk) <= 4 * sem + 0.02 * abs(qk) + 0.05, (ests.mean(), qk, sem)
    # a key whose three-round transform has all |y_i| equal: ||y|| = d^1.5 ||k||, so
    # C = sum|y| / (d ||k||) = d (the single-round value 1 times the extra scale d of two more rounds)
    S = oracle.signs(5, d, rounds=3)
    H = sylvester(d).astype(np.float64)
    R = np.eye(d)
    for r in range(3):
        R = H @ np.diag(S[r * d:(r + 1) * d].astype(np.float64)) @ R
    kk = (R.T @ np.ones(d) / d ** 3).astype(np.float32)  # R kk = (1, ..., 1) up to fp32 rounding
    enc = oracle.encode(kk[None, :], np.zeros((1, d), np.float32), S)
    assert abs(1.0 / enc["cinv"][0] - d) <= 1e-4 * d


def test_attend_partial_sums_normalise_to_attend_and_merge_by_log_sum_exp():
    # the unnormalised sums of a token range: o / l is the range's attention; two ranges merged by
    # log-sum-exp give the attention over both (a context split over devices); an empty range is the
    # identity of the merge
    rng = np.random.default_rng(4)
    K = rng.standard_normal((900, 128)).astype(np.float32)
    V = rng.standard_normal((900, 128)).astype(np.float32)
    q = rng.standard_normal(128).astype(np.float32)
    D = oracle.signs(2)
    whole = oracle.encode(K, V, D)
    ref = oracle.attend(whole, q, D, 0.4)
    m, l, o = oracle.attend_partial(whole, q, D, 0.4)
    assert np.abs(o / l - ref).max() <= 1e-12 * np.abs(ref).max()
    parts = [oracle.attend_partial(oracle.encode(K[a:b], V[a:b], D), q, D, 0.4) for a, b in ((0, 333), (333, 900))]
    M = max(p[0] for p in parts)
    num = sum(2.0 ** (p[0] - M) * p[2] for p in parts)
    den = sum(2.0 ** (p[0] - M) * p[1] for p in parts)
    assert np.abs(num / den - ref).max() <= 1e-12 * np.abs(ref).max()
    assert abs(M - m) == 0.0  # the larger range maximum is the whole maximum
    me, le, oe = oracle.attend_partial(oracle.encode(K[:0], V[:0], D), q, D, 0.4)
    assert me == -math.inf and le == 0.0 and not oe.any()
