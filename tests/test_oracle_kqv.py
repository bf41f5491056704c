"""Pins of the KQV oracle (oracle.kqv): the Lloyd-Max quantizer of the Beta coordinate
marginal against closed forms and textbook tables, and the QJL sketch against its
closed-form mean and variance by Monte Carlo over seeded sketch matrices."""
import math

import numpy as np
import pytest

from oracle import kqv


@pytest.mark.parametrize("d", [3, 8, 128, 2049])
def test_marginal_is_a_symmetric_density(d):
    L = min(1.0, 14.0 / math.sqrt(d))
    x = np.linspace(-L, L, 400001)
    f = kqv.marginal_pdf(x, d)
    assert abs(np.trapezoid(f, x) - 1.0) < 1e-5   # (d = 3: half a cell lost at each open end)
    np.testing.assert_allclose(f, f[::-1], rtol=1e-9, atol=1e-12 * f.max())


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_d3_marginal_is_uniform_so_lloyd_max_is_the_uniform_quantizer(bits):
    # a coordinate of a random unit vector in R^3 is uniform on [-1, 1] (Archimedes)
    k = 1 << bits
    want = (2 * np.arange(k) + 1) / k - 1.0
    np.testing.assert_allclose(kqv.lloyd_max(bits, 3), want, atol=1e-9)


@pytest.mark.parametrize("d", [3, 16, 128, 2049])
def test_one_bit_centroid_is_the_mean_absolute_coordinate(d):
    # E|x| = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    ex = math.exp(math.lgamma(d / 2.0) - math.lgamma(0.5) - math.lgamma((d + 1) / 2.0))
    c = kqv.lloyd_max(1, d)
    np.testing.assert_allclose(c, [-ex, ex], rtol=1e-8)


def test_large_d_approaches_the_gaussian_lloyd_max_table():
    # Max (1960), N(0, 1): 1 bit 0.7979; 2 bits 0.4528, 1.510; 3 bits 0.2451, 0.7560,
    # 1.344, 2.152 (positive halves); the marginal tends to N(0, 1/d)
    table = {1: [0.7979], 2: [0.4528, 1.510], 3: [0.2451, 0.7560, 1.344, 2.152]}
    d = 20001
    for bits, pos in table.items():
        c = kqv.lloyd_max(bits, d) * math.sqrt(d)
        np.testing.assert_allclose(c[len(c) // 2:], pos, atol=2e-3)
        np.testing.assert_allclose(c[: len(c) // 2], -np.array(pos[::-1]), atol=2e-3)


def test_lloyd_max_is_a_fixed_point():
    # centroids are the conditional means of the cells between midpoints
    c = kqv.lloyd_max(2, 128)
    np.testing.assert_allclose(kqv.lloyd_max(2, 128, iters=301), c, atol=1e-12)


def _sketch_samples(q, r, m, n, seed):
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((n, m, q.size))
    signs = np.where(S @ r >= 0, 1.0, -1.0)
    return math.sqrt(math.pi / 2) / m * np.linalg.norm(r) * np.einsum("nm,nm->n", S @ q, signs), S, signs


@pytest.mark.parametrize("orthogonal", [True, False])
def test_qjl_inner_product_is_unbiased_with_the_stated_variance(orthogonal):
    d = m = 64
    rng = np.random.default_rng(1)
    r = rng.standard_normal(d) * 0.3
    q = rng.standard_normal(d)
    if orthogonal:
        q -= (q @ r) / (r @ r) * r
    est, S, signs = _sketch_samples(q, r, m, 4000, 2)
    # the library-facing function agrees with the vectorized estimate
    assert est[0] == pytest.approx(kqv.qjl_inner(q, signs[0], np.linalg.norm(r), S[0]), rel=1e-12)
    var = (math.pi / 2 * (q @ q) * (r @ r) - (q @ r) ** 2) / m
    if orthogonal:   # the page's pi/2 ||r||^2 / d, for a unit query
        assert var == pytest.approx(math.pi / 2 * (r @ r) * (q @ q) / d, rel=1e-9)
    assert abs(est.mean() - q @ r) < 4 * math.sqrt(var / est.size)
    assert est.var() == pytest.approx(var, rel=0.1)


def test_qjl_vector_and_kqv_values_are_unbiased():
    d = 32
    rng = np.random.default_rng(3)
    v = rng.standard_normal(d)
    n = 3000
    Ss = rng.standard_normal((n, d, d))
    cb = kqv.lloyd_max(1, d)
    recon = np.array([kqv.kqv_value(v, 2, S, cb) for S in Ss])
    err = recon.mean(axis=0) - v
    # per-coordinate standard error of the mean of the sketch estimate
    se = recon.std(axis=0) / math.sqrt(n)
    assert np.all(np.abs(err) < 5 * se + 1e-12)
    # one draw: the scalar part alone is biased towards the codebook, the sketch removes it
    yh_only = kqv.rotation(d) @ kqv.scalar_decode(*kqv.scalar_encode(kqv.rotation(d) @ v, cb), cb)
    assert np.linalg.norm(recon.mean(axis=0) - v) < 0.25 * np.linalg.norm(yh_only - v)


def test_key_codes_reconstruct_within_the_codebook_error():
    d = 128
    rng = np.random.default_rng(4)
    k = rng.standard_normal(d)
    for bits in (2, 3, 4):
        kh = kqv.kqv_key(k, bits)
        rel = np.linalg.norm(kh - k) / np.linalg.norm(k)
        # Lloyd-Max MSE of a Gaussian: 0.1175 (2 bits), 0.03454 (3), 0.009497 (4), per unit variance
        mse = {2: 0.1175, 3: 0.03454, 4: 0.009497}[bits]
        assert rel < 2.0 * math.sqrt(mse)


def test_stored_codebooks_are_the_oracle_s():
    # tests/golden/kqv_codebooks.json is written by tests/golden/make_kqv_codebooks.py
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "kqv_codebooks.json")
    stored = json.load(open(path))
    assert stored["d"] == 128
    for b in ("1", "2", "3"):
        np.testing.assert_allclose(stored["f64"][b], kqv.lloyd_max(int(b), 128), rtol=0, atol=1e-12)
        np.testing.assert_array_equal(np.float32(stored["f64"][b]), np.float32(stored["f32"][b]))
    # symmetric, strictly increasing, inside [-1, 1]
    for b, c in stored["f64"].items():
        c = np.array(c)
        assert c.size == 1 << int(b) and np.all(np.diff(c) > 0) and np.all(np.abs(c) < 1)
        np.testing.assert_allclose(c, -c[::-1], atol=1e-6)


def test_keys_without_the_sketch_give_lower_attention_kl():
    # [TQ] "Key Contributions" 2: at the 4-bit budget KQV (4-bit scalar keys) has a lower
    # KL divergence of the attention weights than QKQV (3-bit keys + 1-bit sketch): the
    # sketch's variance is amplified by the softmax.  The page reports 2.25x on its data.
    d, T, G = 64, 256, 4
    cb4, cb3 = kqv.lloyd_max(4, d), kqv.lloyd_max(3, d)
    for seed in range(3):
        rng = np.random.default_rng(seed)
        q = rng.standard_normal((G, d))
        K = rng.standard_normal((T, d))
        Kk = np.array([kqv.kqv_key(k, 4, cb4) for k in K])
        Kq = np.array([kqv.qkqv_key(k, 4, rng.standard_normal((d, d)), cb3) for k in K])

        def probs(Kx):
            s = (q @ Kx.T) / math.sqrt(d)
            s -= s.max(axis=1, keepdims=True)
            p = np.exp(s)
            return p / p.sum(axis=1, keepdims=True)

        p0, pk, pq = probs(K), probs(Kk), probs(Kq)
        kl_k = float((p0 * np.log(p0 / pk)).sum(axis=1).mean())
        kl_q = float((p0 * np.log(p0 / pq)).sum(axis=1).mean())
        assert kl_q > 2.0 * kl_k


# ---- stored format ---------------------------------------------------------------------

def test_tree_sum_is_the_pairwise_tree():
    # brute-force recursion over halves, and exact on small integers
    rng = np.random.default_rng(3)
    a = rng.standard_normal((5, 128)).astype(np.float32)

    def rec(v):
        if len(v) == 1:
            return np.float32(v[0])
        h = len(v) // 2
        return np.float32(rec(v[:h]) + rec(v[h:]))

    got = kqv.tree_sum_f32(a)
    for i in range(5):
        assert got[i] == rec(a[i])
    ints = rng.integers(-1000, 1000, (4, 64)).astype(np.float32)
    np.testing.assert_array_equal(kqv.tree_sum_f32(ints), ints.sum(axis=1))


def test_stored_codes_are_the_nearest_centroid_of_the_rotated_direction():
    # the fp32 decision against a float64 brute force, wherever the float64 distance gap is
    # wide enough that fp32 rounding cannot swap the two nearest centroids
    from oracle import rotate
    rng = np.random.default_rng(4)
    D = 128
    x = (rng.standard_t(4, (64, D)) * 2.0).astype(np.float32)
    cb = kqv.lloyd_max(3, D)
    codes, nrm = kqv.stored_encode(x, cb)
    y = np.asarray(rotate.wht_f32(x), np.float64)
    np.testing.assert_allclose(nrm, np.linalg.norm(y, axis=1), rtol=2 ** -20)
    u = y / np.linalg.norm(y, axis=1, keepdims=True)
    c32 = np.asarray(cb, np.float32).astype(np.float64)
    dist = np.abs(u[..., None] - c32)
    best = dist.argmin(axis=-1)
    srt = np.sort(dist, axis=-1)
    clear = (srt[..., 1] - srt[..., 0]) > 1e-5
    assert clear.mean() > 0.99
    np.testing.assert_array_equal(codes[clear], best[clear])


def test_stored_value_is_the_float64_scheme_up_to_fp32_rounding():
    # codes, norms and sketch signs of the stored format reconstruct the float64 KQV value
    # (kqv_value) to fp32 accuracy; the sketch signs agree wherever S r is not tiny
    rng = np.random.default_rng(5)
    D = 128
    S = rng.standard_normal((D, D)).astype(np.float32)
    cb = kqv.lloyd_max(3, D)
    x = rng.standard_normal((16, D)).astype(np.float32)
    codes, nrm, signs, rn = kqv.stored_encode(x, cb, S)
    got = kqv.stored_value(codes, nrm, signs, rn, cb, S)
    want = np.stack([kqv.kqv_value(x[i].astype(np.float64), 4, S.astype(np.float64), cb=cb.astype(np.float32))
                     for i in range(16)])
    np.testing.assert_allclose(got, want, rtol=0, atol=2e-5 * np.abs(want).max())
    from oracle import rotate
    y = np.asarray(rotate.wht_f32(x), np.float64)
    yh = nrm.astype(np.float64)[:, None] * np.asarray(cb, np.float32)[codes]
    t = (y - yh) @ S.astype(np.float64).T
    big = np.abs(t) > 1e-4 * np.abs(t).max()
    np.testing.assert_array_equal(signs[big], (t >= 0)[big])


def test_stored_key_round_trip_error_matches_lloyd_max():
    # relative key error of 4-bit KQV keys on Gaussian rows: the Lloyd-Max MSE of the
    # marginal at d = 128 (about 0.0095 of ||x||^2, Max's table) within sampling noise
    rng = np.random.default_rng(6)
    D = 128
    cb = kqv.lloyd_max(4, D)
    x = rng.standard_normal((400, D)).astype(np.float32)
    codes, nrm = kqv.stored_encode(x, cb)
    kh = kqv.stored_key(codes, nrm, cb)
    err = np.sum((kh - x) ** 2) / np.sum(x.astype(np.float64) ** 2)
    assert 0.0075 < err < 0.0115
