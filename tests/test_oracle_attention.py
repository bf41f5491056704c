"""Pins of oracle.attention: textbook special cases, a pure-Python brute force on tiny
shapes and RoPE identities."""
import math

import numpy as np

from oracle import attention


def _brute(q, K, V, scale):
    """Softmax attention with Python loops and math.exp (no max subtraction)."""
    G, D = len(q), len(q[0])
    T = len(K)
    out = []
    for h in range(G):
        w = []
        for t in range(T):
            s = sum(q[h][d] * K[t][d] for d in range(D)) * scale
            w.append(math.exp(s))
        tot = sum(w)
        out.append([sum(w[t] * V[t][d] for t in range(T)) / tot for d in range(D)])
    return np.array(out)


def test_brute_force_tiny():
    r = np.random.default_rng(0)
    for T in (1, 2, 5, 16):
        q = r.standard_normal((3, 8))
        K = r.standard_normal((T, 8))
        V = r.standard_normal((T, 8))
        got = attention.attention(q, K, V, 0.35)
        want = _brute(q.tolist(), K.tolist(), V.tolist(), 0.35)
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-14)


def test_single_token_returns_its_value():
    r = np.random.default_rng(1)
    V = r.standard_normal((1, 16))
    out = attention.attention(r.standard_normal((4, 16)), r.standard_normal((1, 16)), V, 1.0)
    np.testing.assert_allclose(out, np.repeat(V, 4, 0), rtol=0, atol=0)


def test_zero_query_or_equal_keys_give_the_mean():
    r = np.random.default_rng(2)
    V = r.standard_normal((10, 16))
    K = r.standard_normal((10, 16))
    np.testing.assert_allclose(attention.attention(np.zeros((1, 16)), K, V, 1.0)[0], V.mean(0),
                               rtol=1e-13)
    Ke = np.repeat(K[:1], 10, 0)
    np.testing.assert_allclose(attention.attention(r.standard_normal((1, 16)), Ke, V, 1.0)[0],
                               V.mean(0), rtol=1e-13)


def test_shift_invariance():
    # adding the same vector to every key shifts all scores of a query equally
    r = np.random.default_rng(3)
    q = r.standard_normal((2, 16))
    K = r.standard_normal((20, 16))
    V = r.standard_normal((20, 16))
    a = attention.attention(q, K, V, 0.25)
    b = attention.attention(q, K + r.standard_normal(16), V, 0.25)
    np.testing.assert_allclose(a, b, rtol=1e-12)


def test_large_scores_are_stable():
    q = np.full((1, 4), 100.0)
    K = np.array([[10.0] * 4, [9.0] * 4])
    V = np.array([[1.0] * 4, [0.0] * 4])
    out = attention.attention(q, K, V, 1.0)
    assert np.all(np.isfinite(out))
    np.testing.assert_allclose(out[0, 0], 1 / (1 + math.exp(-400)), rtol=1e-15)


def test_rope_identities():
    r = np.random.default_rng(4)
    D = 16
    k = r.standard_normal((6, D))
    pos = np.array([0, 1, 7, 100, 5000, 131071])
    rk = attention.rope_rotate(k, pos, 10000.0)
    np.testing.assert_allclose(rk[0], k[0], rtol=0, atol=0)               # t = 0
    np.testing.assert_allclose(np.linalg.norm(rk, axis=1), np.linalg.norm(k, axis=1), rtol=1e-13)
    # rotate-half pairs (i, i + D/2) by t * base^(-2i/D), checked with complex numbers
    for t_i, t in enumerate(pos):
        z = (k[t_i, :D // 2] + 1j * k[t_i, D // 2:]) * np.exp(
            1j * t * 10000.0 ** (-2.0 * np.arange(D // 2) / D))
        np.testing.assert_allclose(rk[t_i], np.concatenate([z.real, z.imag]), rtol=1e-9, atol=1e-12)
    # q_m . k_n depends only on n - m
    q = r.standard_normal((1, D))
    kk = r.standard_normal((1, D))
    a = attention.rope_rotate(q, [3], 10000.0) @ attention.rope_rotate(kk, [10], 10000.0).T
    b = attention.rope_rotate(q, [103], 10000.0) @ attention.rope_rotate(kk, [110], 10000.0).T
    np.testing.assert_allclose(a, b, rtol=1e-11)


def test_rel_l2():
    assert attention.rel_l2([3.0, 4.0], [3.0, 4.0]) == 0.0
    assert abs(attention.rel_l2([3.0, 4.0], [0.0, 5.0]) - math.sqrt(10) / 5) < 1e-15


def test_merge_of_disjoint_parts_is_attention_over_the_union():
    # the softmax over a union of token sets splits into per-set weights exp(lse_r - lse)
    from oracle.attention import attention_lse, merge_parts
    rng = np.random.default_rng(17)
    q = rng.standard_normal((4, 32)) * 2.0
    K = rng.standard_normal((50, 32))
    V = rng.standard_normal((50, 32))
    whole, lse = attention_lse(q, K, V, 0.3)
    np.testing.assert_allclose(whole, attention.attention(q, K, V, 0.3), rtol=1e-13, atol=1e-14)
    # lse by brute force
    brute = np.array([np.log(sum(np.exp(0.3 * float(q[g] @ K[t])) for t in range(50))) for g in range(4)])
    np.testing.assert_allclose(lse, brute, rtol=1e-13)
    cuts = [0, 7, 30, 31, 50]
    parts = [attention_lse(q, K[a:b], V[a:b], 0.3) for a, b in zip(cuts, cuts[1:])]
    merged, mlse = merge_parts([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(merged, whole, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(mlse, lse, rtol=1e-13)
    # one part is the identity
    one, one_lse = merge_parts([whole], [lse])
    np.testing.assert_allclose(one, whole, rtol=1e-15)


def test_merge_with_empty_parts():
    # a part with no tokens (lse = -inf) has no weight, whatever its out holds; a row whose
    # every part is empty merges to out = 0, lse = -inf
    from oracle.attention import attention_lse, merge_parts
    rng = np.random.default_rng(23)
    q = rng.standard_normal((3, 16))
    K = rng.standard_normal((20, 16))
    V = rng.standard_normal((20, 16))
    whole, lse = attention_lse(q, K, V, 0.25)
    a = attention_lse(q, K[:9], V[:9], 0.25)
    b = attention_lse(q, K[9:], V[9:], 0.25)
    empty_out = np.full_like(whole, np.nan)
    empty_lse = np.full_like(lse, -np.inf)
    merged, mlse = merge_parts([a[0], empty_out, b[0]], [a[1], empty_lse, b[1]])
    np.testing.assert_allclose(merged, whole, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(mlse, lse, rtol=1e-13)
    # rows 0 and 2 lose every token: zeros and -inf there, row 1 unchanged
    la, lb = a[1].copy(), b[1].copy()
    la[[0, 2]] = -np.inf
    lb[[0, 2]] = -np.inf
    merged, mlse = merge_parts([a[0], b[0]], [la, lb])
    assert np.all(merged[[0, 2]] == 0.0) and np.all(np.isneginf(mlse[[0, 2]]))
    np.testing.assert_allclose(merged[1], whole[1], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(mlse[1], lse[1], rtol=1e-13)
