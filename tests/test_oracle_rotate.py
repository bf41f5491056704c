"""Pins of the oracle's key rotation (oracle.rotate) and of rotated-key caches, on CPU.

The transform is pinned to scipy's Sylvester Hadamard matrix (a library routine),
within an error bound derived from the butterfly: at stride h every intermediate is a
signed sum of a disjoint block of inputs, so its fp32 rounding is at most u times the
sum of |x| over that block, and the intermediates that feed one output partition all
D inputs; log2(D) stages, the product with c and the rounding of c itself add at most
(log2(D) + 2) u sum|x| / sqrt(D), u = 2^-24."""
import math

import numpy as np
import pytest
import scipy.linalg

import synth
from oracle import cache as ocache
from oracle import formats, rotate
from oracle.attention import attention, rel_l2

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")
U = 2.0 ** -24


def _rows(D, n, seed, heavy=False):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(3, size=(n, D)) if heavy else rng.standard_normal((n, D))
    return x.astype(np.float32).astype(np.float64)


@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_butterfly_matches_hadamard_product_within_bound(D):
    x = np.concatenate([_rows(D, 40, D), _rows(D, 40, D + 1, heavy=True) * 37.0])
    exact = x @ scipy.linalg.hadamard(D).astype(np.float64).T / math.sqrt(D)
    got = rotate.wht_f32(x)
    bound = (math.log2(D) + 2) * U * np.abs(x).sum(axis=1, keepdims=True) / math.sqrt(D) * 1.001
    assert np.all(np.abs(got - exact) <= bound)
    # the bound is tight enough to see a wrong sign or a missing stage
    assert np.abs(got - exact).max() > 0 or D in (64, 256)
    assert bound.max() < 1e-5 * np.abs(x).sum(axis=1).max()


@pytest.mark.parametrize("D", [32, 128, 256])
def test_one_hot_gives_the_sylvester_column(D):
    H = scipy.linalg.hadamard(D).astype(np.float64)
    c = float(rotate.rot_scale(D))
    for j in (0, 1, D // 2 - 1, D // 2, D - 1):
        e = np.zeros(D)
        e[j] = 1.0
        assert np.array_equal(rotate.wht_f32(e), H[:, j] * c)


@pytest.mark.parametrize("D", [64, 256])
def test_involution_is_exact_when_the_scale_is_a_power_of_two(D):
    rng = np.random.default_rng(3)
    x = rng.integers(-8, 9, size=(16, D)).astype(np.float64)
    assert float(rotate.rot_scale(D)) == 1.0 / math.sqrt(D)
    assert np.array_equal(rotate.wht_f32(rotate.wht_f32(x)), x)


def test_involution_and_norm_within_rounding_at_d128():
    x = _rows(128, 64, 5, heavy=True)
    y = rotate.wht_f32(x)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-6)
    back = rotate.wht_f32(y)
    bound = 2 * (7 + 2) * U * np.abs(x).sum(axis=1, keepdims=True) * 1.01
    assert np.all(np.abs(back - x) <= bound)


def test_rot_scale_is_the_rounded_reciprocal_root():
    assert rotate.rot_scale(128) == np.float32(0.08838834764831845)
    assert rotate.rot_scale(32) == np.float32(1.0 / math.sqrt(32.0))


def _outlier_keys(B, H, n, D, seed, factor=10.0, channels=(3, 77, 101)):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((B, H, n, D))
    k[..., list(channels)] *= factor
    return k.astype(np.float32).astype(np.float64)


def _cache(fmt, B, H, C):
    return ocache.Cache(fmt, B, H, C)


@pytest.mark.parametrize("scheme,axis,bits", [(formats.ASYM, formats.CHANNEL, 4),
                                               (formats.ASYM, formats.CHANNEL, 2),
                                               (formats.SYM8, formats.TOKEN, 8),
                                               (formats.SYM8, formats.CHANNEL, 8)])
def test_rotated_cache_reconstructs_within_the_rotated_error_bound(scheme, axis, bits):
    B, H, n, D, g = 1, 2, 96, 128, 32
    fmt = formats.Format(**synth._fmt(src_dtype=formats.F32, group_tokens=g, k_scheme=scheme,
                                      k_bits=bits, k_axis=axis, k_rotate=1))
    k = _outlier_keys(B, H, n, D, 11)
    c = _cache(fmt, B, H, 128)
    ocache.quantize(fmt, c, formats.KEYS, k, 0, n)
    back = ocache.dequantize(fmt, c, formats.KEYS, 0, n)
    # |y - y^| <= s / 2 (+ the quotient's rounding) in the rotated basis, elementwise;
    # the inverse transform is orthogonal, so the row norms of the errors obey the same
    if scheme == formats.ASYM:
        s = ocache.raw_decode(c["k_scale"], formats.F16)
    else:
        s = np.asarray(c["k_scale"], np.float64)
    if axis == formats.CHANNEL:
        s_row = np.repeat(s[:, :, : (n + g - 1) // g], g, axis=2)[:, :, :n]
    else:
        s_row = np.broadcast_to(s[:, :, :n, None], (B, H, n, D))
    lim = np.sqrt(((s_row * (0.5 + 2.0 ** -20)) ** 2).sum(axis=-1))
    err = np.linalg.norm(back - k, axis=-1)
    assert np.all(err <= lim * (1 + 1e-5) + 1e-4)
    # the stored basis holds the rotated keys, elementwise within s / 2
    stored = ocache._deq_slab_stored(fmt, c, formats.KEYS, 0, 0, 0, n)
    y = rotate.wht_f32(k[0, 0])
    assert np.all(np.abs(stored - y) <= s_row[0, 0] * (0.5 + 2.0 ** -20) + 1e-6)
    assert np.linalg.norm(stored - k[0, 0]) > np.linalg.norm(back[0, 0] - k[0, 0])


def _key_error(fmt, k):
    B, H, n, _ = k.shape
    c = _cache(fmt, B, H, n)
    ocache.quantize(fmt, c, formats.KEYS, k, 0, n)
    kh = ocache.dequantize(fmt, c, formats.KEYS, 0, n)
    return kh, np.linalg.norm(kh - k) / np.linalg.norm(k)


def test_rotation_tames_an_outlier_channel_under_per_token_grouping():
    """[K4V2] "Rotation Integration": the gain of key-only rotation comes from the key
    outliers.  With per-token INT8 key groups and three channels scaled x10, the key
    error and the attention error both drop when the keys are rotated first."""
    B, H, n, D = 1, 1, 256, 128
    k = _outlier_keys(B, H, n, D, 21)
    rng = np.random.default_rng(22)
    q = rng.standard_normal((4, D))
    v = rng.standard_normal((n, D))
    ref = attention(q, k[0, 0], v, 1.0 / math.sqrt(D))
    errs, atts = {}, {}
    for rot in (0, 1):
        fmt = formats.Format(**synth._fmt(src_dtype=formats.F32, k_scheme=formats.SYM8, k_bits=8,
                                          k_axis=formats.TOKEN, k_rotate=rot))
        kh, errs[rot] = _key_error(fmt, k)
        atts[rot] = rel_l2(attention(q, kh[0, 0], v, 1.0 / math.sqrt(D)), ref)
    assert errs[1] < 0.5 * errs[0]
    assert atts[1] < atts[0]


def test_rotation_tames_heavy_tailed_keys_under_per_channel_k4():
    """[TQ] "Fat-Tail Robustness": after the transform the marginals of heavy-tailed
    keys concentrate, so a per-channel 4-bit group spends its range on the bulk.  On
    Student-t (nu = 2) keys the K4 reconstruction error drops with the rotation."""
    B, H, n, D = 2, 2, 256, 128
    rng = np.random.default_rng(31)
    k = rng.standard_t(2, size=(B, H, n, D)).astype(np.float32).astype(np.float64)
    e = {}
    for rot in (0, 1):
        fmt = formats.Format(**synth._fmt(src_dtype=formats.F32, k_rotate=rot))
        _, e[rot] = _key_error(fmt, k)
    assert e[1] < 0.9 * e[0]
