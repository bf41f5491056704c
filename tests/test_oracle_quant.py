"""Pins of the quantizer rules in oracle.quant against what the pages and the
mathematics fix: code ranges, the half-step error bound, zero and constant groups,
the absmax element at +-127, a brute-force nearest centroid, a uniform-codebook
special case and the top-k outlier rule."""
import numpy as np
import pytest

from oracle import fp, quant


def _f32(x):
    return np.asarray(x, np.float32).astype(np.float64)


# ---- symmetric INT8 ([AXES] "What rows and columns mean") ----------------------

def test_sym8_range_and_bound():
    r = np.random.default_rng(0)
    for trial in range(50):
        x = _f32(r.standard_normal(64) * np.exp(r.uniform(-20, 20)))
        m = np.abs(x).max()
        s = quant.sym8_scale(m)
        c = quant.sym8_encode(x, s)
        assert c.min() >= -127 and c.max() <= 127
        xh = c.astype(np.float64) * s
        # no clipping can occur, so every element is within half a step (plus the fp32
        # quotient's rounding)
        assert np.all(np.abs(x - xh) <= s * (0.5 + 2.0 ** -20))
        # the absmax element lands on +-127
        i = np.argmax(np.abs(x))
        assert abs(int(c[i])) == 127


def test_sym8_zero_group_uses_scale_one():
    s = quant.sym8_scale(0.0)
    assert s == 1.0
    assert np.all(quant.sym8_encode(np.zeros(8), s) == 0)


def test_sym8_ties_round_to_even():
    # m = 127 -> s = 1 exactly; x = k + 0.5 must go to the even neighbour
    s = quant.sym8_scale(127.0)
    assert s == 1.0
    x = np.array([0.5, 1.5, 2.5, -0.5, -1.5, 126.5, -126.5])
    assert quant.sym8_encode(x, s).tolist() == [0, 2, 2, 0, -2, 126, -126]


def test_sym8_scale_is_fp32_division():
    m = _f32(3.3)
    assert quant.sym8_scale(m) == float(np.float32(m) / np.float32(127))


# ---- asymmetric b-bit ----------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 4, 8])
def test_asym_range_and_bound(bits):
    r = np.random.default_rng(bits)
    for trial in range(100):
        x = _f32(r.standard_normal(128) * np.exp(r.uniform(-6, 6)) + r.uniform(-5, 5))
        s, z = quant.asym_params(x.min(), x.max(), bits)
        # metadata are fp16 numbers, z <= min, (2^b - 1) s >= max - z
        assert fp.f16(z) == z and fp.f16(s) == s
        assert z <= x.min()
        assert (2 ** bits - 1) * s >= (x.max() - z) * (1 - 2.0 ** -22)
        c = quant.asym_encode(x, s, z, bits)
        assert c.min() >= 0 and c.max() <= 2 ** bits - 1
        xh = quant.asym_decode(c, s, z)
        assert np.all(np.abs(x - xh) <= s * (0.5 + 2.0 ** -20))


def test_asym_constant_group():
    x = np.full(16, 0.75)          # representable in fp16
    s, z = quant.asym_params(x.min(), x.max(), 4)
    assert s == 1.0 and z == 0.75
    c = quant.asym_encode(x, s, z, 4)
    assert np.all(c == 0)
    assert np.all(quant.asym_decode(c, s, z) == 0.75)


def test_asym_decode_product_is_exact():
    # code * s exact in fp32: fused and unfused evaluation agree
    r = np.random.default_rng(5)
    s = fp.f16(np.abs(r.standard_normal(1000)) + 1e-3, "ru")
    z = fp.f16(r.standard_normal(1000), "rd")
    c = r.integers(0, 256, 1000)
    exact = c * s + z                     # float64, exact product and sum
    np.testing.assert_array_equal(quant.asym_decode(c, s, z), fp.f32(exact))


def test_asym_rejects_fp16_overflow():
    with pytest.raises(quant.RangeExceeded):
        quant.asym_params(-1e6, 1.0, 4)


# ---- nuq3 ----------------------------------------------------------------------

def _brute_nearest(y, C):
    """Index of the nearest centroid, an exact tie going to the lower one."""
    out = []
    for v in np.atleast_1d(y):
        d = [abs(v - c) for c in C]
        best = min(range(len(C)), key=lambda j: (d[j], j))
        out.append(best)
    return np.array(out)


def test_nuq_encode_is_nearest_centroid():
    C = fp.f16(np.array([-1.0, -0.62, -0.31, -0.09, 0.1, 0.33, 0.64, 1.0]))
    r = np.random.default_rng(1)
    y = _f32(r.uniform(-1.2, 1.2, 20000))
    mids = quant.nuq_midpoints(C)
    y = np.concatenate([y, mids])          # exact midpoints go low
    code = quant.nuq_encode(y, 1.0, 0.0, C)
    np.testing.assert_array_equal(code, _brute_nearest(y, C))


def test_nuq_uniform_codebook_is_uniform_quantizer():
    # C_j = (j - 3.5) / 4: eight equally spaced levels.  With z, s from the group and
    # y = (x - z) / s, the code is the textbook uniform quantizer on [-1, 1] with step
    # 1/4: floor(4 y + 4) clipped to [0, 7] (ties at the cell edges go low).
    C = (np.arange(8) - 3.5) / 4
    r = np.random.default_rng(2)
    for trial in range(50):
        x = _f32(r.standard_normal(128) * 3)
        s, z = quant.nuq_params(x.min(), x.max())
        y = fp.div32(fp.sub32(x, z), s)
        code = quant.nuq_encode(x, s, z, C)
        t = 4 * y + 4
        want = np.clip(np.ceil(t) - 1, 0, 7)
        np.testing.assert_array_equal(code, want)


def test_nuq_params_cover_the_range():
    r = np.random.default_rng(3)
    for trial in range(100):
        x = _f32(r.standard_normal(64) * np.exp(r.uniform(-5, 5)))
        s, z = quant.nuq_params(x.min(), x.max())
        assert z - s <= x.min() and x.max() <= z + s


def test_topk_outliers_ties_lower_index():
    v = np.array([1.0, -3.0, 3.0, 0.5, -3.0])
    assert quant.topk_outliers(v, 2).tolist() == [1, 2]
    assert quant.topk_outliers(v, 3).tolist() == [1, 2, 4]
    assert quant.topk_outliers(np.array([2.0]), 2).tolist() == [0]
    # brute force over all small vectors with repeated magnitudes
    r = np.random.default_rng(4)
    for trial in range(200):
        v = r.integers(-3, 4, 7).astype(float)
        k = int(r.integers(0, 5))
        got = quant.topk_outliers(v, k)
        want = sorted(sorted(range(7), key=lambda i: (-abs(v[i]), i))[:k])
        assert got.tolist() == want


def test_reject_nonfinite():
    with pytest.raises(quant.RejectedInput):
        quant.check_finite(np.array([1.0, np.nan]))
    with pytest.raises(quant.RejectedInput):
        quant.check_finite(np.array([np.inf]))
