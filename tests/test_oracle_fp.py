"""Pins of oracle.fp (rounding from the IEEE-754 definition) against numpy's own
float16 / float32 conversions and against the defining properties of the directed
roundings."""
import numpy as np
import pytest

from oracle import fp


def _samples(seed=0, n=200000):
    r = np.random.default_rng(seed)
    x = r.standard_normal(n) * np.exp(r.uniform(-30, 30, n))
    # fp16 midpoints and neighbours, subnormal range, overflow edge
    h = np.arange(0, 0x7C00, 7, dtype=np.uint16).view(np.float16).astype(np.float64)
    nxt = np.nextafter(h.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    mids = (h + nxt) / 2
    extra = np.concatenate([h, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                            [65504.0, 65519.99, 65520.0, 65536.0, 1e-8, 2.0 ** -25, 3 * 2.0 ** -26]])
    return np.concatenate([x, extra, -extra])


def test_f16_nearest_matches_numpy():
    x = _samples()
    with np.errstate(over="ignore"):
        want = x.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(fp.f16(x, "rn"), want)


def test_f32_nearest_matches_numpy():
    r = np.random.default_rng(1)
    x = r.standard_normal(200000) * np.exp(r.uniform(-200, 200, 200000))
    with np.errstate(over="ignore"):
        want = x.astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(fp.f32(x, "rn"), want)


@pytest.mark.parametrize("fmt,npdt", [(fp.FP16, np.float16), (fp.FP32, np.float32)])
def test_directed_roundings_bracket(fmt, npdt):
    x = _samples(2, 50000)
    big = float(np.finfo(npdt).max)
    x = x[np.abs(x) < big]
    lo = fp.round_to(x, fmt, "rd")
    hi = fp.round_to(x, fmt, "ru")
    assert np.all(lo <= x) and np.all(x <= hi)
    # representable and adjacent: nothing representable strictly between lo and x
    np.testing.assert_array_equal(lo.astype(npdt).astype(np.float64), lo)
    np.testing.assert_array_equal(hi.astype(npdt).astype(np.float64), hi)
    up_from_lo = np.nextafter(lo.astype(npdt), npdt(np.inf)).astype(np.float64)
    exact = lo == x
    assert np.all(exact | (up_from_lo >= hi))
    assert np.all((lo == hi) == exact)


def test_overflow_rules():
    assert fp.f16(65520.0, "rn") == np.inf
    assert fp.f16(65519.0, "rn") == 65504.0
    assert fp.f16(70000.0, "rd") == 65504.0
    assert fp.f16(70000.0, "ru") == np.inf
    assert fp.f16(-70000.0, "rd") == -np.inf
    assert fp.f16(-70000.0, "ru") == -65504.0


def test_bf16_bits_roundtrip():
    x = np.array([1.0, -2.5, 3.140625, 1e-3], np.float64)
    xb = fp.bf16(x)
    np.testing.assert_array_equal(fp.bf16_from_bits(fp.bf16_bits(xb)), xb)
    assert fp.bf16(1.0 + 2 ** -8) == 1.0          # tie to even
    assert fp.bf16(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6


def test_fp32_ops_are_single_roundings():
    r = np.random.default_rng(3)
    a = r.standard_normal(100000).astype(np.float32)
    b = (r.standard_normal(100000) + 3).astype(np.float32)
    np.testing.assert_array_equal(fp.div32(a, b), (a / b).astype(np.float64))
    np.testing.assert_array_equal(fp.sub32(a, b), (a - b).astype(np.float64))
    np.testing.assert_array_equal(fp.add32(a, b), (a + b).astype(np.float64))
    np.testing.assert_array_equal(fp.mul32(a, b), (a * b).astype(np.float64))
