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


def _f32_patterns(seed, n):
    """Finite float32 values from random bit patterns: normals over the whole exponent
    range, subnormals, exact bf16 ties (low 16 bits 0x8000) and their neighbours, and
    the overflow edge."""
    r = np.random.default_rng(seed)
    bits = r.integers(0, 1 << 32, n, dtype=np.uint64).astype(np.uint32)
    sub = r.integers(1, 1 << 23, n // 4, dtype=np.uint64).astype(np.uint32)          # subnormal
    ties = (r.integers(0, 1 << 16, n // 4, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    near = np.concatenate([ties - 1, ties + 1])
    edge = np.array([0x7F7F7FFF, 0x7F7F8000, 0x7F7F8001, 0x7F7FFFFF, 0x00008000, 0x00018000,
                     0x00000001, 0x007FFFFF, 0x00800000], np.uint32)
    allb = np.concatenate([bits, sub, ties, near, edge])
    allb = np.concatenate([allb, allb ^ np.uint32(0x80000000)])
    x = allb.view(np.float32)
    return x[np.isfinite(x)]


def test_bf16_nearest_matches_torch():
    # bf16 round-to-nearest-even against torch's float32 -> bfloat16 conversion (one
    # rounding: the float32 inputs are exact in float64)
    torch = pytest.importorskip("torch")
    x = _f32_patterns(4, 400000)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(fp.bf16(x.astype(np.float64), "rn"), want)


def test_bf16_directed_roundings_bracket():
    torch = pytest.importorskip("torch")
    x = _f32_patterns(5, 100000).astype(np.float64)
    big = float(torch.finfo(torch.bfloat16).max)
    x = x[np.abs(x) < big]
    lo, hi = fp.bf16(x, "rd"), fp.bf16(x, "ru")
    assert np.all(lo <= x) and np.all(x <= hi)
    # both representable in bf16, adjacent unless exact
    rt = lambda v: torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(rt(lo), lo)
    np.testing.assert_array_equal(rt(hi), hi)
    exact = lo == x
    assert np.all((lo == hi) == exact)
    bl = torch.from_numpy(lo).to(torch.bfloat16)
    up = torch.nextafter(bl, torch.full_like(bl, float("inf"))).to(torch.float64).numpy()
    assert np.all(exact | (up >= hi))
