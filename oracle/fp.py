"""Rounding to fp16 / bf16 / fp32 from the IEEE-754 definition, in float64.

The quantizers fix some steps in reduced precision (fp32 division, fp16 scale and
zero-point with a directed rounding).  This module states those roundings directly:
a finite float64 value x is written as an integer multiple of the target format's
quantum at x's binade (clamped to the subnormal quantum), the multiple is rounded
with the requested mode, and overflow follows IEEE-754 (round-to-nearest and the
direction away from the finite range give infinity; the other directions give the
largest finite value).

Pinned by tests/test_oracle_fp.py: fp16 round-to-nearest equals numpy's float16
conversion; fp32 round-to-nearest equals numpy's float32 conversion; directed modes
bracket x with no representable value in between.
"""
from __future__ import annotations

import numpy as np

# (precision p incl. the implicit bit, minimum normal exponent, maximum exponent)
FP16 = (11, -14, 15)
BF16 = (8, -126, 127)
FP32 = (24, -126, 127)


def _max_finite(fmt):
    p, _, emax = fmt
    return (2.0 - 2.0 ** (1 - p)) * 2.0 ** emax


def round_to(x, fmt, mode: str = "rn") -> np.ndarray:
    """Round float64 values to the format `fmt`; the result is returned as float64.

    mode: 'rn' (nearest, ties to even), 'rd' (toward -inf), 'ru' (toward +inf),
    'rz' (toward zero).
    """
    p, emin, emax = fmt
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, dtype=np.float64, copy=True)
    fin = np.isfinite(x) & (x != 0.0)
    if np.any(fin):
        xf = x[fin]
        _, e = np.frexp(np.abs(xf))          # |x| = m * 2**e, m in [0.5, 1)
        e = np.maximum(e - 1, emin)          # exponent of the leading bit, >= emin
        quantum = np.ldexp(1.0, e - (p - 1))
        q = xf / quantum                     # exact: scaling by a power of two
        if mode == "rn":
            r = np.rint(q)
        elif mode == "rd":
            r = np.floor(q)
        elif mode == "ru":
            r = np.ceil(q)
        elif mode == "rz":
            r = np.trunc(q)
        else:
            raise ValueError(mode)
        y = r * quantum
        big = _max_finite(fmt)
        over_pos = y > big
        over_neg = y < -big
        if mode == "rn":
            y = np.where(over_pos, np.inf, np.where(over_neg, -np.inf, y))
        elif mode == "rd":
            y = np.where(over_pos, big, np.where(over_neg, -np.inf, y))
        elif mode == "ru":
            y = np.where(over_pos, np.inf, np.where(over_neg, -big, y))
        else:
            y = np.where(over_pos, big, np.where(over_neg, -big, y))
        # keep the sign of a result that rounded to zero
        y = np.where(y == 0.0, np.copysign(0.0, xf), y)
        out[fin] = y
    return out


def f16(x, mode="rn"):
    return round_to(x, FP16, mode)


def bf16(x, mode="rn"):
    return round_to(x, BF16, mode)


def f32(x, mode="rn"):
    return round_to(x, FP32, mode)


# ---- bit encodings (for comparing stored bytes) -------------------------------

def f16_bits(x) -> np.ndarray:
    """uint16 encoding of values that are exactly representable in fp16."""
    x = np.asarray(x, dtype=np.float64)
    h = x.astype(np.float16)
    if not np.array_equal(h.astype(np.float64), x, equal_nan=True):
        raise ValueError("value not representable in fp16")
    return h.view(np.uint16)


def f16_from_bits(b) -> np.ndarray:
    return np.asarray(b, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_from_bits(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def bf16_bits(x) -> np.ndarray:
    """uint16 encoding of values that are exactly representable in bf16."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    if not np.array_equal(f.astype(np.float64), x, equal_nan=True):
        raise ValueError("value not representable in bf16")
    u = f.view(np.uint32)
    if np.any(u & np.uint32(0xFFFF)):
        raise ValueError("value not representable in bf16")
    return (u >> np.uint32(16)).astype(np.uint16)


def f32_bits(x) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    if not np.array_equal(f.astype(np.float64), x, equal_nan=True):
        raise ValueError("value not representable in fp32")
    return f.view(np.uint32)


# ---- the fp32 steps of the quantizers ----------------------------------------
# An IEEE fp32 operation is the exact result rounded once to fp32.  For +, -, *
# and / of two fp32 operands the float64 result rounded to fp32 equals that: a
# float64 product of two fp32 values is exact, and for sums and quotients the
# double rounding cannot change the result because 53 >= 2 * 24 + 2.

def add32(a, b):
    return f32(np.asarray(a, np.float64) + np.asarray(b, np.float64))


def sub32(a, b):
    return f32(np.asarray(a, np.float64) - np.asarray(b, np.float64))


def mul32(a, b):
    return f32(np.asarray(a, np.float64) * np.asarray(b, np.float64))


def div32(a, b):
    return f32(np.asarray(a, np.float64) / np.asarray(b, np.float64))


def rint_even(x):
    """Round half to even (numpy's rint)."""
    return np.rint(np.asarray(x, np.float64))
