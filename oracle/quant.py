"""Per-group quantizer rules, restated from the pages in float64 with the fp32 / fp16
steps spelled out.

Symmetric INT8 -- [AXES] "What rows and columns mean":
    scale = max|group| / 127 ; code = clip(round(x / scale), -127, 127) ;
    x_hat = code * scale ; a zero group uses scale 1 ([AXES] "Reproduce" notes).
    Readings: round is half-to-even (numpy's round, which the page's code runs on);
    the division is an fp32 division (sources and scales are float32 on that page).

Asymmetric b-bit (keys per channel, values per token, [KVQ] "Approach" and the
ablation table; the min/max form is the KIVI-style quantizer the pages compare with;
the pages print no formula, so this is the plainest reading):
    z = fp16 rounded down from min, s = fp16 rounded up from fl32(fl32(max - z) / (2^b - 1)),
    code = clip(rint(fl32(fl32(x - z) / s)), 0, 2^b - 1), x_hat = fl32(code * s + z).
    Rounding z down and s up keeps every element within s/2 of its reconstruction.

Non-uniform 3-bit codebook (nuq3) with per-vector dense-and-sparse outliers
([KVQ] "Approach", "per-vector outlier thresholds" in the ablation table):
    the k largest |x| of a vector (ties: lower index) are kept as fp16 outliers and
    left out of min / max; z = fp16(fl32(fl32(mx + mn) * 0.5)),
    s = fp16 rounded up from max(fl32(mx - z), fl32(z - mn)),
    y = fl32(fl32(clip(x, mn, mx) - z) / s), code = #{ j : y > fl32(fl32(C_j + C_j+1) * 0.5) }
    (the nearest centroid, an exact midpoint going to the lower one),
    x_hat = fl32(C[code] * s + z), replaced by the fp16 outlier value where one is kept.

Pinned by tests/test_oracle_quant.py (code ranges, the |x - x_hat| <= s/2 bound, zero
and constant groups, the absmax element mapping to +-127, brute-force nearest
centroid, the uniform-codebook special case, the top-k rule on tiny vectors).
"""
from __future__ import annotations

import numpy as np

from . import fp


class RejectedInput(ValueError):
    """NaN or Inf in a quantizer input ([AXES]: NaN/Inf inputs are rejected)."""


class RangeExceeded(ValueError):
    """A scale, zero-point or outlier value does not fit fp16."""


def check_finite(x):
    if not np.all(np.isfinite(x)):
        raise RejectedInput("non-finite input")


# ---- symmetric INT8 -----------------------------------------------------------

def sym8_scale(m):
    """fp32 scale from the group's max |x| (float64 array of fp32 values)."""
    m = np.asarray(m, np.float64)
    s = fp.div32(m, 127.0)
    return np.where(m == 0.0, 1.0, s)


def sym8_encode(x, s):
    q = fp.div32(x, s)
    return np.clip(fp.rint_even(q), -127, 127).astype(np.int8)


def sym8_decode(code, s):
    return fp.mul32(np.asarray(code, np.float64), s)


# ---- asymmetric b-bit ---------------------------------------------------------

def asym_params(mn, mx, bits):
    """(s, z) as float64 values of fp16 numbers."""
    mn = np.asarray(mn, np.float64)
    mx = np.asarray(mx, np.float64)
    z = fp.f16(mn, "rd")
    d = fp.sub32(mx, z)
    t = fp.div32(d, float(2 ** bits - 1))
    s = fp.f16(t, "ru")
    s = np.where(s == 0.0, 1.0, s)
    if not (np.all(np.isfinite(z)) and np.all(np.isfinite(s))):
        raise RangeExceeded("asym scale / zero-point beyond fp16")
    return s, z


def asym_encode(x, s, z, bits):
    u = fp.sub32(x, z)
    q = fp.div32(u, s)
    return np.clip(fp.rint_even(q), 0, 2 ** bits - 1).astype(np.int64)


def asym_decode(code, s, z):
    # code * s is exact in fp32 (<= 8-bit integer times an 11-bit significand)
    return fp.add32(fp.mul32(np.asarray(code, np.float64), s), z)


# ---- nuq3 ---------------------------------------------------------------------

def nuq_params(mn, mx):
    mn = np.asarray(mn, np.float64)
    mx = np.asarray(mx, np.float64)
    h = fp.mul32(fp.add32(mx, mn), 0.5)
    z = fp.f16(h, "rn")
    a = fp.sub32(mx, z)
    b = fp.sub32(z, mn)
    s = fp.f16(np.maximum(a, b), "ru")
    s = np.where(s == 0.0, 1.0, s)
    if not (np.all(np.isfinite(z)) and np.all(np.isfinite(s))):
        raise RangeExceeded("nuq scale / zero-point beyond fp16")
    return s, z


def nuq_midpoints(C):
    C = np.asarray(C, np.float64)
    return fp.mul32(fp.add32(C[:-1], C[1:]), 0.5)


def nuq_encode(x, s, z, C):
    y = fp.div32(fp.sub32(x, z), s)
    mids = nuq_midpoints(C)
    return (np.asarray(y)[..., None] > mids).sum(axis=-1).astype(np.int64)


def nuq_decode(code, s, z, C):
    C = np.asarray(C, np.float64)
    # C[code] * s is exact in fp32 (two 11-bit significands)
    return fp.add32(fp.mul32(C[np.asarray(code)], s), z)


def topk_outliers(vec, k):
    """Indices of the k largest |x| of a 1-D vector, ties to the lower index,
    returned in ascending index order."""
    vec = np.asarray(vec, np.float64)
    k = min(k, vec.shape[0])
    if k <= 0:
        return np.zeros(0, np.int64)
    # a stable sort of -|x| keeps equal magnitudes in index order
    order = np.argsort(-np.abs(vec), kind="stable")
    return np.sort(order[:k]).astype(np.int64)


def dense_minmax(vec, outlier_idx):
    """min and max over the entries that are not outliers (0, 0 when none remain)."""
    mask = np.ones(vec.shape[0], bool)
    mask[outlier_idx] = False
    rest = vec[mask]
    if rest.size == 0:
        return 0.0, 0.0
    return float(rest.min()), float(rest.max())
