"""KQV: scalar MSE codes for the keys, scalar codes plus a 1-bit QJL sketch of the
residual for the values, both after a Walsh-Hadamard rotation.

TEST INFRASTRUCTURE ONLY (see the package docstring).  The float64 functions below state
the scheme; the "stored format" section at the end states the fp32 arithmetic the
library's kernels store codes with, which decides every code and sign bit.

[TQ] "Statistical Inference and Quality Measures of KV Cache Quantisations Inspired by
TurboQuant", Technical Summary: "Theoretical Framework" (a coordinate of a uniformly
random unit vector in d dimensions is Beta((d-1)/2, (d-1)/2)-distributed on [-1, 1]),
"Quantization Schemes" (KQV: rotation of K and V; K by n-bit scalar MSE codes; V by
(n-1)-bit scalar MSE codes and a 1-bit QJL sketch) and "Key Contributions" (the sketch
is unbiased; its inner-product variance is pi/2 ||r||^2 / d).

Readings (the page names the pieces, not their constants):
  * "n bits" is a per-coordinate budget: K n bits a coordinate, V n - 1 bits and one
    sketch bit;
  * the scalar MSE quantizer is the Lloyd-Max quantizer of that Beta marginal, applied to
    the rotated vector divided by its norm; the norm is kept in float64 here;
  * the sketch of a residual r is s = sign(S r) in {-1, +1}^m (sign(0) = +1) with the
    norm ||r|| kept, S an m x d matrix of independent N(0, 1) entries that is an input
    (the method's random numbers are drawn outside and passed in); m = d;
  * the estimators are <q, r> ~ sqrt(pi/2) / m ||r|| <S q, s> and
    r ~ sqrt(pi/2) / m ||r|| S^T s (both unbiased over S);
  * the rotation is the orthonormal Sylvester Walsh-Hadamard matrix in float64.

Pins (tests/test_oracle_kqv.py): at d = 3 the marginal is uniform and Lloyd-Max is the
uniform quantizer; the 1-bit centroid is E|x| in closed form at every d; for large d the
scaled centroids approach the Gaussian Lloyd-Max table; the sketch's mean and variance
match the closed forms by Monte Carlo over seeded S; and the page's effect holds at the
4-bit budget: KQV keys give a lower attention KL divergence than QKQV keys.
"""
from __future__ import annotations

import math

import numpy as np
import scipy.linalg


def marginal_pdf(x, d):
    """Density of one coordinate of a uniformly random unit vector in R^d, on [-1, 1]:
    (1 - x^2)^((d - 3) / 2) / B(1/2, (d - 1)/2)."""
    x = np.asarray(x, np.float64)
    logc = math.lgamma(d / 2.0) - math.lgamma(0.5) - math.lgamma((d - 1) / 2.0)
    inside = np.abs(x) < 1.0
    xi = np.where(inside, x, 0.0)
    return np.where(inside, np.exp(logc + (d - 3) / 2.0 * np.log1p(-xi * xi)), 0.0)


def lloyd_max(bits, d, iters=300, grid=400000):
    """Lloyd-Max centroids (2^bits, ascending) of the marginal at dimension d: thresholds at
    midpoints, centroids at the conditional means, by midpoint quadrature on a uniform grid
    over [-L, L], L = min(1, 14 / sqrt(d)) (the mass beyond 14 standard deviations is below
    1e-40).  The density is symmetric, so each iteration keeps the centroids symmetric
    (on a discrete grid an off-centre fixed point, one grid point away, exists as well);
    an even number of grid points keeps the central threshold 0 off the grid."""
    k = 1 << bits
    L = min(1.0, 14.0 / math.sqrt(d))
    x = (np.arange(grid) + 0.5) / grid * 2.0 * L - L
    w = marginal_pdf(x, d)
    w = w / w.sum()
    cdf = np.cumsum(w)
    c = np.interp((np.arange(k) + 0.5) / k, cdf, x)
    for _ in range(iters):
        t = (c[:-1] + c[1:]) / 2.0
        lab = np.searchsorted(t, x, side="left")
        mass = np.bincount(lab, weights=w, minlength=k)
        mom = np.bincount(lab, weights=w * x, minlength=k)
        c = np.where(mass > 0, mom / np.maximum(mass, 1e-300), c)
        c = (c - c[::-1]) / 2.0   # the density is symmetric, so is its Lloyd-Max quantizer
    return np.sort(c)


def rotation(d):
    """The orthonormal Walsh-Hadamard matrix H_d / sqrt(d) (symmetric, its own inverse)."""
    return scipy.linalg.hadamard(d).astype(np.float64) / math.sqrt(d)


def scalar_encode(y, cb):
    """Codes of y / ||y|| against the centroids cb (nearest, a midpoint going low), and ||y||."""
    y = np.asarray(y, np.float64)
    nrm = float(np.linalg.norm(y))
    u = y / nrm if nrm > 0 else np.zeros_like(y)
    mids = (cb[:-1] + cb[1:]) / 2.0
    return np.searchsorted(mids, u, side="left"), nrm


def scalar_decode(codes, nrm, cb):
    return nrm * np.asarray(cb)[codes]


def qjl_sketch(r, S):
    """(signs of S r in {-1, +1}, ||r||)."""
    p = np.asarray(S, np.float64) @ np.asarray(r, np.float64)
    return np.where(p >= 0.0, 1.0, -1.0), float(np.linalg.norm(r))


def qjl_inner(q, signs, rnorm, S):
    """Unbiased estimate of <q, r> from the sketch of r."""
    m = S.shape[0]
    return math.sqrt(math.pi / 2.0) / m * rnorm * float((np.asarray(S) @ np.asarray(q, np.float64)) @ signs)


def qjl_vector(signs, rnorm, S):
    """Unbiased estimate of r itself from its sketch."""
    m = S.shape[0]
    return math.sqrt(math.pi / 2.0) / m * rnorm * (np.asarray(S).T @ signs)


def kqv_key(k, bits, cb=None):
    """Reconstruction of a key row under KQV: rotate, n-bit scalar codes, back."""
    d = k.shape[-1]
    R = rotation(d)
    cb = lloyd_max(bits, d) if cb is None else cb
    codes, nrm = scalar_encode(R @ k, cb)
    return R @ scalar_decode(codes, nrm, cb)


def kqv_value(v, bits, S, cb=None):
    """Reconstruction of a value row under KQV: rotate, (n-1)-bit scalar codes, plus the
    sketch estimate of the residual, back."""
    d = v.shape[-1]
    R = rotation(d)
    cb = lloyd_max(bits - 1, d) if cb is None else cb
    y = R @ v
    codes, nrm = scalar_encode(y, cb)
    yh = scalar_decode(codes, nrm, cb)
    signs, rn = qjl_sketch(y - yh, S)
    return R @ (yh + qjl_vector(signs, rn, S))


def qkqv_key(k, bits, S, cb=None):
    """A key row under QKQV (the comparison scheme): (n-1)-bit scalar codes plus the sketch
    of the residual, like a KQV value.  Its scores q . k^ are the scalar part plus the
    sketch's unbiased inner-product estimate."""
    return kqv_value(k, bits, S, cb)


# ---- stored format (the library's KVQ_KQV scheme) ------------------------------------
# The float64 definitions above leave the precision of every decision open.  The stored
# format fixes it in fp32, each operation one IEEE rounding and no fused multiply-add, so
# that codes and sign bits are reproducible:
#   y     = the key-only rotation's fp32 Walsh-Hadamard transform (oracle.rotate.wht_f32);
#   ||y|| = fl32(sqrt(T(fl32(y_c * y_c)))), T the pairwise tree over the channel index
#           (level 1 adds elements 2i and 2i + 1, level 2 the results 2i and 2i + 1, ...,
#           every sum rounded to fp32);
#   u_c   = fl32(y_c / ||y||)  (0 when ||y|| = 0);
#   code  = #{j : u_c > m_j},  m_j = fl32(fl32(C_j + C_{j+1}) * 0.5), C the fp32 centroids;
#   values also: yh_c = fl32(||y|| * C[code_c]), r_c = fl32(y_c - yh_c),
#           ||r|| = fl32(sqrt(T(fl32(r_c * r_c)))), and sign bit i = (T_c(fl32(S_ic * r_c)) >= 0).
# Reconstruction (decode, dequantize) is a real-valued formula evaluated in float64 here:
#   k^ = R (||y|| C[code]),   v^ = R (||y|| C[code] + sqrt(pi/2) / m ||r|| S^T s),
# R the same orthonormal transform (its own inverse), s_i = +1 for a set bit, -1 otherwise.


def tree_sum_f32(a):
    """Pairwise sum over the last axis (a power of two long) in fp32: each level adds the
    elements 2i and 2i + 1 of the previous one, every sum rounded to fp32."""
    a = np.asarray(a, np.float32)
    while a.shape[-1] > 1:
        a = (a[..., 0::2] + a[..., 1::2]).astype(np.float32)
    return a[..., 0]


def centroids_f32(cb):
    """The fp32 centroids and their fp32 midpoints fl32(fl32(C_j + C_{j+1}) * 0.5)."""
    c = np.asarray(cb, np.float32)
    mids = ((c[:-1] + c[1:]).astype(np.float32) * np.float32(0.5)).astype(np.float32)
    return c, mids


def stored_encode(x, cb, S=None):
    """Rows x [n, D] of exact fp32 source values -> (codes [n, D], norms fp32 [n]) for keys;
    with S (fp32 [D, D], values): also (signs bool [n, D], residual norms fp32 [n])."""
    from . import rotate
    x = np.asarray(x, np.float32)
    y = np.asarray(rotate.wht_f32(x), np.float32)
    nrm = np.sqrt(tree_sum_f32((y * y).astype(np.float32))).astype(np.float32)
    safe = np.where(nrm > 0, nrm, np.float32(1.0)).astype(np.float32)
    u = np.where(nrm[..., None] > 0, (y / safe[..., None]).astype(np.float32), np.float32(0.0))
    c, mids = centroids_f32(cb)
    codes = (u[..., None] > mids).sum(axis=-1)
    if S is None:
        return codes, nrm
    yh = (nrm[..., None] * c[codes]).astype(np.float32)
    r = (y - yh).astype(np.float32)
    rn = np.sqrt(tree_sum_f32((r * r).astype(np.float32))).astype(np.float32)
    S = np.asarray(S, np.float32)
    t = tree_sum_f32((S[None, :, :] * r[:, None, :]).astype(np.float32))   # [n, m]
    return codes, nrm, t >= 0, rn


def stored_key(codes, nrm, cb):
    """k^ [n, D] float64 from stored key codes and norms."""
    R = rotation(np.asarray(codes).shape[-1])
    c = np.asarray(cb, np.float32).astype(np.float64)
    return (np.asarray(nrm, np.float64)[..., None] * c[codes]) @ R


def stored_value(codes, nrm, signs, rn, cb, S):
    """v^ [n, D] float64 from stored value codes, norms, sign bits and residual norms."""
    D = np.asarray(codes).shape[-1]
    R = rotation(D)
    S = np.asarray(S, np.float32).astype(np.float64)
    c = np.asarray(cb, np.float32).astype(np.float64)
    sv = np.where(np.asarray(signs), 1.0, -1.0)
    yh = np.asarray(nrm, np.float64)[..., None] * c[codes]
    sk = math.sqrt(math.pi / 2.0) / S.shape[0] * np.asarray(rn, np.float64)[..., None] * (sv @ S)
    return (yh + sk) @ R
