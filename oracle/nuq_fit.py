"""Codebook for the 3-bit non-uniform datatype (nuq3).

[KVQ] "Approach" derives the nuqX levels offline by sensitivity-weighted k-means;
the Fisher weights need gradients of a trained model on a dataset, which is out of
scope.  The plainest stand-in, used here: unweighted 1-D Lloyd k-means (float64,
100 iterations, initial centroids at the (j + 1/2)/8 quantiles) over values
normalized per vector to [-1, 1] by the vector's midpoint and half-range (the
NormalFloat convention the page says KVQuant builds on), with the vector's outliers
left out, then rounded to fp16 and sorted.

Pinned (tests/test_oracle_nuq_fit.py): Lloyd recovers eight point masses, gives equal
cells on a uniform grid and the brute-force best split for k = 2; the normalization maps
the dense range onto [-1, 1] without the outliers.  Parity unpinned: the centroid values
for real data (the page gives none).  The fit only produces an input (the codebook)
that both the library and the oracle then take as given.
"""
from __future__ import annotations

import numpy as np

from . import fp, quant


def lloyd_1d(samples, k=8, iters=100):
    x = np.sort(np.asarray(samples, np.float64).ravel())
    c = np.quantile(x, (np.arange(k) + 0.5) / k)
    for _ in range(iters):
        mids = (c[:-1] + c[1:]) / 2.0
        lab = np.searchsorted(mids, x, side="left")   # a value on a midpoint goes low
        for j in range(k):
            sel = x[lab == j]
            if sel.size:
                c[j] = sel.mean()
        c = np.sort(c)
    return c


def normalized_vectors(vectors, n_outliers):
    """Each row of `vectors` mapped to [-1, 1] by its dense midpoint / half-range."""
    out = []
    for v in np.asarray(vectors, np.float64):
        idx = quant.topk_outliers(v, n_outliers)
        mn, mx = quant.dense_minmax(v, idx)
        keep = np.ones(v.shape[0], bool)
        keep[idx] = False
        half = (mx - mn) / 2.0
        if half > 0:
            out.append((v[keep] - (mx + mn) / 2.0) / half)
    return np.concatenate(out) if out else np.zeros(0)


def fit_codebook(vectors, n_outliers, k=8):
    c = lloyd_1d(normalized_vectors(vectors, n_outliers), k)
    c = np.clip(fp.f16(c, "rn"), -1.0, 1.0)
    return np.sort(c)
