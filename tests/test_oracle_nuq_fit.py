"""Pins of the nuq3 codebook fit (oracle.nuq_fit): 1-D Lloyd k-means on textbook cases,
the per-vector normalization to [-1, 1], and the shape of the fitted codebook.  (The
centroid values for real data stay unpinned: the pages print none.)"""
import numpy as np

from oracle import fp, nuq_fit


def test_lloyd_recovers_eight_point_masses():
    masses = np.array([-0.9, -0.6, -0.35, -0.1, 0.05, 0.3, 0.55, 0.95])
    x = np.repeat(masses, 37)
    # (each centroid is the float64 mean of 37 equal values: equal up to the sum's rounding)
    np.testing.assert_allclose(nuq_fit.lloyd_1d(x, 8), masses, rtol=0, atol=1e-15)


def test_lloyd_on_a_uniform_grid_gives_equal_cells():
    # 8 m evenly spaced points: the fixed point is 8 equal cells, centroid = cell mean
    m = 25
    x = np.linspace(-1.0, 1.0, 8 * m)
    c = nuq_fit.lloyd_1d(x, 8)
    want = x.reshape(8, m).mean(axis=1)
    np.testing.assert_allclose(c, want, rtol=0, atol=1e-12)


def test_lloyd_two_clusters_brute_force():
    # k = 2 on a small sample: compare with the best split found by brute force
    rng = np.random.default_rng(4)
    x = np.sort(np.concatenate([rng.normal(-2, 0.3, 20), rng.normal(1.5, 0.5, 15)]))
    best = min(range(1, x.size), key=lambda s: ((x[:s] - x[:s].mean()) ** 2).sum() +
               ((x[s:] - x[s:].mean()) ** 2).sum())
    np.testing.assert_allclose(nuq_fit.lloyd_1d(x, 2), [x[:best].mean(), x[best:].mean()], rtol=1e-12)


def test_normalization_maps_the_dense_range_to_unit_interval():
    v = np.array([[3.0, -1.0, 2.0, 40.0, 0.0, 1.0]])     # 40 is the outlier (top-1)
    y = nuq_fit.normalized_vectors(v, 1)
    # dense min -1, max 3: midpoint 1, half-range 2
    np.testing.assert_array_equal(np.sort(y), np.sort((np.array([3.0, -1.0, 2.0, 0.0, 1.0]) - 1.0) / 2.0))
    assert y.min() == -1.0 and y.max() == 1.0
    # a constant vector carries no shape and is left out
    assert nuq_fit.normalized_vectors(np.full((1, 8), 2.5), 0).size == 0


def test_fitted_codebook_is_sorted_fp16_in_unit_interval():
    rng = np.random.default_rng(9)
    c = nuq_fit.fit_codebook(rng.standard_normal((64, 128)), 2)
    assert c.shape == (8,)
    assert np.all(np.diff(c) > 0)
    assert c.min() >= -1.0 and c.max() <= 1.0
    np.testing.assert_array_equal(fp.f16(c), c)
    # symmetric data gives a nearly symmetric codebook
    assert np.abs(c + c[::-1]).max() < 0.05
