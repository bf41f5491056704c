"""Pins of oracle.salience ([MIX] Figure 3: A = I * S ranks key channels)."""
import numpy as np

from oracle import salience


def test_query_aware_ranking_beats_key_scale():
    # Channel 0: large key range, tiny |Q| (a "blue dot" of Figure 3(a)).
    # Channel 1: small key range, large |Q|.  Channel 2: moderate both.
    G, R, D = 2, 4, 4
    q = np.zeros((G, R, D))
    q[:, :, 0] = 0.01
    q[:, :, 1] = 4.0
    q[:, :, 2] = 1.0
    q[:, :, 3] = 0.5
    k = np.zeros((R, D))
    k[:, 0] = [-50, 50, 0, 0]       # S = 100, I = 0.01 -> A = 1
    k[:, 1] = [0, 1, 0.5, 0]        # S = 1,   I = 4    -> A = 4
    k[:, 2] = [-1, 1, 0, 0]         # S = 2,   I = 1    -> A = 2
    k[:, 3] = [0, 0, 0, 0]          # S = 0             -> A = 0
    A, order = salience.key_salience(q, k)
    np.testing.assert_allclose(A, [1.0, 4.0, 2.0, 0.0])
    assert order.tolist() == [1, 2, 0, 3]
    # ranking by key scale alone would have put channel 0 first
    assert int(np.argmax(k.max(0) - k.min(0))) == 0


def test_ties_go_to_lower_channel():
    q = np.ones((1, 2, 6))
    k = np.zeros((2, 6))
    k[1, :] = [1, 2, 2, 1, 2, 0]
    A, order = salience.key_salience(q, k)
    assert order.tolist() == [1, 2, 4, 0, 3, 5]


def test_mean_over_heads_and_rows():
    r = np.random.default_rng(0)
    q = r.standard_normal((5, 16, 8))
    k = r.standard_normal((16, 8))
    A, order = salience.key_salience(q, k)
    want = np.abs(q).mean(axis=(0, 1)) * (k.max(0) - k.min(0))
    np.testing.assert_allclose(A, want, rtol=1e-14)
    assert sorted(order.tolist()) == list(range(8))


def test_tiers_partition_channels():
    order = np.arange(128)[::-1]
    hi, mid, lo = salience.tiers(order, 8, 24)
    assert len(hi) == 8 and len(mid) == 24 and len(lo) == 96
    assert sorted(np.concatenate([hi, mid, lo]).tolist()) == list(range(128))
    assert hi.tolist() == list(range(127, 119, -1))
