"""MixKVQ key-channel salience ([MIX] Figure 3 caption and Figure 4 caption).

Figure 3 defines the salience of key channel d as A_d = I_d * S_d, where I_d is the
average activation intensity of the query in channel d and S_d the key scale of the
channel; the channels with the largest A keep BF16, the next ones INT4, the rest INT2
(bar colours of Figure 3(b)).  Figure 4 recomputes the scores every R tokens over the
window of a full-precision buffer of size R.

Readings (the captions leave these open):
  * I_d averages |Q[d]| over the R query rows of the window and over the G query
    heads that share the KV head;  the sum is taken in float64 in the order
    (head, then row), then divided by G * R;
  * S_d is the range max - min of K[:, d] over the window, in float64;
  * ranking is by descending A_d, ties to the lower channel index.

Pinned by tests/test_oracle_salience.py (a hand-built window in which one channel has
large |Q| but a small key range and another the reverse, as in Figure 3's argument;
ties; tier sizes).
"""
from __future__ import annotations

import numpy as np


def key_salience(q_win, k_win):
    """q_win [G, R, D], k_win [R, D] (exact source values) -> (A [D] float64, order [D])."""
    q_win = np.asarray(q_win, np.float64)
    k_win = np.asarray(k_win, np.float64)
    G, R, D = q_win.shape
    acc = np.zeros(D, np.float64)
    for h in range(G):
        for r in range(R):
            acc = acc + np.abs(q_win[h, r])
    intensity = acc / float(G * R)
    key_range = k_win.max(axis=0) - k_win.min(axis=0)
    A = intensity * key_range
    order = sorted(range(D), key=lambda d: (-A[d], d))
    return A, np.array(order, dtype=np.uint8)


def tiers(order, n_hi, n_mid):
    """Channel sets of the BF16, INT4 and INT2 tiers for one group."""
    order = np.asarray(order, np.int64)
    return order[:n_hi], order[n_hi:n_hi + n_mid], order[n_hi + n_mid:]
