"""Key-only Walsh-Hadamard rotation.

TEST INFRASTRUCTURE ONLY (see the package docstring).

[K4V2] "Quantize What Counts: More for Keys, Less for Values", Results, "Rotation
Integration": rotating the keys alone, before K4V2 quantization, recovers most of the
accuracy of K4V4, because the rotation spreads the key outlier channels over all
channels.  [TQ] "Statistical Inference and Quality Measures of KV Cache Quantisations
Inspired by TurboQuant", Technical Summary (the KQV scheme): the rotation is a
Walsh-Hadamard transform, which makes the marginals of a heavy-tailed vector tame
("Fat-Tail Robustness").

Reading (the pages name the transform, not its normalisation, order or precision):
  * the orthonormal transform y = H_D x / sqrt(D), H_D the Sylvester-ordered
    Hadamard matrix (H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]), no random signs;
  * the rotated key decides the quantized codes, so its precision is part of the
    stored format: the transform is evaluated in fp32 as the in-place butterfly
    over strides h = 1, 2, 4, ..., D/2 (each pair (i, i + h), i & h = 0, becomes
    (a + b, a - b), each sum rounded to fp32), followed by one fp32 product with
    c = fl32(1 / sqrt(D));
  * H_D / sqrt(D) is symmetric and orthogonal, hence its own inverse: the same
    transform maps reconstructed keys back, and a query rotated by it gives
    q' . k' = q . k, which is how decode attention reads rotated keys.

Pins (tests/test_oracle_rotate.py): the fp32 butterfly against the float64 product
with scipy's Hadamard matrix, within the error bound derived there; one-hot inputs
map to constant-magnitude vectors with the Sylvester signs; exact involution on
small integers for D = 64 and 256 (where 1/sqrt(D) is a power of two); norm
preservation; and the effect the pages report (lower key error under an outlier
channel with per-token grouping).
"""
from __future__ import annotations

import numpy as np


def rot_scale(D: int) -> np.float32:
    """c = fl32(1 / sqrt(D)) (division and square root correctly rounded in float64)."""
    return np.float32(1.0 / np.sqrt(np.float64(D)))


def wht_f32(x) -> np.ndarray:
    """Normalised Walsh-Hadamard transform of the last axis of x, in fp32 as stated in
    the module docstring.  x: values exactly representable in fp32; returns float64
    holding fp32 values."""
    y = np.array(x, dtype=np.float32, copy=True)
    D = y.shape[-1]
    assert D >= 1 and D & (D - 1) == 0
    lead = y.shape[:-1]
    h = 1
    while h < D:
        blocks = y.reshape(lead + (D // (2 * h), 2, h))
        a = blocks[..., 0, :]
        b = blocks[..., 1, :]
        y = np.stack([a + b, a - b], axis=-2).reshape(lead + (D,))   # fp32 sums
        h *= 2
    y = y * rot_scale(D)                                                # one fp32 product
    return y.astype(np.float64)
