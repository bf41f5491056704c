"""Pins of the [AXES] INT8 experiment (oracle.toy) and of the byte accounting
(oracle.formats) against the page's tables, stored under tests/golden/."""
import os

import numpy as np
import pytest

import synth
from oracle import formats, toy

SEEDS = (7, 19, 41)
LENGTHS = (64, 256)


def _load_table(path):
    rows = {}
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        t, s, c, v = line.split()
        rows[(t, s, c)] = float(v)
    return rows


@pytest.fixture(scope="module")
def inputs():
    return [synth.toy(s, N) for s in SEEDS for N in LENGTHS]


@pytest.fixture(scope="module")
def table(inputs):
    return toy.table(inputs)


def test_k_channel_outlier_ordering(table):
    # "Both K/V quantized", K-channel outlier row: tensor > token > K-channel / V-token
    for target in ("both", "k_only"):
        e = [table[(target, s, "k_col_outlier")] for s in ("tensor", "token", "hybrid")]
        assert e[0] > e[1] > e[2], (target, e)
    # the hybrid isolates the column: several times lower than token grouping
    assert table[("both", "token", "k_col_outlier")] > 3 * table[("both", "hybrid", "k_col_outlier")]


def test_v_only_token_equals_hybrid_bit_for_bit(inputs):
    # their V rules coincide (both per token), so the outputs are identical
    for (Q, K, V) in inputs:
        for cond in toy.CONDITIONS:
            Kc, Vc = toy.conditioned(K, V, cond)
            a = toy.run_case(Q, Kc, Vc, "token", "v_only")[1]
            b = toy.run_case(Q, Kc, Vc, "hybrid", "v_only")[1]
            np.testing.assert_array_equal(a, b)


def test_v_row_outlier_tensor_much_worse_than_token(table):
    for target in ("both", "v_only"):
        assert table[(target, "tensor", "v_row_outlier")] > 5 * table[(target, "token", "v_row_outlier")]


def test_magnitudes_close_to_page(table, golden_dir):
    page = _load_table(os.path.join(golden_dir, "axes_toy_table.txt"))
    for key, want in page.items():
        got = table[key]
        # different random arrays than the page's: magnitudes agree within 2x
        assert want / 2 <= got <= want * 2, (key, got, want)


def test_clean_error_about_one_percent(table):
    for s in toy.SCHEMES:
        assert 0.3 < table[("both", s, "clean")] < 3.0


def test_scale_shapes(inputs):
    Q, K, V = inputs[0]
    N, D = K.shape
    assert toy.quantize_matrix(K, "token")[1].shape == (N, 1)
    assert toy.quantize_matrix(K, "channel")[1].shape == (1, D)
    assert toy.quantize_matrix(K, "tensor")[1].shape == (1, 1)


def test_byte_table(golden_dir):
    D = 32
    for line in open(os.path.join(golden_dir, "axes_bytes_table.txt")):
        if line.startswith("#") or not line.strip():
            continue
        N, f32kv, tens, tok, hyb = map(int, line.split())
        assert 2 * N * D * 4 == f32kv
        for scheme, want in (("tensor", tens), ("token", tok), ("hybrid", hyb)):
            f = formats.Format(**synth.toy_format(scheme, "both", N, D))
            assert formats.payload_bytes(f, 1, 1, N) == want, (scheme, N)
        assert hyb == 2 * N * D + 4 * D + 4 * N
    # "At N=256 it reduces cache-array bytes by 73.24 %"
    assert round(100 * (1 - 17536 / 65536), 2) == 73.24


def test_k4v2_saves_a_quarter_of_k4v4_codes():
    # [K4V2] "Key Contributions": K4V2 uses 25 % less KV memory than K4V4
    f42 = formats.Format(k_bits=4, v_bits=2)
    f44 = formats.Format(k_bits=4, v_bits=4)
    c42 = formats.code_row_bytes(f42, 0) + formats.code_row_bytes(f42, 1)
    c44 = formats.code_row_bytes(f44, 0) + formats.code_row_bytes(f44, 1)
    assert c42 == 0.75 * c44
