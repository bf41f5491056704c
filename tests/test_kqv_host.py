"""Host-side KQV entry points (no GPU): the Lloyd-Max codebook of kvq_kqv_codebook
against closed forms and the oracle's codebooks, the array sizes of the stored format,
and the format checks."""
import json
import math
import os

import numpy as np
import pytest

import synth
from quantized_decode_attention_quantize_b200 import kvq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kqv_codebooks.json")


def kqv_fmt(kb=4, vb=4, **kw):
    return kvq.make_format(synth._fmt(k_scheme=synth.KQV, k_bits=kb, k_axis=synth.TOKEN,
                                      v_scheme=synth.KQV, v_bits=vb, v_axis=synth.TOKEN, **kw))


def test_codebook_uniform_at_d3():
    # d = 3: the coordinate marginal is uniform on [-1, 1]; Lloyd-Max is the uniform quantizer
    for b in (1, 2, 3):
        K = 1 << b
        want = [(2 * k + 1) / K - 1 for k in range(K)]
        np.testing.assert_allclose(kvq.kqv_codebook(b, 3), want, atol=2e-5)


def test_codebook_one_bit_closed_form():
    # one bit: the centroids are -+E|x| = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    for d in (4, 16, 128, 1024):
        e = math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
        np.testing.assert_allclose(kvq.kqv_codebook(1, d), [-e, e], rtol=1e-6)


def test_codebook_matches_the_oracle():
    with open(GOLDEN) as f:
        gold = json.load(f)["f64"]
    for b in (1, 2, 3, 4):
        got = np.asarray(kvq.kqv_codebook(b, 128), np.float64)
        want = np.asarray(gold[str(b)], np.float64)
        np.testing.assert_allclose(got, want, rtol=1e-6, atol=0)
        assert np.all(np.diff(got) > 0)
        np.testing.assert_array_equal(got, -got[::-1])


def test_codebook_rejects_bad_arguments():
    L = kvq.lib()
    import ctypes
    buf = (ctypes.c_float * 16)()
    assert L.kvq_kqv_codebook(0, 128, buf) == kvq.KVQ_ERR_INVALID
    assert L.kvq_kqv_codebook(5, 128, buf) == kvq.KVQ_ERR_INVALID
    assert L.kvq_kqv_codebook(2, 2, buf) == kvq.KVQ_ERR_INVALID
    assert L.kvq_kqv_codebook(2, 128, None) == kvq.KVQ_ERR_INVALID


@pytest.mark.parametrize("kb,vb", [(4, 4), (3, 3), (2, 2), (4, 3)])
def test_array_sizes(kb, vb):
    f = kqv_fmt(kb, vb)
    B, H, C, D = 2, 3, 256, 128
    sz = {name: kvq.cache_array_bytes(f, B, H, C, i) for i, name in enumerate(kvq.ARRAYS)}
    assert sz["k_codes"] == B * H * C * kb * D // 8
    assert sz["v_codes"] == B * H * C * vb * D // 8     # vb - 1 code bits and the sketch bit
    assert sz["k_scale"] == sz["v_scale"] == sz["v_zero"] == B * H * C * 4
    assert sz["k_zero"] == 0
    assert sz["k_lut"] == 4 << kb and sz["v_lut"] == 4 << (vb - 1)
    assert sz["v_sketch"] == D * D * 4
    for name in ("k_order", "k_out_rowptr", "k_out_col", "k_out_val", "v_out_col", "v_out_val"):
        assert sz[name] == 0


def test_format_checks():
    assert kvq.format_check(kqv_fmt()) == kvq.KVQ_OK
    assert kvq.format_check(kqv_fmt(5, 4)) == kvq.KVQ_ERR_INVALID
    assert kvq.format_check(kqv_fmt(4, 1)) == kvq.KVQ_ERR_INVALID
    assert kvq.format_check(kqv_fmt(head_dim=64)) == kvq.KVQ_ERR_UNSUPPORTED
    assert kvq.format_check(kqv_fmt(rope=1)) == kvq.KVQ_ERR_UNSUPPORTED
    assert kvq.format_check(kqv_fmt(k_rotate=1)) == kvq.KVQ_ERR_UNSUPPORTED
    one_sided = kvq.make_format(synth._fmt(k_scheme=synth.KQV, k_bits=4, k_axis=synth.TOKEN))
    assert kvq.format_check(one_sided) == kvq.KVQ_ERR_UNSUPPORTED
    chan = kvq.make_format(synth._fmt(k_scheme=synth.KQV, k_bits=4, k_axis=synth.CHANNEL,
                                      v_scheme=synth.KQV, v_bits=4, v_axis=synth.TOKEN))
    assert kvq.format_check(chan) == kvq.KVQ_ERR_UNSUPPORTED


def test_decode_rejects_wide_groups():
    # the KQV decode takes up to 8 query heads per KV head
    f = kqv_fmt()
    assert kvq.decode_workspace_bytes(f, 1, 16, 1, 256, 0) == 0
    assert kvq.decode_workspace_bytes(f, 1, 8, 1, 256, 0) > 0
