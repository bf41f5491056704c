"""GPU parity of key-only Walsh-Hadamard rotation ([K4V2] "Rotation Integration"; [TQ]
KQV scheme): the rotated cache byte for byte against the oracle, its dequantized keys
bit for bit (back in the original basis), and decode attention -- which rotates the
query instead of the keys -- on each decode path (tensor-core K4V2, CUDA-core nuq3,
generic) within the attention tolerance, over raw sinks and residual windows that stay
unrotated."""
import json
import os

import numpy as np
import pytest

import synth
from oracle.formats import ASYM, BF16, CHANNEL, F16, F32, KEYS, NUQ, SYM8, TENSOR, TOKEN, VALUES
from tests.gpu_util import assert_attn, Pair, rel_l2, tolerance
from tests.test_gpu_decode import build, run
from tests.test_gpu_quantize import deq_check, values

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LUT = json.load(open(os.path.join(ROOT, "tests", "golden", "nuq3_codebook.json")))


@pytest.mark.parametrize("dt", [F16, BF16, F32])
@pytest.mark.parametrize("kw", [
    dict(k_scheme=ASYM, k_bits=4),
    dict(k_scheme=ASYM, k_bits=2),
    dict(k_scheme=ASYM, k_bits=8),
    dict(k_scheme=SYM8, k_bits=8, k_axis=TOKEN),
    dict(k_scheme=SYM8, k_bits=8, k_axis=CHANNEL),
    dict(k_scheme=SYM8, k_bits=8, k_axis=TENSOR),
])
def test_rotated_keys_quantize_and_dequantize(dt, kw):
    B, H, D, g, n = 2, 3, 128, 128, 3 * 128 + 77
    p = Pair(synth._fmt(head_dim=D, group_tokens=g, src_dtype=dt, k_rotate=1, **kw), B, H, 4 * g)
    p.quantize(KEYS, values(1, (B, H, n, D), dt, 2.0, outlier_cols=4), 0, n, strided=True)
    p.quantize(VALUES, values(2, (B, H, n, D), dt), 0, n)
    p.assert_arrays_equal()
    assert p.status_bits() == 0
    deq_check(p, KEYS, 0, n)
    deq_check(p, KEYS, 131, 77)
    deq_check(p, VALUES, 0, n)


@pytest.mark.parametrize("g,kb", [(16, 4), (64, 2), (112, 8)])
def test_rotated_keys_group_sizes_and_partial_rewrite(g, kb):
    # the whole-group register kernel at g < 128, a partial last group, then its rewrite
    B, H, D = 2, 2, 128
    p = Pair(synth._fmt(head_dim=D, group_tokens=g, src_dtype=BF16, k_bits=kb, k_rotate=1), B, H, 4 * g)
    K = values(7, (B, H, 4 * g, D), BF16, 2.0, outlier_cols=3)
    p.quantize(KEYS, K[:, :, :g + 5], 0, g + 5)
    p.assert_arrays_equal()
    p.quantize(KEYS, K[:, :, g:3 * g + 1], g, 2 * g + 1)
    p.assert_arrays_equal()
    deq_check(p, KEYS, 0, 3 * g + 1)


@pytest.mark.parametrize("D,g", [(32, 16), (64, 48), (256, 128)])
def test_rotated_keys_other_head_dims(D, g):
    B, H, n = 1, 2, 5 * g - 3
    p = Pair(synth._fmt(head_dim=D, group_tokens=g, src_dtype=F16, k_rotate=1), B, H, 5 * g)
    p.quantize(KEYS, values(3, (B, H, n, D), F16, 3.0, outlier_cols=2), 0, n)
    p.quantize(VALUES, values(4, (B, H, n, D), F16), 0, n)
    p.assert_arrays_equal()
    deq_check(p, KEYS, 0, n)


@pytest.mark.parametrize("nout", [0, 2])
def test_rotated_nuq3_keys_with_outliers(nout):
    B, H, D, g, n = 2, 2, 128, 128, 2 * 128 + 50
    fd = synth._fmt(src_dtype=F16, k_scheme=NUQ, k_bits=3, k_outliers=nout, v_scheme=NUQ,
                    v_bits=3, v_outliers=nout, k_rotate=1)
    p = Pair(fd, B, H, 3 * g, k_lut=LUT["k"], v_lut=LUT["v"])
    p.quantize(KEYS, values(5, (B, H, n, D), F16, 1.5, outlier_cols=3), 0, n)
    p.quantize(VALUES, values(6, (B, H, n, D), F16), 0, n)
    p.assert_arrays_equal()
    assert p.status_bits() == 0
    deq_check(p, KEYS, 0, n)


@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("splits", [0, 3])
def test_rotated_k4v2_decode_tensor_core_path(G, splits):
    B, H, tq, tr = 2, 3, 3 * 128 + 45, 37
    fd = synth._fmt(src_dtype=BF16, n_sink=1, residual_cap=128, k_rotate=1)
    p = build(fd, B, H, G * H, tq, tr, seed=70 + G)
    out, ref = run(p, G * H, tq, tr, BF16, F32, seed=70 + G, num_splits=splits)
    assert_attn(out, ref, tolerance(F32))
    assert p.status_bits() == 0


@pytest.mark.parametrize("B,H,G,tq,ns,tr,splits", [
    (2, 3, 4, 2 * 128 + 40, 1, 21, 0),      # ranges that cross heads and raw -> packed
    (16, 120, 2, 70, 1, 3, 0),              # more heads than warps
    (5, 3, 2, 7 * 128 + 64, 1, 100, 1),
])
def test_rotated_partition_shapes(B, H, G, tq, ns, tr, splits):
    fd = synth._fmt(src_dtype=BF16, n_sink=ns, residual_cap=128, k_rotate=1)
    p = build(fd, B, H, G * H, tq, tr, seed=80 + tq)
    out, ref = run(p, G * H, tq, tr, BF16, F32, seed=80 + tq, num_splits=splits)
    assert_attn(out, ref, 1e-3)


@pytest.mark.parametrize("G", [1, 4])
def test_rotated_nuq3_decode_cuda_core_path(G):
    B, H, tq, tr = 1, 2, 2 * 128 + 33, 20
    fd = synth._fmt(src_dtype=F16, k_scheme=NUQ, k_bits=3, k_outliers=2, v_scheme=NUQ, v_bits=3,
                    v_outliers=2, n_sink=1, residual_cap=32, k_rotate=1)
    p = build(fd, B, H, G * H, tq, tr, seed=60 + G, luts=(LUT["k"], LUT["v"]))
    out, ref = run(p, G * H, tq, tr, F16, F32, seed=60 + G)
    assert_attn(out, ref, 1e-3)


@pytest.mark.parametrize("kw", [
    dict(k_scheme=SYM8, k_bits=8, k_axis=TOKEN),     # generic path, D = 128
    dict(head_dim=64, group_tokens=64),              # generic path, K4V2 at D = 64
    dict(head_dim=256, group_tokens=64),
])
def test_rotated_decode_generic_path(kw):
    B, H, G, tq, tr = 2, 2, 2, 2 * 64 + 29, 5
    fd = synth._fmt(src_dtype=BF16, n_sink=1, residual_cap=16, k_rotate=1, **kw)
    p = build(fd, B, H, G * H, tq, tr, seed=50)
    out, ref = run(p, G * H, tq, tr, BF16, F32, seed=50)
    assert_attn(out, ref, 1e-3)
