"""GPU parity of quantize, dequantize and salience: every cache array byte for byte
against the oracle, on seeded inputs that span several groups and a ragged tail."""
import json
import os

import numpy as np
import pytest
import torch

import synth
from oracle import fp, salience
from oracle.cache import dequantize as odeq
from oracle.formats import (ASYM, BF16, CHANNEL, F16, F32, KEYS, MIXED, NONE, NUQ, SYM8,
                            TENSOR, TOKEN, VALUES)
from quantized_decode_attention_quantize_b200 import kvq
from oracle import cache as ocache
from tests.gpu_util import Pair, dev

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LUT = json.load(open(os.path.join(ROOT, "tests", "golden", "nuq3_codebook.json")))


def fmt(**kw):
    return synth._fmt(**kw)


def values(seed, shape, dtype, scale=1.0, outlier_cols=0):
    r = np.random.default_rng(seed)
    x = r.standard_normal(shape).astype(np.float32) * np.float32(scale)
    x += np.float32(r.uniform(-2, 2))
    if outlier_cols:
        cols = r.choice(shape[-1], outlier_cols, replace=False)
        x[..., cols] *= np.float32(20)
    return synth.to_dtype_values(x, dtype)


def deq_check(p, which, t0, n):
    for od in (F32, F16, BF16):
        got = kvq.dequantize(p.fmt, p.gpu, which, t0, n, od).float().cpu().numpy()
        want = odeq(p.of, p.ora, which, t0, n)
        if od == F16:
            want = fp.f16(want)
        elif od == BF16:
            want = fp.bf16(want)
        np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("dt", [F16, BF16, F32])
@pytest.mark.parametrize("kb,vb", [(4, 2), (2, 4), (8, 8), (4, 4), (2, 2)])
def test_asym(dt, kb, vb):
    B, H, D, g, n = 2, 3, 128, 128, 3 * 128 + 77
    p = Pair(fmt(head_dim=D, group_tokens=g, src_dtype=dt, k_bits=kb, v_bits=vb), B, H, 4 * g)
    K = values(1, (B, H, n, D), dt, 2.0, outlier_cols=4)
    V = values(2, (B, H, n, D), dt)
    p.quantize(KEYS, K, 0, n, strided=True)
    p.quantize(VALUES, V, 0, n)
    p.assert_arrays_equal()
    assert p.status_bits() == 0
    deq_check(p, KEYS, 0, n)
    deq_check(p, VALUES, 0, n)
    deq_check(p, VALUES, 37, 101)       # odd start inside a token pair


@pytest.mark.parametrize("D,g", [(32, 16), (64, 48), (256, 128)])
def test_asym_shapes(D, g):
    B, H, n = 1, 2, 5 * g - 3
    p = Pair(fmt(head_dim=D, group_tokens=g, src_dtype=F16), B, H, 5 * g)
    p.quantize(KEYS, values(3, (B, H, n, D), F16, 3.0), 0, n)
    p.quantize(VALUES, values(4, (B, H, n, D), F16), 0, n)
    p.assert_arrays_equal()
    deq_check(p, KEYS, 0, n)
    deq_check(p, VALUES, 0, n)


def test_appends_and_partial_group_rewrite():
    B, H, D, g = 1, 2, 128, 128
    p = Pair(fmt(), B, H, 4 * g)
    K = values(5, (B, H, 4 * g, D), F16, 2.0)
    V = values(6, (B, H, 4 * g, D), F16)
    p.quantize(KEYS, K[:, :, :g + 5], 0, g + 5)          # one group + a 5-token partial group
    p.quantize(VALUES, V[:, :, :g + 5], 0, g + 5)
    p.assert_arrays_equal()
    p.quantize(KEYS, K[:, :, g:3 * g], g, 2 * g)          # rewrite it whole and append one more
    p.quantize(VALUES, V[:, :, g:3 * g], g, 2 * g)
    p.assert_arrays_equal()


@pytest.mark.parametrize("scheme", ["tensor", "token", "hybrid"])
@pytest.mark.parametrize("target", ["both", "k_only", "v_only"])
@pytest.mark.parametrize("N", [64, 256])
def test_sym8_toy(scheme, target, N):
    Q, K, V = synth.toy(7, N)
    Kc, Vc = K.copy(), V.copy()
    Kc[:, 0] *= np.float32(40)
    p = Pair(synth.toy_format(scheme, target, N), 1, 1, N)
    p.quantize(KEYS, Kc[None, None], 0, N)
    p.quantize(VALUES, Vc[None, None], 0, N)
    p.assert_arrays_equal()
    deq_check(p, KEYS, 0, N)
    deq_check(p, VALUES, 0, N)


def test_sym8_zero_group_and_ties():
    N, D = 64, 32
    K = np.zeros((1, 1, N, D), np.float32)
    K[0, 0, 5] = np.arange(D, dtype=np.float32) + 0.5   # scale 1 would make .5 ties
    K[0, 0, 5, 0] = 127.0
    p = Pair(synth.toy_format("token", "both", N), 1, 1, N)
    p.quantize(KEYS, K, 0, N)
    p.quantize(VALUES, np.zeros_like(K), 0, N)
    p.assert_arrays_equal()


@pytest.mark.parametrize("nout", [0, 2, 3])
@pytest.mark.parametrize("dt", [F16, BF16])
def test_nuq3_outliers(nout, dt):
    B, H, D, g, n = 1, 3, 128, 128, 2 * 128 + 50
    f = fmt(src_dtype=dt, k_scheme=NUQ, k_bits=3, k_outliers=nout, v_scheme=NUQ, v_bits=3,
            v_outliers=nout)
    p = Pair(f, B, H, 3 * g, k_lut=LUT["k"], v_lut=LUT["v"])
    K = values(7, (B, H, n, D), dt, 1.0) * np.exp(np.random.default_rng(8).uniform(-2, 2, D)).astype(np.float32)
    K = synth.to_dtype_values(K, dt)
    V = values(9, (B, H, n, D), dt)
    # plant exact magnitude ties to exercise the lower-index rule
    K[0, 0, 3, 7] = 50.0
    K[0, 0, 9, 7] = -50.0
    V[0, 1, 4, 10] = 9.0
    V[0, 1, 4, 20] = -9.0
    V[0, 1, 4, 30] = 9.0
    p.quantize(KEYS, K, 0, n)
    p.quantize(VALUES, V, 0, n)
    p.assert_arrays_equal()
    deq_check(p, KEYS, 0, n)
    deq_check(p, VALUES, 0, n)


def test_mixed_with_salience():
    B, Hq, H, D, g = 2, 10, 2, 128, 128
    G = Hq // H
    n = 2 * g + 31
    f = fmt(src_dtype=BF16, k_scheme=MIXED, k_bits=0, mixed_hi=8, mixed_mid=24)
    p = Pair(f, B, H, 3 * g)
    r = np.random.default_rng(10)
    K = (r.standard_normal((B, H, n, D)) * np.exp(r.uniform(np.log(0.1), np.log(20), (1, H, 1, D))))
    K = synth.to_dtype_values(K.astype(np.float32), BF16)
    Q = (r.standard_normal((B, Hq, n, D)) * np.exp(r.uniform(np.log(0.1), np.log(5), (1, Hq, 1, D))))
    Q = synth.to_dtype_values(Q.astype(np.float32), BF16)
    ng = 3
    order_dev = p.gpu.array("k_order")
    sal = torch.zeros((B, H, D), dtype=torch.float64, device="cuda")
    orders = np.zeros((B, H, ng, D), np.uint8)
    for gi in range(3):
        t0, ln = gi * g, min(g, n - gi * g)
        qd = torch.tensor(Q[:, :, t0:t0 + ln], device="cuda").to(torch.bfloat16)
        kd = torch.tensor(K[:, :, t0:t0 + ln], device="cuda").to(torch.bfloat16)
        kvq.key_salience(p.fmt, qd, kd, order_dev[gi * D:], H * ng * D, ng * D, salience_out=sal)
        torch.cuda.synchronize()
        for b in range(B):
            for h in range(H):
                A, order = salience.key_salience(Q[b, h * G:(h + 1) * G, t0:t0 + ln], K[b, h, t0:t0 + ln])
                orders[b, h, gi] = order
                np.testing.assert_array_equal(sal[b, h].cpu().numpy(), A)   # bit-exact fp64
    p.ora["k_order"][...] = orders
    p.assert_arrays_equal(["k_order"])
    p.quantize(KEYS, K, 0, n)
    p.quantize(VALUES, values(11, (B, H, n, D), BF16), 0, n)
    p.assert_arrays_equal()
    deq_check(p, KEYS, 0, n)


def test_salience_ties_and_full_window():
    B, Hq, H, D, R = 1, 4, 1, 128, 128
    f = fmt(src_dtype=F16)
    fm = kvq.make_format(f)
    Q = np.ones((B, Hq, R, D), np.float32)
    K = np.zeros((B, H, R, D), np.float32)
    K[0, 0, 1, :] = (np.arange(D) % 5).astype(np.float32)     # many equal ranges
    order = torch.zeros(D, dtype=torch.uint8, device="cuda")
    kvq.key_salience(fm, torch.tensor(Q, device="cuda").half(), torch.tensor(K, device="cuda").half(),
                     order, 0, 0)
    _, want = salience.key_salience(Q[0], K[0, 0])
    np.testing.assert_array_equal(order.cpu().numpy(), want)


def test_status_flags():
    B, H, D, g = 1, 1, 128, 128
    p = Pair(fmt(src_dtype=F32), B, H, g)
    K = values(12, (B, H, g, D), F32)
    K[0, 0, 3, 3] = np.nan
    t = torch.tensor(K, device="cuda")
    kvq.quantize_keys(p.fmt, p.gpu, t, 0, g, status=p.status)
    assert p.status_bits() & kvq.KVQ_DEV_NONFINITE
    p.status.zero_()
    K2 = values(13, (B, H, g, D), F32)
    K2[0, 0, :, 5] = np.float32(-1e6)   # zero-point beyond fp16
    kvq.quantize_keys(p.fmt, p.gpu, torch.tensor(K2, device="cuda"), 0, g, status=p.status)
    assert p.status_bits() & kvq.KVQ_DEV_RANGE


def test_none_scheme_copies_raw():
    N = 64
    Q, K, V = synth.toy(19, N)
    p = Pair(synth.toy_format("token", "v_only", N), 1, 1, N)
    p.quantize(KEYS, K[None, None], 0, N)
    p.quantize(VALUES, V[None, None], 0, N)
    p.assert_arrays_equal()


@pytest.mark.parametrize("fd", [
    dict(src_dtype=BF16),                                              # K4/V2: one fused launch
    dict(src_dtype=F16, k_bits=2, v_bits=4),
    dict(src_dtype=BF16, k_scheme=NUQ, k_bits=3, k_outliers=2, v_scheme=NUQ, v_bits=3, v_outliers=2),
    dict(src_dtype=BF16, k_rotate=1),                                  # rotated keys: fused launch
    dict(src_dtype=F32, k_bits=8, k_rotate=1),
])
def test_quantize_kv_matches_separate_calls_and_oracle(fd):
    # kvq_quantize_kv = kvq_quantize_keys then kvq_quantize_values, bit for bit
    B, H, D, g = 2, 3, 128, 128
    n = 2 * g + 40
    f = fmt(**fd)
    luts = (LUT["k"], LUT["v"]) if fd.get("k_scheme") == NUQ else (None, None)
    p = Pair(f, B, H, 3 * g, k_lut=luts[0], v_lut=luts[1])
    K = values(21, (B, H, n, D), fd["src_dtype"])
    V = values(22, (B, H, n, D), fd["src_dtype"])
    kd, vd = dev(K, fd["src_dtype"]), dev(V, fd["src_dtype"])
    kvq.quantize_kv(p.fmt, p.gpu, kd, vd, 0, n, status=p.status)
    ocache.quantize(p.of, p.ora, KEYS, K.astype(np.float64), 0, n)
    ocache.quantize(p.of, p.ora, VALUES, V.astype(np.float64), 0, n)
    p.assert_arrays_equal()
    assert p.status_bits() == 0
    other = kvq.Cache(p.fmt, B, H, 3 * g, k_lut=luts[0], v_lut=luts[1])
    kvq.quantize_keys(p.fmt, other, kd, 0, n)
    kvq.quantize_values(p.fmt, other, vd, 0, n)
    torch.cuda.synchronize()
    for name, t in other.tensors.items():
        assert torch.equal(t, p.gpu.array(name)), name
