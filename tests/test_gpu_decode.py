"""GPU parity of decode attention against the float64 oracle on small seeded caches
of every format, with sinks, residual windows, ragged tails and the degenerate
cases (one token, raw tokens only, a split per group, split-count invariance)."""
import json
import os

import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from oracle import cache as ocache
from oracle import salience
from oracle.formats import BF16, F16, F32, KEYS, MIXED, NUQ, VALUES
from quantized_decode_attention_quantize_b200 import kvq
from tests.gpu_util import assert_attn, Pair, dev, rel_l2, tolerance

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LUT = json.load(open(os.path.join(ROOT, "tests", "golden", "nuq3_codebook.json")))


def fmt(**kw):
    return synth._fmt(**kw)


def vals(seed, shape, dt, scale=1.0, heavy=False):
    r = np.random.default_rng(seed)
    x = r.standard_t(4, shape) if heavy else r.standard_normal(shape)
    return synth.to_dtype_values((x * scale).astype(np.float32), dt)


def build(fd, B, H, Hq, tq, tr, seed=0, k_scale=1.0, luts=(None, None), mixed_q=None):
    D, g, dt = fd["head_dim"], fd["group_tokens"], fd["src_dtype"]
    C = max(g, -(-tq // g) * g)
    p = Pair(fd, B, H, C, k_lut=luts[0], v_lut=luts[1])
    K = vals(seed + 1, (B, H, tq, D), dt, k_scale, heavy=True)
    V = vals(seed + 2, (B, H, tq, D), dt)
    if fd["k_scheme"] == MIXED:
        G = Hq // H
        Q = vals(seed + 3, (B, Hq, tq, D), dt)
        ng = C // g
        order = np.zeros((B, H, ng, D), np.uint8)
        for gi in range(-(-tq // g)):
            for b in range(B):
                for h in range(H):
                    order[b, h, gi] = salience.key_salience(Q[b, h * G:(h + 1) * G, gi * g:(gi + 1) * g],
                                                            K[b, h, gi * g:(gi + 1) * g])[1]
        p.set_order(order)
    if tq:
        p.quantize(KEYS, K, 0, tq)
        p.quantize(VALUES, V, 0, tq)
    if fd["n_sink"]:
        p.set_raw("sink_k", vals(seed + 4, (B, H, fd["n_sink"], D), dt, k_scale))
        p.set_raw("sink_v", vals(seed + 5, (B, H, fd["n_sink"], D), dt))
    if fd["residual_cap"]:
        rk = np.zeros((B, H, fd["residual_cap"], D), np.float32)
        rv = np.zeros_like(rk)
        rk[:, :, :tr] = vals(seed + 6, (B, H, tr, D), dt, k_scale)
        rv[:, :, :tr] = vals(seed + 7, (B, H, tr, D), dt)
        p.set_raw("res_k", rk)
        p.set_raw("res_v", rv)
    return p


def run(p, Hq, tq, tr, q_dtype, out_dtype, seed=0, num_splits=0, q=None):
    D = p.fd["head_dim"]
    if q is None:
        q = vals(seed + 9, (p.B, Hq, D), q_dtype, 1.0)
    out = kvq.decode_attention(p.fmt, p.gpu, dev(q, q_dtype), tq, tr, 1.0 / np.sqrt(D), out_dtype,
                               num_splits=num_splits, status=p.status)
    torch.cuda.synchronize()
    ref = oatt.decode_attention(p.of, p.ora, q.astype(np.float64), tq, tr)
    return out.float().cpu().numpy(), ref


@pytest.mark.parametrize("G", [1, 2, 4, 5, 8])
@pytest.mark.parametrize("out_dtype", [F32, BF16])
def test_k4v2(G, out_dtype):
    B, H, tq = 2, 2, 3 * 128 + 45
    fd = fmt(src_dtype=BF16)
    p = build(fd, B, H, G * H, tq, 0, seed=G)
    out, ref = run(p, G * H, tq, 0, BF16, out_dtype, seed=G)
    assert_attn(out, ref, tolerance(out_dtype), out_dtype)
    assert p.status_bits() == 0


@pytest.mark.parametrize("G", [1, 4])
def test_sink_and_residual(G):
    B, H, tq, tr = 2, 2, 2 * 128 + 17, 37
    fd = fmt(src_dtype=BF16, n_sink=1, residual_cap=128)
    p = build(fd, B, H, G * H, tq, tr, seed=10)
    out, ref = run(p, G * H, tq, tr, BF16, F32, seed=10)
    assert_attn(out, ref, 1e-3)


def test_raw_tokens_only():
    fd = fmt(src_dtype=F16, n_sink=2, residual_cap=16)
    p = build(fd, 1, 2, 8, 0, 9, seed=11)
    out, ref = run(p, 8, 0, 9, F16, F32, seed=11)
    assert_attn(out, ref, 1e-3)


def test_single_token_returns_its_value():
    fd = fmt(src_dtype=F16)
    p = build(fd, 1, 2, 4, 1, 0, seed=12)
    out, ref = run(p, 4, 1, 0, F16, F32, seed=12)
    assert_attn(out, ref, 1e-6)


@pytest.mark.parametrize("splits", [1, 2, 3, 7])
def test_split_count_invariance(splits):
    B, H, G, tq = 1, 2, 4, 7 * 128 - 5
    fd = fmt(src_dtype=BF16)
    p = build(fd, B, H, G * H, tq, 0, seed=13)
    out, ref = run(p, G * H, tq, 0, BF16, F32, seed=13, num_splits=splits)
    assert_attn(out, ref, 1e-3)


@pytest.mark.parametrize("dt", [F16, F32])
@pytest.mark.parametrize("D", [32, 64, 256])
def test_head_dims(dt, D):
    g = 64 if D == 256 else 128
    fd = fmt(head_dim=D, group_tokens=g, src_dtype=dt, k_bits=4, v_bits=2)
    p = build(fd, 1, 2, 4, 2 * g + 3, 0, seed=14)
    out, ref = run(p, 4, 2 * g + 3, 0, dt, F32, seed=14)
    assert_attn(out, ref, 1e-3)


def test_nuq3_outliers_rope():
    fd = fmt(src_dtype=F16, k_scheme=NUQ, k_bits=3, k_outliers=2, v_scheme=NUQ, v_bits=3,
             v_outliers=2, rope=1)
    p = build(fd, 1, 3, 3, 3 * 128 + 20, 0, seed=15, k_scale=3.0, luts=(LUT["k"], LUT["v"]))
    out, ref = run(p, 3, 3 * 128 + 20, 0, F16, F32, seed=15)
    assert_attn(out, ref, 1e-3)


def test_rope_at_long_positions():
    # keys at positions past 100k: the angle t * theta_0 exceeds 1e5 rad
    fd = fmt(src_dtype=F16, rope=1)
    tq = 782 * 128 + 37
    p = build(fd, 1, 1, 2, tq, 0, seed=16)
    out, ref = run(p, 2, tq, 0, F16, F32, seed=16)
    assert_attn(out, ref, 1e-3)


def test_mixed_decode():
    B, H, G = 2, 2, 5
    fd = fmt(src_dtype=BF16, k_scheme=MIXED, k_bits=0, mixed_hi=8, mixed_mid=24)
    p = build(fd, B, H, G * H, 2 * 128 + 60, 0, seed=17, k_scale=4.0)
    out, ref = run(p, G * H, 2 * 128 + 60, 0, BF16, BF16, seed=17)
    assert_attn(out, ref, 2e-3, BF16)


@pytest.mark.parametrize("G", [1, 2, 4, 5, 8])
@pytest.mark.parametrize("splits", [0, 3])
def test_mixed_decode_tensor_core_path(G, splits):
    # the [MIX] Figure 3 tiers on tensor cores: 2-bit and 4-bit slots as fp16 subnormals,
    # raw bf16 slots in their own bf16 product, slot order per group; sink, residual
    # window, a ragged last group
    B, H, tq, tr = 2, 3, 3 * 128 + 45, 29
    fd = fmt(src_dtype=BF16, k_scheme=MIXED, k_bits=0, mixed_hi=8, mixed_mid=24, n_sink=1,
             residual_cap=64)
    p = build(fd, B, H, G * H, tq, tr, seed=110 + G, k_scale=4.0)
    out, ref = run(p, G * H, tq, tr, BF16, F32, seed=110 + G, num_splits=splits)
    assert_attn(out, ref, 1e-3)
    assert p.status_bits() == 0


@pytest.mark.parametrize("kw", [dict(mixed_hi=16, mixed_mid=16), dict(src_dtype=F16)])
def test_mixed_decode_cuda_core_path(kw):
    # tiers other than 8 / 24 / 96, and fp16 sources, take the CUDA-core kernel
    B, H, G, tq = 2, 2, 4, 2 * 128 + 60
    fd = fmt(**dict(dict(src_dtype=BF16, k_scheme=MIXED, k_bits=0, mixed_hi=8, mixed_mid=24), **kw))
    p = build(fd, B, H, G * H, tq, 0, seed=18, k_scale=4.0)
    out, ref = run(p, G * H, tq, 0, fd["src_dtype"], F32, seed=18)
    assert_attn(out, ref, 1e-3)


def test_mixed_decode_heavy_raw_slots():
    # raw slots carrying most of the score: keys x 40 on a few channels of every group
    B, H, G, tq = 1, 2, 4, 2 * 128
    fd = fmt(src_dtype=BF16, k_scheme=MIXED, k_bits=0, mixed_hi=8, mixed_mid=24)
    p = build(fd, B, H, G * H, tq, 0, seed=19, k_scale=40.0)
    out, ref = run(p, G * H, tq, 0, BF16, F32, seed=19)
    assert_attn(out, ref, 1e-3)


@pytest.mark.parametrize("scheme", ["tensor", "token", "hybrid"])
@pytest.mark.parametrize("target", ["both", "k_only", "v_only"])
def test_toy_int8(scheme, target):
    # [AXES] toy as decode: 8 query rows are 8 query heads sharing one KV head
    N = 64
    Q, K, V = synth.toy(41, N)
    fd = synth.toy_format(scheme, target, N)
    p = Pair(fd, 1, 1, N)
    p.quantize(KEYS, K[None, None], 0, N)
    p.quantize(VALUES, V[None, None], 0, N)
    out, ref = run(p, 8, N, 0, F32, F32, q=Q[None])
    assert_attn(out, ref, 1e-5)


def test_nonfinite_query_flagged():
    fd = fmt(src_dtype=F16)
    p = build(fd, 1, 1, 2, 128, 0, seed=18)
    q = vals(19, (1, 2, 128), F16)
    q[0, 1, 5] = np.inf
    kvq.decode_attention(p.fmt, p.gpu, dev(q, F16), 128, 0, 0.1, F32, status=p.status)
    assert p.status_bits() & kvq.KVQ_DEV_NONFINITE


@pytest.mark.parametrize("B,H,G,tq,ns,tr,splits,src", [
    (3, 5, 2, 2 * 128 + 1, 2, 3, 0, BF16),
    (3, 5, 2, 2 * 128 + 1, 2, 3, 1, BF16),
    (3, 5, 2, 2 * 128 + 1, 2, 3, 13, BF16),
    (2, 3, 8, 5, 1, 0, 4, BF16),
    (1, 7, 4, 9 * 128, 0, 100, 0, BF16),
    (4, 2, 3, 3 * 128 - 7, 4, 11, 2, BF16),
    (2, 3, 4, 64, 1, 13, 0, BF16),          # one half group, two raw items
    (2, 3, 4, 65, 1, 13, 3, BF16),          # a second half with one token
    (5, 3, 2, 7 * 128 + 64, 1, 100, 1, BF16),   # fifteen heads, one CTA asked: two
    (2, 2, 4, 300, 1, 20, 0, F32),          # fp32 raw items of six tokens
    (2, 2, 6, 5 * 128 + 3, 3, 0, 2, F16),
    (16, 120, 2, 70, 1, 3, 0, BF16),        # more heads than warps on the GPU
])
def test_partition_shapes(B, H, G, tq, ns, tr, splits, src):
    # the item partition: raw items and half groups cut into equal warp ranges, heads
    # spanning several CTAs, CTAs spanning several heads, ranges that cross heads,
    # tiny and ragged regions, more CTAs than SMs
    fd = fmt(src_dtype=src, n_sink=ns, residual_cap=128)
    p = build(fd, B, H, G * H, tq, tr, seed=40 + tq)
    out, ref = run(p, G * H, tq, tr, src, F32, seed=40 + tq, num_splits=splits)
    assert_attn(out, ref, 1e-3)
    assert p.status_bits() == 0


@pytest.mark.parametrize("B,H,G,tq,ns,tr,splits", [
    (8, 8, 4, 32 * 128 - 1, 1, 128, 0),
    (3, 5, 2, 2 * 128 + 1, 2, 3, 13),
    (5, 3, 8, 7 * 128 + 64, 1, 100, 1),
])
def test_decode_attention_matches_partial_then_combine(B, H, G, tq, ns, tr, splits):
    # the one-call entry point and the separate partial + combine calls give the same bits
    fd = fmt(src_dtype=BF16, n_sink=ns, residual_cap=128)
    p = build(fd, B, H, G * H, tq, tr, seed=90 + G)
    q = dev(vals(91, (B, G * H, 128), BF16), BF16)
    scale = 1.0 / np.sqrt(128.0)
    one = kvq.decode_attention(p.fmt, p.gpu, q, tq, tr, scale, F32, num_splits=splits, status=p.status)
    ws = torch.empty(kvq.decode_workspace_bytes(p.fmt, B, G * H, H, tq, tr, splits), dtype=torch.uint8,
                     device="cuda")
    kvq.decode_partial(p.fmt, p.gpu, q, tq, tr, scale, ws, num_splits=splits, status=p.status)
    two = torch.empty_like(one)
    kvq.decode_combine(p.fmt, B, G * H, H, tq, tr, ws, two, num_splits=splits)
    torch.cuda.synchronize()
    assert torch.equal(one, two)
    ref = oatt.decode_attention(p.of, p.ora, q.float().cpu().numpy().astype(np.float64), tq, tr)
    assert_attn(one.cpu().numpy(), ref, 1e-3)
    assert p.status_bits() == 0


def clone_cache(p, luts=(None, None)):
    c = kvq.Cache(p.fmt, p.B, p.H, p.C, k_lut=luts[0], v_lut=luts[1])
    for name, t in p.gpu.tensors.items():
        c.tensors[name].copy_(t)
    return c


@pytest.mark.parametrize("kw,G,t0,n", [
    (dict(), 4, 7 * 128, 128),                      # the split kernel appends the group itself
    (dict(), 4, 7 * 128, 37),                       # a partial group, appended the same way
    (dict(), 2, 3 * 128, 128),                      # a group inside the decoded rows (fused)
    (dict(), 1, 0, 5),                              # the first rows of the first group (fused)
    (dict(), 2, 3 * 128, 256),                      # two groups: append launch, deferred wait
    (dict(k_rotate=1), 4, 7 * 128, 128),            # rotated keys: a plain append launch
    (dict(), 8, 7 * 128, 128),                      # G = 8: the general tensor-core kernel
    (dict(), 4, 7 * 128, 0),                        # nothing appended
    (dict(k_scheme=NUQ, k_bits=3, v_scheme=NUQ, v_bits=3, v_axis=1, k_outliers=2, v_outliers=2), 4, 7 * 128, 128),
])
def test_append_decode_matches_separate_calls(kw, G, t0, n):
    # kvq_append_decode_attention == kvq_quantize_kv then kvq_decode_attention, bit for bit,
    # cache bytes included; and the result is the oracle's attention over the updated cache
    fd = fmt(src_dtype=BF16, n_sink=1, residual_cap=128, **kw)
    luts = (LUT["k"], LUT["v"]) if fd["k_scheme"] == NUQ else (None, None)
    B, H, tq, tr = 2, 3, 8 * 128 - 5, 20
    p = build(fd, B, H, G * H, tq, tr, seed=300 + G + n, luts=luts)
    other = clone_cache(p, luts)
    Kn = vals(301, (B, H, max(n, 1), 128), BF16, heavy=True)[:, :, :n]
    Vn = vals(302, (B, H, max(n, 1), 128), BF16)[:, :, :n]
    q = dev(vals(303, (B, G * H, 128), BF16), BF16)
    scale = 1.0 / np.sqrt(128.0)
    kd, vd = dev(Kn, BF16), dev(Vn, BF16)
    one = kvq.append_decode_attention(p.fmt, p.gpu, kd, vd, t0, n, q, tq, tr, scale, F32, status=p.status)
    if n:
        kvq.quantize_kv(p.fmt, other, kd, vd, t0, n, status=p.status)
    two = kvq.decode_attention(p.fmt, other, q, tq, tr, scale, F32, status=p.status)
    torch.cuda.synchronize()
    assert torch.equal(one, two)
    for name, t in p.gpu.tensors.items():
        assert torch.equal(t, other.tensors[name]), name
    if n:
        ocache.quantize(p.of, p.ora, KEYS, Kn.astype(np.float64), t0, n)
        ocache.quantize(p.of, p.ora, VALUES, Vn.astype(np.float64), t0, n)
    ref = oatt.decode_attention(p.of, p.ora, q.float().cpu().numpy().astype(np.float64), tq, tr)
    assert_attn(one.cpu().numpy(), ref, 1e-3)
    assert p.status_bits() == 0
