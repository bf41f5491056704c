"""GPU parity of the KQV scheme ([TQ] "Quantization Schemes") against oracle.kqv's stored
format: every packed code word, sketch word and fp32 norm bit for bit; dequantized rows
within fp32 rounding of the real-valued reconstruction; decode attention within a bar
derived from fp32 accumulation against float64 attention over the reconstructed rows.

The centroids are the oracle's Lloyd-Max codebooks (tests/golden/kqv_codebooks.json,
written by a script that calls only the oracle) rounded to fp32; the sketch matrix is a
seeded N(0, 1) draw passed to both sides."""
import json
import os

import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from oracle import kqv as okqv
from oracle import pack as opack
from oracle.formats import BF16, F16, F32, KEYS, VALUES
from quantized_decode_attention_quantize_b200 import kvq
from tests.gpu_util import assert_attn, dev, raw_bits, tolerance

pytestmark = pytest.mark.gpu
D = 128
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kqv_codebooks.json")


def codebook(bits):
    with open(GOLDEN) as f:
        return np.asarray(json.load(f)["f64"][str(bits)], np.float64).astype(np.float32)


def kqv_fmt(kb=4, vb=4, **kw):
    return synth._fmt(k_scheme=synth.KQV, k_bits=kb, k_axis=synth.TOKEN,
                      v_scheme=synth.KQV, v_bits=vb, v_axis=synth.TOKEN, **kw)


def vals(rng, shape, dt, heavy=False, outlier_cols=()):
    x = rng.standard_t(4, shape) if heavy else rng.standard_normal(shape)
    x[..., list(outlier_cols)] *= 10.0
    return synth.to_dtype_values(x.astype(np.float32), dt)


class KqvPair:
    """A KQV cache on the device and the oracle's stored arrays for the same rows."""

    def __init__(self, fd, B, H, C, seed):
        self.fd, self.B, self.H, self.C = fd, B, H, C
        self.kb, self.vb = fd["k_bits"], fd["v_bits"] - 1
        self.ck, self.cv = codebook(self.kb), codebook(self.vb)
        rng = np.random.default_rng(seed)
        self.S = rng.standard_normal((D, D)).astype(np.float32)
        self.fmt = kvq.make_format(fd)
        self.gpu = kvq.Cache(self.fmt, B, H, C, k_lut=self.ck, v_lut=self.cv, sketch=self.S)
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.K = np.zeros((B, H, C, D), np.float32)
        self.V = np.zeros((B, H, C, D), np.float32)

    def append(self, K, V, t0):
        n = K.shape[2]
        dt = self.fd["src_dtype"]
        kvq.quantize_kv(self.fmt, self.gpu, dev(K, dt), dev(V, dt), t0, n, status=self.status)
        self.K[:, :, t0:t0 + n] = K
        self.V[:, :, t0:t0 + n] = V

    def oracle_rows(self, t):
        """Stored key / value arrays of rows [0, t) from the oracle."""
        K = self.K[:, :, :t].reshape(-1, D)
        V = self.V[:, :, :t].reshape(-1, D)
        kc, kn = okqv.stored_encode(K, self.ck)
        parts = [okqv.stored_encode(V[i:i + 512], self.cv, self.S) for i in range(0, len(V), 512)]
        vc, vn, sg, rn = (np.concatenate([x[j] for x in parts]) for j in range(4))
        return kc, kn, vc, vn, sg, rn

    def packed_codes(self, codes, b):
        return opack.pack_3bit(codes) if b == 3 else opack.pack_row(codes, b)

    def check_arrays(self, t):
        torch.cuda.synchronize()
        assert int(self.status.item()) == 0
        kc, kn, vc, vn, sg, rn = self.oracle_rows(t)
        B, H, C = self.B, self.H, self.C
        kw = self.kb * D // 32
        vw = (self.vb + 1) * D // 32
        got_k = self.gpu.array("k_codes").view(torch.int32).view(B, H, C, kw)[:, :, :t].cpu().numpy().view(np.uint32)
        want_k = self.packed_codes(kc, self.kb).reshape(B, H, t, kw)
        np.testing.assert_array_equal(got_k, want_k)
        got_v = self.gpu.array("v_codes").view(torch.int32).view(B, H, C, vw)[:, :, :t].cpu().numpy().view(np.uint32)
        want_v = np.concatenate([self.packed_codes(vc, self.vb), opack.pack_row(sg.astype(np.int64), 1)],
                                axis=-1).reshape(B, H, t, vw)
        np.testing.assert_array_equal(got_v, want_v)
        for name, want in (("k_scale", kn), ("v_scale", vn), ("v_zero", rn)):
            got = self.gpu.array(name).view(torch.float32).view(B, H, C)[:, :, :t].cpu().numpy()
            np.testing.assert_array_equal(got.view(np.uint32), want.reshape(B, H, t).view(np.uint32))

    def reconstructed(self, t):
        kc, kn, vc, vn, sg, rn = self.oracle_rows(t)
        Kh = okqv.stored_key(kc, kn, self.ck).reshape(self.B, self.H, t, D)
        Vh = okqv.stored_value(vc, vn, sg, rn, self.cv, self.S).reshape(self.B, self.H, t, D)
        return Kh, Vh


@pytest.mark.parametrize("kb,vb,dt", [(4, 4, BF16), (3, 3, F16), (2, 2, F32), (4, 3, BF16), (3, 4, F16)])
def test_quantize_bit_exact(kb, vb, dt):
    fd = kqv_fmt(kb, vb, src_dtype=dt)
    p = KqvPair(fd, 2, 3, 384, seed=10 + kb * 7 + vb)
    rng = np.random.default_rng(kb * 10 + vb)
    # two appends: a full group and a ragged one (rows 128 .. 128 + 37)
    for t0, n in ((0, 128), (128, 37)):
        K = vals(rng, (2, 3, n, D), dt, heavy=True, outlier_cols=rng.choice(D, 3, replace=False))
        V = vals(rng, (2, 3, n, D), dt)
        p.append(K, V, t0)
    p.check_arrays(165)


def test_quantize_zero_and_constant_rows():
    # n = 0 gives the codes of u = 0 (the centroids below zero) and an all-ones sketch
    # (T(S r) = 0 >= 0); a constant row is one Walsh-Hadamard coefficient
    fd = kqv_fmt(4, 4, src_dtype=BF16)
    p = KqvPair(fd, 1, 2, 128, seed=3)
    K = np.zeros((1, 2, 16, D), np.float32)
    V = np.zeros((1, 2, 16, D), np.float32)
    K[0, 1, :8] = 2.0
    V[0, 1, 8:] = -0.5
    p.append(K, V, 0)
    p.check_arrays(16)


def test_dequantize_matches_reconstruction():
    fd = kqv_fmt(4, 4, src_dtype=BF16)
    p = KqvPair(fd, 2, 2, 256, seed=4)
    rng = np.random.default_rng(4)
    K = vals(rng, (2, 2, 200, D), BF16, heavy=True)
    V = vals(rng, (2, 2, 200, D), BF16)
    p.append(K, V, 0)
    Kh, Vh = p.reconstructed(200)
    for which, want in ((KEYS, Kh), (VALUES, Vh)):
        got = kvq.dequantize(p.fmt, p.gpu, which, 0, 200, F32).cpu().numpy().reshape(want.shape)
        err = np.abs(got - want).max(axis=-1) / np.linalg.norm(want, axis=-1)
        assert err.max() < 2e-6, (which, err.max())
    # 16-bit output: the fp32 value rounded once
    got16 = kvq.dequantize(p.fmt, p.gpu, VALUES, 0, 200, BF16).float().cpu().numpy().reshape(Vh.shape)
    np.testing.assert_allclose(got16, Vh, rtol=2 ** -8, atol=1e-6 * np.abs(Vh).max())


def kqv_reference(p, q, t_quant, sink, res, scale):
    """float64 attention per query head over raw sink rows, reconstructed packed rows and
    raw residual rows."""
    Kh, Vh = p.reconstructed(t_quant) if t_quant else (np.zeros((p.B, p.H, 0, D)),) * 2
    B, Hq = q.shape[:2]
    G = Hq // p.H
    out = np.zeros((B, Hq, D))
    for b in range(B):
        for h in range(p.H):
            K = np.concatenate([sink[0][b, h], Kh[b, h], res[0][b, h]])
            V = np.concatenate([sink[1][b, h], Vh[b, h], res[1][b, h]])
            out[b, h * G:(h + 1) * G] = oatt.attention(q[b, h * G:(h + 1) * G], K, V, scale)
    return out


def run_decode(p, G, t_quant, n_sink, t_res, out_dtype, seed, q_dtype=BF16):
    rng = np.random.default_rng(seed)
    dt = p.fd["src_dtype"]
    B, H = p.B, p.H
    sink = [vals(rng, (B, H, n_sink, D), dt) for _ in range(2)]
    res = [vals(rng, (B, H, t_res, D), dt, heavy=i == 0) for i in range(2)]
    cap = p.fd["residual_cap"]
    for name, x, rows in (("sink_k", sink[0], n_sink), ("sink_v", sink[1], n_sink),
                          ("res_k", res[0], cap), ("res_v", res[1], cap)):
        if rows:
            full = np.zeros((B, H, rows, D), np.float32)
            full[:, :, :x.shape[2]] = x
            p.gpu.array(name).copy_(torch.from_numpy(
                np.ascontiguousarray(raw_bits(full, dt)).reshape(-1).view(np.uint8)).cuda())
    q = vals(rng, (B, G * H, D), q_dtype)
    scale = 1.0 / np.sqrt(D)
    out = kvq.decode_attention(p.fmt, p.gpu, dev(q, q_dtype), t_quant, t_res, scale, out_dtype,
                               status=p.status)
    torch.cuda.synchronize()
    assert int(p.status.item()) == 0
    ref = kqv_reference(p, q.astype(np.float64), t_quant, sink, res, scale)
    return out.float().cpu().numpy(), ref


# fp32 path: codes enter as the exact fp32 centroids, so the error is fp32 accumulation
# (about 1e-6 relative); the bar leaves a hundredfold margin
KQV_TOL = 1e-4


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_decode_kqv_gqa(G):
    fd = kqv_fmt(4, 4, src_dtype=BF16, n_sink=1, residual_cap=64)
    p = KqvPair(fd, 2, 2, 1024, seed=20 + G)
    rng = np.random.default_rng(G)
    t = 3 * 128 + 77
    K = vals(rng, (2, 2, t, D), BF16, heavy=True, outlier_cols=rng.choice(D, 3, replace=False))
    V = vals(rng, (2, 2, t, D), BF16)
    p.append(K, V, 0)
    out, ref = run_decode(p, G, t, 1, 40, F32, 100 + G)
    assert_attn(out, ref, KQV_TOL)


@pytest.mark.parametrize("kb,vb,out_dtype", [(3, 3, BF16), (2, 2, F16), (4, 3, F32)])
def test_decode_kqv_bits_and_outputs(kb, vb, out_dtype):
    fd = kqv_fmt(kb, vb, src_dtype=F16, n_sink=0, residual_cap=16)
    p = KqvPair(fd, 1, 4, 2048, seed=30 + kb)
    rng = np.random.default_rng(kb + 5 * vb)
    t = 2000
    p.append(vals(rng, (1, 4, t, D), F16, heavy=True), vals(rng, (1, 4, t, D), F16), 0)
    out, ref = run_decode(p, 4, t, 0, 16, out_dtype, 200 + kb)
    assert_attn(out, ref, KQV_TOL if out_dtype == F32 else tolerance(out_dtype), out_dtype)


def test_decode_kqv_raw_only_and_single_token():
    fd = kqv_fmt(4, 4, src_dtype=BF16, n_sink=1, residual_cap=8)
    p = KqvPair(fd, 1, 2, 128, seed=40)
    out, ref = run_decode(p, 4, 0, 1, 5, F32, 300)      # no packed rows at all
    assert_attn(out, ref, KQV_TOL)
    rng = np.random.default_rng(41)
    p.append(vals(rng, (1, 2, 1, D), BF16), vals(rng, (1, 2, 1, D), BF16), 0)
    fd0 = kqv_fmt(4, 4, src_dtype=BF16, n_sink=0, residual_cap=8)
    p0 = KqvPair(fd0, 1, 2, 128, seed=40)
    p0.append(vals(rng, (1, 2, 1, D), BF16), vals(rng, (1, 2, 1, D), BF16), 0)
    out, ref = run_decode(p0, 2, 1, 0, 0, F32, 301)      # one packed token: out = v^_0
    assert_attn(out, ref, KQV_TOL)


def test_decode_kqv_long_context_splits():
    # many splits per head and the lse of the combine
    fd = kqv_fmt(4, 4, src_dtype=BF16, n_sink=1, residual_cap=128)
    p = KqvPair(fd, 1, 2, 16384, seed=50)
    rng = np.random.default_rng(50)
    t = 16384 - 5
    p.append(vals(rng, (1, 2, t, D), BF16, heavy=True, outlier_cols=[3, 70, 101]),
             vals(rng, (1, 2, t, D), BF16), 0)
    out, ref = run_decode(p, 4, t, 1, 128, F32, 400)
    assert_attn(out, ref, KQV_TOL)


@pytest.mark.timeout(1800)
def test_full_size_llama3_8b_kqv():
    # the Llama-3-8B KQV workload at full size, built and decoded as the benchmark does; two
    # sampled (batch, KV-head) slabs take host-generated values and are checked against the
    # oracle byte for byte and on their query heads' outputs
    cfg = synth.CONFIGS["llama3_8b_kqv"]
    fd = cfg["fmt"]
    B, Hq, H, g = cfg["B"], cfg["Hq"], cfg["Hkv"], fd["group_tokens"]
    G = Hq // H
    ns, tq, tr = synth.split_tokens(cfg)
    C = -(-tq // g) * g
    ck, cv = codebook(fd["k_bits"]), codebook(fd["v_bits"] - 1)
    S = np.random.default_rng(77).standard_normal((D, D)).astype(np.float32)
    fmt = kvq.make_format(fd)
    cache = kvq.Cache(fmt, B, H, C, k_lut=ck, v_lut=cv, sketch=S)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    K = synth.device_kv(cfg, "k")
    V = synth.device_kv(cfg, "v")
    slabs = [(0, 0), (7, 7)]
    host = {}
    for b, h in slabs:
        hk, hv = synth.kv_slab(cfg, b, h, which="k"), synth.kv_slab(cfg, b, h, which="v")
        K[b, h] = torch.from_numpy(np.ascontiguousarray(hk)).to(K)
        V[b, h] = torch.from_numpy(np.ascontiguousarray(hv)).to(V)
        host[(b, h)] = (hk, hv)
    kvq.quantize_kv(fmt, cache, K[:, :, ns:ns + tq], V[:, :, ns:ns + tq], 0, tq, status=status)
    a0 = (tq // g) * g - g   # the step's flush of one group
    kvq.quantize_kv(fmt, cache, K[:, :, ns + a0:ns + a0 + g].contiguous(), V[:, :, ns + a0:ns + a0 + g].contiguous(),
                    a0, g, status=status)
    cache.array("sink_k").copy_(K[:, :, :ns].contiguous().view(-1).view(torch.uint8))
    cache.array("sink_v").copy_(V[:, :, :ns].contiguous().view(-1).view(torch.uint8))
    cache.array("res_k").copy_(K[:, :, ns + tq:].contiguous().view(-1).view(torch.uint8))
    cache.array("res_v").copy_(V[:, :, ns + tq:].contiguous().view(-1).view(torch.uint8))
    del K, V
    q = synth.device_queries(cfg)
    out = kvq.decode_attention(fmt, cache, q, tq, tr, 1.0 / np.sqrt(D), F32, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got_out = out.cpu().numpy()
    kw, vw = fd["k_bits"] * D // 32, fd["v_bits"] * D // 32
    for (b, h), (hk, hv) in host.items():
        Kp, Vp = hk[ns:ns + tq], hv[ns:ns + tq]
        kc, kn = okqv.stored_encode(Kp, ck)
        parts = [okqv.stored_encode(Vp[i:i + 512], cv, S) for i in range(0, tq, 512)]
        vc, vn, sg, rn = (np.concatenate([x[j] for x in parts]) for j in range(4))
        pk = opack.pack_3bit(kc) if fd["k_bits"] == 3 else opack.pack_row(kc, fd["k_bits"])
        pv = np.concatenate([opack.pack_3bit(vc) if fd["v_bits"] == 4 else opack.pack_row(vc, fd["v_bits"] - 1),
                             opack.pack_row(sg.astype(np.int64), 1)], axis=-1)
        sl = b * H + h
        got_k = cache.array("k_codes").view(torch.int32).view(B * H, C, kw)[sl, :tq].cpu().numpy().view(np.uint32)
        got_v = cache.array("v_codes").view(torch.int32).view(B * H, C, vw)[sl, :tq].cpu().numpy().view(np.uint32)
        np.testing.assert_array_equal(got_k, pk)
        np.testing.assert_array_equal(got_v, pv)
        for name, want in (("k_scale", kn), ("v_scale", vn), ("v_zero", rn)):
            got = cache.array(name).view(torch.float32).view(B * H, C)[sl, :tq].cpu().numpy()
            np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
        Kh = np.concatenate([hk[:ns], okqv.stored_key(kc, kn, ck), hk[ns + tq:]])
        Vh = np.concatenate([hv[:ns], okqv.stored_value(vc, vn, sg, rn, cv, S), hv[ns + tq:]])
        qh = np.stack([synth.query(cfg, b, hq) for hq in range(h * G, (h + 1) * G)]).astype(np.float64)
        ref = oatt.attention(qh, Kh.astype(np.float64), Vh, 1.0 / np.sqrt(D))
        assert_attn(got_out[b, h * G:(h + 1) * G], ref, KQV_TOL)
