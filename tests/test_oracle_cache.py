"""Pins of oracle.cache (grouping, packing into the cache arrays, outlier lists, mixed
tiers, sink / residual assembly) against brute-force restatements on small inputs."""
import numpy as np
import pytest

import synth
from oracle import attention, fp, quant, salience
from oracle.cache import Cache, dequantize, quantize
from oracle.formats import (ASYM, BF16, CHANNEL, F16, F32, KEYS, MIXED, NONE, NUQ,
                            SYM8, TENSOR, TOKEN, VALUES, Format)

UNIFORM_LUT = (np.arange(8) - 3.5) / 4


def _src(seed, shape, dtype=F16, scale=1.0):
    r = np.random.default_rng(seed)
    x = r.standard_normal(shape).astype(np.float32) * np.float32(scale)
    return synth.to_dtype_values(x, dtype).astype(np.float64)


@pytest.mark.parametrize("kb,vb", [(4, 2), (2, 4), (8, 8)])
def test_asym_cache_bound_and_groups(kb, vb):
    f = Format(head_dim=32, group_tokens=16, k_bits=kb, v_bits=vb)
    B, H, C, n = 2, 3, 64, 37                       # two full groups + a partial one
    c = Cache(f, B, H, C)
    K = _src(0, (B, H, n, 32), scale=3.0)
    V = _src(1, (B, H, n, 32))
    quantize(f, c, KEYS, K, 0, n)
    quantize(f, c, VALUES, V, 0, n)
    Kh = dequantize(f, c, KEYS, 0, n)
    Vh = dequantize(f, c, VALUES, 0, n)
    for b in range(B):
        for h in range(H):
            for g0 in range(0, n, 16):
                blk = K[b, h, g0:g0 + 16]
                s, z = quant.asym_params(blk.min(0), blk.max(0), kb)
                gi = g0 // 16
                np.testing.assert_array_equal(fp.f16_from_bits(c["k_scale"][b, h, gi]), s)
                assert np.all(np.abs(blk - Kh[b, h, g0:g0 + 16]) <= s * (0.5 + 2.0 ** -20))
            sv = fp.f16_from_bits(c["v_scale"][b, h, :n])
            assert np.all(np.abs(V[b, h] - Vh[b, h]) <= sv[:, None] * (0.5 + 2.0 ** -20))
    # rows past n are untouched
    assert not np.any(c["v_scale"][:, :, n:])


def test_rewriting_a_partial_group():
    f = Format(head_dim=32, group_tokens=16)
    c1, c2 = Cache(f, 1, 1, 32), Cache(f, 1, 1, 32)
    K = _src(2, (1, 1, 32, 32))
    quantize(f, c1, KEYS, K[:, :, :20], 0, 20)       # group 1 partial (4 tokens)
    quantize(f, c1, KEYS, K[:, :, 16:], 16, 16)      # rewrite group 1 whole
    quantize(f, c2, KEYS, K, 0, 32)
    for k in ("k_codes", "k_scale", "k_zero"):
        np.testing.assert_array_equal(c1[k], c2[k])


def test_sym8_axes_match_page_scale_shapes():
    N, D = 64, 32
    Q, K, V = synth.toy(7, N)
    for scheme in ("tensor", "token", "hybrid"):
        f = Format(**synth.toy_format(scheme, "both", N, D))
        c = Cache(f, 1, 1, N)
        quantize(f, c, KEYS, K[None, None].astype(np.float64), 0, N)
        quantize(f, c, VALUES, V[None, None].astype(np.float64), 0, N)
        ka = {"tensor": TENSOR, "token": TOKEN, "hybrid": CHANNEL}[scheme]
        n_k = {TENSOR: 1, TOKEN: N, CHANNEL: D}[ka]
        assert c["k_scale"].size == n_k
        assert c["v_scale"].size == (1 if scheme == "tensor" else N)
        # reconstruction code * scale within half a step
        Kh = dequantize(f, c, KEYS, 0, N)[0, 0]
        sk = c["k_scale"].astype(np.float64).reshape({TENSOR: (1, 1), TOKEN: (N, 1), CHANNEL: (1, D)}[ka])
        assert np.all(np.abs(Kh - K) <= sk * (0.5 + 2.0 ** -20))


def test_nuq_outliers_csr():
    f = Format(head_dim=32, group_tokens=16, k_scheme=NUQ, k_bits=3, k_outliers=2,
               v_scheme=NUQ, v_bits=3, v_outliers=2)
    B, H, n = 1, 2, 27
    c = Cache(f, B, H, 32, k_lut=UNIFORM_LUT, v_lut=UNIFORM_LUT)
    K = _src(3, (B, H, n, 32), scale=2.0)
    V = _src(4, (B, H, n, 32))
    quantize(f, c, KEYS, K, 0, n)
    quantize(f, c, VALUES, V, 0, n)
    Kh = dequantize(f, c, KEYS, 0, n)
    Vh = dequantize(f, c, VALUES, 0, n)
    for b in range(B):
        for h in range(H):
            for gi, (g0, ln) in enumerate(((0, 16), (16, 11))):
                rp = c["k_out_rowptr"][b, h, gi]
                assert rp[0] == 0 and np.all(np.diff(rp) >= 0) and rp[-1] == 32 * 2
                cols = c["k_out_col"][b, h, gi]
                # every channel has exactly 2 outliers in the group, at its top-2 |x|
                for ch in range(32):
                    col = K[b, h, g0:g0 + ln, ch]
                    idx = quant.topk_outliers(col, 2)
                    for t in idx:
                        ent = range(rp[t], rp[t + 1])
                        assert ch in [int(cols[e]) for e in ent]
                        assert Kh[b, h, g0 + t, ch] == fp.f16(col[t])
                # entries sorted by (row, channel)
                for t in range(16):
                    cs = cols[rp[t]:rp[t + 1]]
                    assert np.all(np.diff(cs.astype(int)) > 0)
            for t in range(n):
                idx = quant.topk_outliers(V[b, h, t], 2)
                assert c["v_out_col"][b, h, t].tolist() == idx.tolist()
                np.testing.assert_array_equal(Vh[b, h, t, idx], V[b, h, t, idx])
                # dense entries are within half a level spacing of their value
                rest = np.setdiff1d(np.arange(32), idx)
                s = fp.f16_from_bits(c["v_scale"][b, h, t])
                assert np.all(np.abs(Vh[b, h, t, rest] - V[b, h, t, rest]) <= s * (0.125 + 2.0 ** -18))


def test_mixed_tiers():
    f = Format(head_dim=64, group_tokens=16, src_dtype=BF16, k_scheme=MIXED, mixed_hi=8,
               mixed_mid=8)
    B, H, n, G = 1, 2, 16, 3
    c = Cache(f, B, H, 16)
    K = _src(5, (B, H, n, 64), BF16) * np.exp(np.random.default_rng(6).uniform(-2, 3, 64))
    K = synth.to_dtype_values(K.astype(np.float32), BF16).astype(np.float64)
    Q = _src(7, (B, H * G, n, 64), BF16)
    for b in range(B):
        for h in range(H):
            A, order = salience.key_salience(Q[b, h * G:(h + 1) * G], K[b, h])
            c["k_order"][b, h, 0] = order
    quantize(f, c, KEYS, K, 0, n)
    Kh = dequantize(f, c, KEYS, 0, n)
    for b in range(B):
        for h in range(H):
            order = c["k_order"][b, h, 0].astype(int)
            hi, mid, lo = order[:8], order[8:16], order[16:]
            np.testing.assert_array_equal(Kh[b, h][:, hi], K[b, h][:, hi])
            s = fp.f16_from_bits(c["k_scale"][b, h, 0])
            for chans, ss in ((mid, s[:8]), (lo, s[8:])):
                assert np.all(np.abs(Kh[b, h][:, chans] - K[b, h][:, chans]) <= ss * (0.5 + 2.0 ** -20))


def test_decode_assembles_sink_packed_residual():
    f = Format(head_dim=32, group_tokens=16, src_dtype=BF16, n_sink=1, residual_cap=8)
    B, H, Hq, tq, tr = 1, 2, 4, 20, 5
    c = Cache(f, B, H, 32)
    Kp = _src(8, (B, H, tq, 32), BF16)
    Vp = _src(9, (B, H, tq, 32), BF16)
    quantize(f, c, KEYS, Kp, 0, tq)
    quantize(f, c, VALUES, Vp, 0, tq)
    sk = _src(10, (B, H, 1, 32), BF16)
    sv = _src(11, (B, H, 1, 32), BF16)
    rk = _src(12, (B, H, 8, 32), BF16)
    rv = _src(13, (B, H, 8, 32), BF16)
    c["sink_k"][...] = fp.bf16_bits(sk)
    c["sink_v"][...] = fp.bf16_bits(sv)
    c["res_k"][...] = fp.bf16_bits(rk)
    c["res_v"][...] = fp.bf16_bits(rv)
    q = _src(14, (B, Hq, 32), BF16)
    out = attention.decode_attention(f, c, q, tq, tr)
    Kh = dequantize(f, c, KEYS, 0, tq)
    Vh = dequantize(f, c, VALUES, 0, tq)
    for hq in range(Hq):
        h = hq // 2
        K = np.concatenate([sk[0, h], Kh[0, h], rk[0, h, :tr]])
        V = np.concatenate([sv[0, h], Vh[0, h], rv[0, h, :tr]])
        want = attention.attention(q[0, hq:hq + 1], K, V, 1 / np.sqrt(32))
        np.testing.assert_allclose(out[0, hq], want[0], rtol=1e-12, atol=1e-15)


def test_rejects_nonfinite_source():
    f = Format(head_dim=32, group_tokens=16)
    c = Cache(f, 1, 1, 16)
    K = np.zeros((1, 1, 16, 32))
    K[0, 0, 3, 4] = np.nan
    with pytest.raises(quant.RejectedInput):
        quantize(f, c, KEYS, K, 0, 16)


def test_paged_decode_equals_contiguous_per_sequence():
    # A paged cache whose sequences own scattered blocks gives each sequence the attention
    # over its own tokens: the same output as a contiguous cache holding that sequence
    # alone, whatever the block placement (lengths with ragged last groups, one group, none)
    from oracle import attention as oatt
    from oracle import cache as ocache
    from oracle import paged
    from oracle.formats import Format

    def vals(shape):
        return fp.f16(rng.standard_normal(shape))
    fd = dict(head_dim=32, group_tokens=16, src_dtype=F16, n_sink=1, residual_cap=8)
    f = Format(**fd)
    H, G, g = 2, 2, 16
    t_quant = [37, 16, 5, 0]
    t_res = [3, 0, 8, 2]
    S = len(t_quant)
    rng = np.random.default_rng(8)
    pc = paged.PagedCache(f, H, num_blocks=9, num_seqs=S, max_blocks=3)
    perm = rng.permutation(9)
    contig, used = [], 0
    for s in range(S):
        ng = -(-t_quant[s] // g)
        c = ocache.Cache(f, 1, H, max(1, ng) * g)
        K = vals((1, H, max(1, ng) * g, 32))
        V = vals((1, H, max(1, ng) * g, 32))
        for gi in range(ng):
            n = min(g, t_quant[s] - gi * g)
            blk = int(perm[used]); used += 1
            pc.block_table[s, gi] = blk
            paged.quantize_group(pc, KEYS, K[0, :, gi * g:gi * g + n], blk, n)
            paged.quantize_group(pc, VALUES, V[0, :, gi * g:gi * g + n], blk, n)
            ocache.quantize(f, c, KEYS, K[:, :, gi * g:gi * g + n], gi * g, n)
            ocache.quantize(f, c, VALUES, V[:, :, gi * g:gi * g + n], gi * g, n)
        for name, shape in (("sink_k", 1), ("sink_v", 1), ("res_k", 8), ("res_v", 8)):
            raw = ocache.raw_encode(vals((H, shape, 32)), F16)
            pc.raw[name][s] = raw
            c[name][0] = raw
        contig.append(c)
    q = vals((S, H * G, 32))
    got = paged.decode_attention(pc, q, t_quant, t_res)
    for s in range(S):
        want = oatt.decode_attention(f, contig[s], q[s:s + 1], t_quant[s], t_res[s])[0]
        np.testing.assert_array_equal(got[s], want)
        # and the gathered cache holds the same packed bytes as the contiguous one
        gc = paged.sequence_cache(pc, s, t_quant[s])
        for name in ("k_codes", "k_scale", "k_zero", "v_codes", "v_scale", "v_zero"):
            n_rows = gc[name].shape[2]
            np.testing.assert_array_equal(gc[name][0][:, :n_rows], contig[s][name][0][:, :n_rows])
