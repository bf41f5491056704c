"""The packed cache as numpy arrays, and the quantize / dequantize operations on it.

Arrays have the exact element types and shapes of the device arrays (fp16 values as
their uint16 encodings), so a test compares them byte for byte.  Operations follow
the library's entry points: `quantize(fmt, cache, which, src, t0, n)` appends whole
token groups, `dequantize(fmt, cache, which, t0, n)` reconstructs fp32 values.  With
`k_rotate` the keys are quantized in the Walsh-Hadamard basis (oracle.rotate) and
reconstructed back into the original one.

Per-group rules come from oracle.quant, packing from oracle.pack; the grouping is
that of [AXES] "What rows and columns mean" (tensor / token / channel) and of
[KVQ] "Approach" (keys per channel over a token group, values per token).
"""
from __future__ import annotations

import numpy as np

from . import fp, pack, quant, rotate
from .formats import (ASYM, BF16, CHANNEL, F16, F32, KEYS, MIXED, NONE, NUQ, SYM8,
                      TENSOR, TOKEN, VALUES, Format, side)


def raw_encode(values, dtype):
    """Exact source values -> stored raw representation."""
    if dtype == F32:
        return fp.f32_bits(values).view(np.float32)
    if dtype == F16:
        return fp.f16_bits(values)
    return fp.bf16_bits(values)


def raw_decode(stored, dtype):
    if dtype == F32:
        return np.asarray(stored, np.float32).astype(np.float64)
    if dtype == F16:
        return fp.f16_from_bits(stored)
    return fp.bf16_from_bits(stored)


def _raw_np(dtype):
    return np.float32 if dtype == F32 else np.uint16


class Cache:
    """Zero-initialised cache arrays for B x H slabs of capacity C tokens."""

    def __init__(self, fmt: Format, B: int, H: int, C: int, k_lut=None, v_lut=None):
        assert C % fmt.group_tokens == 0
        self.fmt, self.B, self.H, self.C = fmt, B, H, C
        D, g = fmt.head_dim, fmt.group_tokens
        ng = C // g
        self.ng = ng
        a = {}
        rawt = _raw_np(fmt.src_dtype)
        for which in (KEYS, VALUES):
            p = "k_" if which == KEYS else "v_"
            scheme, bits, axis, nout = side(fmt, which)
            if scheme == NONE:
                a[p + "codes"] = np.zeros((B, H, C, D), rawt)
            elif scheme == SYM8:
                a[p + "codes"] = np.zeros((B, H, C, D), np.int8)
                shape = {TENSOR: (B, H, ng), TOKEN: (B, H, C), CHANNEL: (B, H, ng, D)}[axis]
                a[p + "scale"] = np.zeros(shape, np.float32)
            elif scheme == ASYM:
                if bits == 8:
                    a[p + "codes"] = np.zeros((B, H, C, D), np.uint8)
                elif which == KEYS:
                    a[p + "codes"] = np.zeros((B, H, C, D * bits // 32), np.uint32)
                else:
                    a[p + "codes"] = np.zeros((B, H, C // 2, D * bits // 16), np.uint32)
                shape = (B, H, ng, D) if axis == CHANNEL else (B, H, C)
                a[p + "scale"] = np.zeros(shape, np.uint16)
                a[p + "zero"] = np.zeros(shape, np.uint16)
            elif scheme == NUQ:
                a[p + "codes"] = np.zeros((B, H, C, 3 * D // 32), np.uint32)
                shape = (B, H, ng, D) if axis == CHANNEL else (B, H, C)
                a[p + "scale"] = np.zeros(shape, np.uint16)
                a[p + "zero"] = np.zeros(shape, np.uint16)
                lut = k_lut if which == KEYS else v_lut
                a[p + "lut"] = fp.f16_bits(np.asarray(lut, np.float64))
                if nout > 0:
                    if which == KEYS:
                        a["k_out_rowptr"] = np.zeros((B, H, ng, g + 1), np.int32)
                        a["k_out_col"] = np.zeros((B, H, ng, D * nout), np.uint8)
                        a["k_out_val"] = np.zeros((B, H, ng, D * nout), np.uint16)
                    else:
                        a["v_out_col"] = np.zeros((B, H, C, nout), np.uint8)
                        a["v_out_val"] = np.zeros((B, H, C, nout), np.uint16)
            elif scheme == MIXED:
                rb = 2 * fmt.mixed_hi + fmt.mixed_mid // 2 + fmt.mixed_lo // 4
                a["k_codes"] = np.zeros((B, H, ng, g * rb), np.uint8)
                a["k_scale"] = np.zeros((B, H, ng, D - fmt.mixed_hi), np.uint16)
                a["k_zero"] = np.zeros((B, H, ng, D - fmt.mixed_hi), np.uint16)
                a["k_order"] = np.zeros((B, H, ng, D), np.uint8)
        if fmt.n_sink:
            a["sink_k"] = np.zeros((B, H, fmt.n_sink, D), rawt)
            a["sink_v"] = np.zeros((B, H, fmt.n_sink, D), rawt)
        if fmt.residual_cap:
            a["res_k"] = np.zeros((B, H, fmt.residual_cap, D), rawt)
            a["res_v"] = np.zeros((B, H, fmt.residual_cap, D), rawt)
        self.arrays = a

    def __getitem__(self, k):
        return self.arrays[k]

    def lut(self, which):
        return fp.f16_from_bits(self.arrays["k_lut" if which == KEYS else "v_lut"])

    # MIXED planes of one group (views into k_codes)
    def mixed_planes(self, b, h, gi):
        f = self.fmt
        g = f.group_tokens
        blk = self.arrays["k_codes"][b, h, gi]
        o1 = g * 2 * f.mixed_hi
        o2 = o1 + g * f.mixed_mid // 2
        raw = blk[:o1].view(np.uint16).reshape(g, f.mixed_hi)
        mid = blk[o1:o2].view(np.uint32).reshape(g, f.mixed_mid // 8)
        lo = blk[o2:].view(np.uint32).reshape(g, f.mixed_lo // 16)
        return raw, mid, lo


def _groups(fmt, t0, n):
    g = fmt.group_tokens
    assert t0 % g == 0
    gi = t0 // g
    t = t0
    while t < t0 + n:
        ln = min(g, t0 + n - t)
        yield gi, t, ln
        gi += 1
        t += ln


def quantize(fmt: Format, cache: Cache, which: int, src, t0: int, n: int):
    """Quantize src [B, H, n, D] (exact source values, float64) into rows [t0, t0+n)."""
    src = np.asarray(src, np.float64)
    quant.check_finite(src)
    if which == KEYS and fmt.k_rotate:
        # [K4V2] "Rotation Integration": keys are rotated before their statistics
        src = rotate.wht_f32(src)
    B, H = cache.B, cache.H
    assert src.shape[:3] == (B, H, n)
    scheme, bits, axis, nout = side(fmt, which)
    p = "k_" if which == KEYS else "v_"
    A = cache.arrays
    for b in range(B):
        for h in range(H):
            for gi, ts, ln in _groups(fmt, t0, n):
                X = src[b, h, ts - t0: ts - t0 + ln]
                if scheme == NONE:
                    A[p + "codes"][b, h, ts:ts + ln] = raw_encode(X, fmt.src_dtype)
                elif scheme == SYM8:
                    _sym8_group(A, p, b, h, gi, ts, X, axis)
                elif scheme == ASYM:
                    _asym_group(A, p, which, b, h, gi, ts, X, bits)
                elif scheme == NUQ:
                    _nuq_group(cache, p, which, b, h, gi, ts, X, nout)
                elif scheme == MIXED:
                    _mixed_group(cache, b, h, gi, X)


def _sym8_group(A, p, b, h, gi, ts, X, axis):
    ln = X.shape[0]
    if axis == TENSOR:
        s = quant.sym8_scale(np.abs(X).max())
        A[p + "scale"][b, h, gi] = s
        S = s
    elif axis == TOKEN:
        s = quant.sym8_scale(np.abs(X).max(axis=1))
        A[p + "scale"][b, h, ts:ts + ln] = s
        S = s[:, None]
    else:
        s = quant.sym8_scale(np.abs(X).max(axis=0))
        A[p + "scale"][b, h, gi] = s
        S = s[None, :]
    A[p + "codes"][b, h, ts:ts + ln] = quant.sym8_encode(X, S)


def _asym_group(A, p, which, b, h, gi, ts, X, bits):
    ln = X.shape[0]
    if which == KEYS:      # per channel over the group
        s, z = quant.asym_params(X.min(axis=0), X.max(axis=0), bits)
        A[p + "scale"][b, h, gi] = fp.f16_bits(s)
        A[p + "zero"][b, h, gi] = fp.f16_bits(z)
        codes = quant.asym_encode(X, s[None, :], z[None, :], bits)
    else:                  # per token row
        s, z = quant.asym_params(X.min(axis=1), X.max(axis=1), bits)
        A[p + "scale"][b, h, ts:ts + ln] = fp.f16_bits(s)
        A[p + "zero"][b, h, ts:ts + ln] = fp.f16_bits(z)
        codes = quant.asym_encode(X, s[:, None], z[:, None], bits)
    if bits == 8:
        A[p + "codes"][b, h, ts:ts + ln] = codes.astype(np.uint8)
    elif which == KEYS:
        A[p + "codes"][b, h, ts:ts + ln] = pack.pack_row(codes, bits)
    else:
        assert ts % 2 == 0
        words = pack.pack_pair(codes, bits)
        A[p + "codes"][b, h, ts // 2: ts // 2 + words.shape[0]] = words


def _nuq_group(cache, p, which, b, h, gi, ts, X, nout):
    A = cache.arrays
    C = cache.lut(which)
    ln, D = X.shape
    g = cache.fmt.group_tokens
    codes = np.zeros((ln, D), np.int64)
    if which == KEYS:
        mask = np.zeros((ln, D), bool)
        vals = np.zeros((ln, D), np.float64)
        s_all = np.zeros(D)
        z_all = np.zeros(D)
        for c in range(D):
            col = X[:, c]
            idx = quant.topk_outliers(col, nout)
            mn, mx = quant.dense_minmax(col, idx)
            s, z = quant.nuq_params(mn, mx)
            s_all[c], z_all[c] = s, z
            codes[:, c] = quant.nuq_encode(np.clip(col, mn, mx), s, z, C)
            mask[idx, c] = True
            vals[idx, c] = col[idx]
        A[p + "scale"][b, h, gi] = fp.f16_bits(s_all)
        A[p + "zero"][b, h, gi] = fp.f16_bits(z_all)
        if nout > 0:
            rowptr = np.zeros(g + 1, np.int32)
            cols, outv = [], []
            for t in range(g):
                if t < ln:
                    for c in np.nonzero(mask[t])[0]:
                        cols.append(c)
                        outv.append(vals[t, c])
                rowptr[t + 1] = len(cols)
            ov = fp.f16(np.array(outv, np.float64), "rn")
            if not np.all(np.isfinite(ov)):
                raise quant.RangeExceeded("outlier value beyond fp16")
            A["k_out_rowptr"][b, h, gi] = rowptr
            A["k_out_col"][b, h, gi] = 0
            A["k_out_val"][b, h, gi] = 0
            A["k_out_col"][b, h, gi, :len(cols)] = np.array(cols, np.uint8)
            A["k_out_val"][b, h, gi, :len(cols)] = fp.f16_bits(ov)
    else:
        s_all = np.zeros(ln)
        z_all = np.zeros(ln)
        for t in range(ln):
            row = X[t]
            idx = quant.topk_outliers(row, nout)
            mn, mx = quant.dense_minmax(row, idx)
            s, z = quant.nuq_params(mn, mx)
            s_all[t], z_all[t] = s, z
            codes[t] = quant.nuq_encode(np.clip(row, mn, mx), s, z, C)
            if nout > 0:
                ov = fp.f16(row[idx], "rn")
                if not np.all(np.isfinite(ov)):
                    raise quant.RangeExceeded("outlier value beyond fp16")
                A["v_out_col"][b, h, ts + t] = idx.astype(np.uint8)
                A["v_out_val"][b, h, ts + t] = fp.f16_bits(ov)
        A[p + "scale"][b, h, ts:ts + ln] = fp.f16_bits(s_all)
        A[p + "zero"][b, h, ts:ts + ln] = fp.f16_bits(z_all)
    A[p + "codes"][b, h, ts:ts + ln] = pack.pack_3bit(codes)


def _mixed_group(cache, b, h, gi, X):
    f = cache.fmt
    A = cache.arrays
    order = A["k_order"][b, h, gi].astype(np.int64)
    raw, mid, lo = cache.mixed_planes(b, h, gi)
    ln = X.shape[0]
    hi_ch = order[: f.mixed_hi]
    mid_ch = order[f.mixed_hi: f.mixed_hi + f.mixed_mid]
    lo_ch = order[f.mixed_hi + f.mixed_mid:]
    raw[:ln] = raw_encode(X[:, hi_ch], f.src_dtype).reshape(ln, f.mixed_hi)
    s_all, z_all = [], []
    for chans, bits, plane in ((mid_ch, 4, mid), (lo_ch, 2, lo)):
        Y = X[:, chans]
        s, z = quant.asym_params(Y.min(axis=0), Y.max(axis=0), bits)
        codes = quant.asym_encode(Y, s[None, :], z[None, :], bits)
        plane[:ln] = pack.pack_row(codes, bits)
        s_all.append(s)
        z_all.append(z)
    A["k_scale"][b, h, gi] = fp.f16_bits(np.concatenate(s_all))
    A["k_zero"][b, h, gi] = fp.f16_bits(np.concatenate(z_all))


# ---- reconstruction ------------------------------------------------------------

def dequantize(fmt: Format, cache: Cache, which: int, t0: int, n: int, b=None, h=None):
    """fp32 reconstruction of rows [t0, t0+n): float64 array [B, H, n, D] (or [n, D]
    for a single slab when b and h are given)."""
    if b is not None:
        return _deq_slab(fmt, cache, which, b, h, t0, n)
    out = np.zeros((cache.B, cache.H, n, fmt.head_dim))
    for bb in range(cache.B):
        for hh in range(cache.H):
            out[bb, hh] = _deq_slab(fmt, cache, which, bb, hh, t0, n)
    return out


def _deq_slab(fmt, cache, which, b, h, t0, n):
    out = _deq_slab_stored(fmt, cache, which, b, h, t0, n)
    if which == KEYS and fmt.k_rotate and n > 0:
        # the stored basis is rotated; the normalised transform is its own inverse
        out = rotate.wht_f32(out)
    return out


def _deq_slab_stored(fmt, cache, which, b, h, t0, n):
    A = cache.arrays
    D, g = fmt.head_dim, fmt.group_tokens
    scheme, bits, axis, nout = side(fmt, which)
    p = "k_" if which == KEYS else "v_"
    out = np.zeros((n, D))
    if n == 0:
        return out
    tok = np.arange(t0, t0 + n)
    gidx = tok // g
    if scheme == NONE:
        return raw_decode(A[p + "codes"][b, h, t0:t0 + n], fmt.src_dtype)
    if scheme == SYM8:
        codes = A[p + "codes"][b, h, t0:t0 + n].astype(np.float64)
        sc = A[p + "scale"][b, h].astype(np.float64)
        if axis == TENSOR:
            S = sc[gidx][:, None]
        elif axis == TOKEN:
            S = sc[tok][:, None]
        else:
            S = sc[gidx]
        return quant.sym8_decode(codes, S)
    if scheme == ASYM:
        if bits == 8:
            codes = A[p + "codes"][b, h, t0:t0 + n].astype(np.int64)
        elif which == KEYS:
            codes = pack.unpack_row(A[p + "codes"][b, h, t0:t0 + n], bits, D)
        else:
            pairs = A[p + "codes"][b, h]
            allc = pack.unpack_pair(pairs, bits, pairs.shape[0] * 2, D)
            codes = allc[t0:t0 + n]
        s = fp.f16_from_bits(A[p + "scale"][b, h])
        z = fp.f16_from_bits(A[p + "zero"][b, h])
        if which == KEYS:
            return quant.asym_decode(codes, s[gidx], z[gidx])
        return quant.asym_decode(codes, s[tok][:, None], z[tok][:, None])
    if scheme == NUQ:
        C = cache.lut(which)
        codes = pack.unpack_3bit(A[p + "codes"][b, h, t0:t0 + n], D)
        s = fp.f16_from_bits(A[p + "scale"][b, h])
        z = fp.f16_from_bits(A[p + "zero"][b, h])
        if which == KEYS:
            out = quant.nuq_decode(codes, s[gidx], z[gidx], C)
        else:
            out = quant.nuq_decode(codes, s[tok][:, None], z[tok][:, None], C)
        if nout > 0:
            for i, t in enumerate(tok):
                if which == KEYS:
                    gi, r = t // g, t % g
                    rp = A["k_out_rowptr"][b, h, gi]
                    for e in range(rp[r], rp[r + 1]):
                        c = int(A["k_out_col"][b, h, gi, e])
                        out[i, c] = fp.f16_from_bits(A["k_out_val"][b, h, gi, e])
                else:
                    for e in range(nout):
                        c = int(A["v_out_col"][b, h, t, e])
                        out[i, c] = fp.f16_from_bits(A["v_out_val"][b, h, t, e])
        return out
    if scheme == MIXED:
        f = fmt
        for i, t in enumerate(tok):
            gi, r = t // g, t % g
            order = A["k_order"][b, h, gi].astype(np.int64)
            raw, mid, lo = cache.mixed_planes(b, h, gi)
            s = fp.f16_from_bits(A["k_scale"][b, h, gi])
            z = fp.f16_from_bits(A["k_zero"][b, h, gi])
            out[i, order[: f.mixed_hi]] = raw_decode(raw[r], f.src_dtype)
            cm = pack.unpack_row(mid[r], 4, f.mixed_mid)
            cl = pack.unpack_row(lo[r], 2, f.mixed_lo)
            codes = np.concatenate([cm, cl])
            out[i, order[f.mixed_hi:]] = quant.asym_decode(codes, s, z)
        return out
    raise ValueError(scheme)
