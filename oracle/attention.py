"""Decode attention over the cache, in float64.

[AXES] "Separate the two error paths": a key error passes through Q K^T / sqrt(D) and
the softmax, a value error straight into the weighted sum; attention uses a stable
softmax in float64.  For one decode step each query head h attends to every cached
token (no mask: the step's query is the newest position):

    out[h] = sum_t softmax_t(scale * q[h] . k_t) v_t ,  scale = 1/sqrt(D) by default,

over the raw sink tokens, the reconstructed packed rows and the raw residual window
([KVQ] "Approach": fp16 first token; [MIX] Figure 4: full-precision buffer).  Query
head h uses KV head h // G.  When the format stores pre-RoPE keys ([KVQ] "Approach":
per-channel quantization before RoPE) every key is rotated at its absolute position
t: pairs (i, i + D/2), theta_i = base^(-2i/D), the rotate-half convention.

Pinned by tests/test_oracle_attention.py (T = 1 returns v_0, q = 0 returns the mean
of v, equal keys return the mean, shift invariance, a pure-Python brute force on
tiny shapes, RoPE identities: norm preservation, identity at t = 0, dependence of
q_m . k_n on n - m only; the log-sum-exp by brute force, and the merge of disjoint
token sets equal to the attention over their union).

attention_lse / merge_parts state the sequence split ([KVQ] "Approach": contexts spread
over GPUs): each set of tokens gives its output and lse = log sum_t exp(scale q . k_t),
and the union's softmax weights split into exp(lse_r - lse) per set.
"""
from __future__ import annotations

import numpy as np

from .cache import dequantize, raw_decode
from .formats import KEYS, VALUES


def rope_rotate(k, pos, base):
    """Rotate rows of k [T, D] by the angles pos[t] * theta_i (float64)."""
    k = np.asarray(k, np.float64)
    T, D = k.shape
    half = D // 2
    i = np.arange(half, dtype=np.float64)
    theta = base ** (-2.0 * i / D)
    ang = np.asarray(pos, np.float64)[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = k[:, :half], k[:, half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=1)


def attention(q, K, V, scale):
    """Stable softmax attention of query rows q [G, D] over K, V [T, D] (float64)."""
    q = np.asarray(q, np.float64)
    s = (q @ np.asarray(K, np.float64).T) * scale
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    return (p @ np.asarray(V, np.float64)) / p.sum(axis=-1, keepdims=True)


def attention_lse(q, K, V, scale):
    """(out [G, D], lse [G]) of stable softmax attention, lse = log sum_t exp(scale q.k_t)."""
    q = np.asarray(q, np.float64)
    s = (q @ np.asarray(K, np.float64).T) * scale
    mx = s.max(axis=-1, keepdims=True)
    p = np.exp(s - mx)
    den = p.sum(axis=-1, keepdims=True)
    return (p @ np.asarray(V, np.float64)) / den, (mx + np.log(den))[..., 0]


def merge_parts(outs, lses):
    """Attention over disjoint token sets from each set's (out, lse): the softmax weights of
    the union split into per-set weights exp(lse_r - lse), lse = log sum_r exp(lse_r).
    A set without tokens has lse = -inf and weight 0 (its out is never read).  When no set
    has tokens (every lse = -inf) the union is empty and carries no softmax mass; the pages
    do not treat that case, and the reading taken is out = 0, lse = -inf."""
    outs = np.asarray(outs, np.float64)
    lses = np.asarray(lses, np.float64)
    n, D = outs.shape[0], outs.shape[-1]
    o2 = outs.reshape(n, -1, D)
    l2 = lses.reshape(n, -1)
    out = np.zeros(o2.shape[1:])
    lse = np.full(l2.shape[1], -np.inf)
    for i in range(l2.shape[1]):
        live = [r for r in range(n) if l2[r, i] != -np.inf]
        if not live:
            continue
        m = max(l2[r, i] for r in live)
        w = {r: np.exp(l2[r, i] - m) for r in live}
        tot = sum(w.values())
        out[i] = sum(w[r] * o2[r, i] for r in live) / tot
        lse[i] = m + np.log(tot)
    return out.reshape(outs.shape[1:]), lse.reshape(lses.shape[1:])


def kv_slab(fmt, cache, b, h, t_quant, t_res):
    """(K [T, D], V [T, D]) float64 of one KV head: sink, packed rows, residual."""
    A = cache.arrays
    parts_k, parts_v = [], []
    if fmt.n_sink:
        parts_k.append(raw_decode(A["sink_k"][b, h], fmt.src_dtype))
        parts_v.append(raw_decode(A["sink_v"][b, h], fmt.src_dtype))
    parts_k.append(dequantize(fmt, cache, KEYS, 0, t_quant, b, h))
    parts_v.append(dequantize(fmt, cache, VALUES, 0, t_quant, b, h))
    if t_res:
        parts_k.append(raw_decode(A["res_k"][b, h, :t_res], fmt.src_dtype))
        parts_v.append(raw_decode(A["res_v"][b, h, :t_res], fmt.src_dtype))
    K = np.concatenate(parts_k, axis=0)
    V = np.concatenate(parts_v, axis=0)
    if fmt.rope:
        K = rope_rotate(K, np.arange(K.shape[0]), fmt.rope_base)
    return K, V


def decode_attention(fmt, cache, q, t_quant, t_res, scale=None, heads=None):
    """q [B, Hq, D] (float64 values) -> out [B, Hq, D] float64.

    heads: optional list of (b, hq) to compute; other rows are left NaN."""
    q = np.asarray(q, np.float64)
    B, Hq, D = q.shape
    G = Hq // cache.H
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.full((B, Hq, D), np.nan)
    want = {}
    for (b, hq) in (heads if heads is not None else [(b, hq) for b in range(B) for hq in range(Hq)]):
        want.setdefault((b, hq // G), []).append(hq)
    for (b, h), hqs in sorted(want.items()):
        K, V = kv_slab(fmt, cache, b, h, t_quant, t_res)
        hqs = sorted(hqs)
        out[b, hqs] = attention(q[b, hqs], K, V, scale)
    return out


def rel_l2(out, ref):
    """||out - ref||_2 / ||ref||_2 ([AXES] "The hybrid wins one condition")."""
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(out - ref) / np.linalg.norm(ref))
