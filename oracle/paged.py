"""Paged cache with per-sequence lengths ([MIX] Figures 4 and 5: a serving cache whose
sequences grow by whole token groups flushed from their raw windows; the pages give no
layout, so the plainest one is taken and stated here).

Test infrastructure: the CUDA library is checked against this module; nothing in the
library imports it.

Layout (a reading, not on the pages): the packed arrays form a pool of blocks, one token
group (group_tokens tokens) of every KV head per block, laid out exactly as an
oracle.cache.Cache of batch = num_blocks, H = kv_heads and capacity = group_tokens.  A
sequence owns the blocks block_table[s][0 .. ceil(t_quant[s] / g)) in token order; its
sink and residual tokens are raw arrays [num_seqs][kv_heads][...] as in the contiguous
cache.  Every group is quantized on its own (keys per channel over the group, values
per token), so a sequence's packed bytes do not depend on where its groups are stored.

decode_attention reconstructs each sequence's tokens from its own blocks and applies
oracle.attention.decode_attention to them: attention over that sequence's n_sink +
t_quant[s] + t_res[s] tokens only.  A sequence with no tokens at all has no softmax mass;
its rows are 0 (the reading taken for an empty union in oracle.attention.merge_parts).
"""
from __future__ import annotations

import numpy as np

from . import attention as oatt
from . import cache as ocache
from .formats import KEYS, MIXED, Format

POOL_ARRAYS = ("k_codes", "k_scale", "k_zero", "k_order", "k_out_rowptr", "k_out_col", "k_out_val",
               "v_codes", "v_scale", "v_zero", "v_out_col", "v_out_val")


class PagedCache:
    """A pool of num_blocks blocks plus per-sequence raw sink / residual arrays."""

    def __init__(self, fmt: Format, kv_heads: int, num_blocks: int, num_seqs: int, max_blocks: int,
                 k_lut=None, v_lut=None):
        self.fmt, self.H, self.num_blocks = fmt, kv_heads, num_blocks
        self.num_seqs, self.max_blocks = num_seqs, max_blocks
        g = fmt.group_tokens
        self.luts = (k_lut, v_lut)
        self.pool = ocache.Cache(fmt, num_blocks, kv_heads, g, k_lut=k_lut, v_lut=v_lut)
        # raw arrays, per sequence (the pool's own raw arrays are unused)
        self.raw = ocache.Cache(fmt, num_seqs, kv_heads, g, k_lut=k_lut, v_lut=v_lut)
        self.block_table = np.full((num_seqs, max_blocks), -1, np.int32)


def quantize_group(pc: PagedCache, which: int, src, block: int, n: int):
    """Quantize the first n <= g tokens of one group, src [kv_heads, n, D] (exact source
    values), into pool block `block`: the group is quantized as group 0 of a one-group
    cache and its bytes are stored in the block."""
    fmt = pc.fmt
    tmp = ocache.Cache(fmt, 1, pc.H, fmt.group_tokens, k_lut=pc.luts[0], v_lut=pc.luts[1])
    if fmt.k_scheme == MIXED and which == KEYS:
        tmp["k_order"][0] = pc.pool["k_order"][block]
    ocache.quantize(fmt, tmp, which, np.asarray(src, np.float64)[None], 0, n)
    p = "k_" if which == KEYS else "v_"
    for name in POOL_ARRAYS:
        if name.startswith(p) and name in tmp.arrays and name != "k_order":
            pc.pool[name][block] = tmp[name][0]


def sequence_cache(pc: PagedCache, s: int, t_quant: int):
    """Sequence s as a contiguous one-sequence oracle cache: its blocks gathered in order,
    its sink and residual rows copied."""
    fmt, g = pc.fmt, pc.fmt.group_tokens
    ng = -(-t_quant // g)
    c = ocache.Cache(fmt, 1, pc.H, max(1, ng) * g, k_lut=pc.luts[0], v_lut=pc.luts[1])
    for gi in range(ng):
        blk = int(pc.block_table[s, gi])
        for name in POOL_ARRAYS:
            if name not in c.arrays:
                continue
            src = pc.pool[name][blk]     # [H, rows of one group, ...]
            per = src.shape[1]
            c[name][0][:, gi * per:(gi + 1) * per] = src
    for name in ("sink_k", "sink_v", "res_k", "res_v"):
        if name in c.arrays:
            c[name][0] = pc.raw[name][s]
    return c


def decode_attention(pc: PagedCache, q, t_quant, t_res, scale=None):
    """q [num_seqs, Hq, D] (float64 values) -> out [num_seqs, Hq, D] float64, each
    sequence over its own tokens."""
    q = np.asarray(q, np.float64)
    out = np.zeros_like(q)
    for s in range(pc.num_seqs):
        tq, tr = int(t_quant[s]), int(t_res[s])
        if pc.fmt.n_sink + tq + tr == 0:
            continue
        c = sequence_cache(pc, s, tq)
        out[s] = oatt.decode_attention(pc.fmt, c, q[s:s + 1], tq, tr, scale)[0]
    return out
