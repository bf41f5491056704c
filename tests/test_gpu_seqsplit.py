"""GPU parity of the sequence split ([KVQ] "Approach": a long context spread over GPUs),
on one GPU: a context is cut into disjoint parts (the first with the attention sink,
the last with the residual window), every part is its own cache decoded by
kvq_decode_partial + kvq_decode_combine_lse, and kvq_merge_states joins the parts.  The
result must match the float64 oracle over the union of the parts' reconstructed tokens;
a single part merges to the plain decode bit for bit.  (The all-gather between ranks is
covered by the two-rank gloo test.)"""
import json
import os

import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from oracle.formats import BF16, F16, F32, NUQ
from quantized_decode_attention_quantize_b200 import kvq, seqsplit
from tests.gpu_util import assert_attn, dev, rel_l2
from tests.test_gpu_decode import build, vals

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LUT = json.load(open(os.path.join(ROOT, "tests", "golden", "nuq3_codebook.json")))


def _parts(kw, B, H, G, spans, seed):
    """spans: (n_sink, t_quant, t_res) per part."""
    parts = []
    for i, (ns, tq, tr) in enumerate(spans):
        fd = synth._fmt(src_dtype=BF16, n_sink=ns, residual_cap=max(tr, 1) if tr else 0, **kw)
        luts = (LUT["k"], LUT["v"]) if fd["k_scheme"] == NUQ else (None, None)
        parts.append((build(fd, B, H, G * H, tq, tr, seed=seed + 10 * i, luts=luts), tq, tr))
    return parts


@pytest.mark.parametrize("kw,G,spans", [
    (dict(), 4, [(1, 3 * 128 + 5, 0), (0, 2 * 128 + 64, 0), (0, 128 + 17, 40)]),   # tensor-core path
    (dict(), 5, [(1, 2 * 128, 0), (0, 3 * 128 + 1, 9)]),
    (dict(k_scheme=NUQ, k_bits=3, k_outliers=2, v_scheme=NUQ, v_bits=3, v_outliers=2), 2,
     [(1, 2 * 128 + 3, 0), (0, 128 + 60, 20)]),                                       # CUDA-core path
])
def test_merged_parts_match_the_oracle_over_the_union(kw, G, spans):
    B, H, D = 2, 3, 128
    parts = _parts(kw, B, H, G, spans, seed=300)
    q = vals(399, (B, G * H, D), BF16)
    qd = dev(q, BF16)
    scale = 1.0 / np.sqrt(D)
    outs, lses = [], []
    for p, tq, tr in parts:
        o, l = seqsplit.decode_local(p.fmt, p.gpu, qd, tq, tr, scale, status=p.status)
        outs.append(o)
        lses.append(l)
        assert p.status_bits() == 0
    merged = kvq.merge_states(torch.stack(outs), torch.stack(lses), kvq.F32)
    torch.cuda.synchronize()
    # the oracle over the union: every part's reconstructed tokens, concatenated
    ref = np.zeros((B, G * H, D))
    ref_lse = np.zeros((B, G * H))
    for b in range(B):
        for h in range(H):
            Ks, Vs = [], []
            for p, tq, tr in parts:
                K, V = oatt.kv_slab(p.of, p.ora, b, h, tq, tr)
                Ks.append(K)
                Vs.append(V)
            o, l = oatt.attention_lse(q[b, h * G:(h + 1) * G].astype(np.float64), np.concatenate(Ks),
                                      np.concatenate(Vs), scale)
            ref[b, h * G:(h + 1) * G] = o
            ref_lse[b, h * G:(h + 1) * G] = l
    assert_attn(merged.cpu().numpy(), ref, 1e-3)
    lse_all = torch.empty((B, G * H), dtype=torch.float32, device="cuda")
    kvq.merge_states(torch.stack(outs), torch.stack(lses), kvq.F32, lse_out=lse_all)
    torch.cuda.synchronize()
    assert np.abs(lse_all.cpu().numpy() - ref_lse).max() <= 1e-3 * max(1.0, np.abs(ref_lse).max())


def test_one_part_merges_to_the_plain_decode():
    B, H, G, D = 2, 2, 4, 128
    (p, tq, tr), = _parts(dict(), B, H, G, [(1, 2 * 128 + 11, 7)], seed=500)
    qd = dev(vals(501, (B, G * H, D), BF16), BF16)
    scale = 1.0 / np.sqrt(D)
    plain = kvq.decode_attention(p.fmt, p.gpu, qd, tq, tr, scale, kvq.F32)
    o, l = seqsplit.decode_local(p.fmt, p.gpu, qd, tq, tr, scale)
    merged = kvq.merge_states(o[None].contiguous(), l[None].contiguous(), kvq.F32)
    torch.cuda.synchronize()
    assert torch.equal(o, plain)
    assert torch.equal(merged, plain)
    assert torch.isfinite(l).all()


def test_empty_part_has_no_weight_and_16_bit_output():
    # a part whose lse is -inf (no tokens) contributes nothing; bf16 output rounds once
    B, H, G, D = 1, 2, 2, 64
    rows = B * G * H
    rng = np.random.default_rng(3)
    outs = torch.tensor(rng.standard_normal((3, rows, D)), dtype=torch.float32, device="cuda")
    lses = torch.tensor(rng.standard_normal((3, rows)), dtype=torch.float32, device="cuda")
    lses[1] = -float("inf")
    outs[1] = float("nan")   # never read with weight: must not leak
    got = kvq.merge_states(outs, lses, kvq.BF16)
    torch.cuda.synchronize()
    o, l = outs.cpu().numpy().astype(np.float64), lses.cpu().numpy().astype(np.float64)
    w0, w2 = np.exp(l[0] - np.maximum(l[0], l[2])), np.exp(l[2] - np.maximum(l[0], l[2]))
    want = (w0[:, None] * o[0] + w2[:, None] * o[2]) / (w0 + w2)[:, None]
    assert np.abs(got.float().cpu().numpy() - want).max() <= 2 ** -7 * np.abs(want).max()


def test_rows_without_tokens_merge_to_zero():
    # every part of rows 1 and 4 is empty (lse = -inf): out = 0 there and lse = -inf,
    # the other rows as the oracle's merge
    from oracle.attention import merge_parts
    rows, D = 6, 128
    rng = np.random.default_rng(5)
    outs = rng.standard_normal((2, rows, D)).astype(np.float32)
    lses = rng.standard_normal((2, rows)).astype(np.float32)
    lses[:, [1, 4]] = -np.inf
    outs[:, [1, 4]] = np.nan
    lse_out = torch.empty(rows, dtype=torch.float32, device="cuda")
    got = kvq.merge_states(torch.tensor(outs, device="cuda"), torch.tensor(lses, device="cuda"), kvq.F32,
                           lse_out=lse_out)
    torch.cuda.synchronize()
    want, want_lse = merge_parts(outs, lses)
    g, gl = got.cpu().numpy(), lse_out.cpu().numpy()
    assert np.all(g[[1, 4]] == 0.0) and np.all(np.isneginf(gl[[1, 4]]))
    live = [0, 2, 3, 5]
    assert np.abs(g[live] - want[live]).max() <= 1e-6 * np.abs(want[live]).max()
    assert np.abs(gl[live] - want_lse[live]).max() <= 1e-6 * max(1.0, np.abs(want_lse[live]).max())
