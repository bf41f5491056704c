"""Full-size parity: every workload at its full shape, run the way the benchmark runs
it (one quantize call over all packed tokens, the flush of one group -- or the
256-token append of the MixKVQ workload -- then decode_partial + decode_combine with
the planned split and the planned workspace).  The bulk of each cache comes from the
device generator; a few sampled (batch, KV-head) slabs are overwritten with the host
generator's values, and the oracle recomputes exactly those slabs on its own: every
byte of their packed arrays must match, and the outputs of their query heads must be
within the attention tolerance."""
import json
import os

import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from oracle import cache as ocache
from oracle import salience as osal
from oracle.formats import F32, KEYS, MIXED, NUQ, VALUES, Format
from quantized_decode_attention_quantize_b200 import kvq
from tests.gpu_util import TORCH, rel_l2, rel_l2_rows, tolerance

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LUT = json.load(open(os.path.join(ROOT, "tests", "golden", "nuq3_codebook.json")))

# (workload, sampled (b, kv-head) slabs): first, last and one in between
CASES = [
    ("llama2_7b", [(0, 0), (0, 31)]),
    ("llama3_8b", [(0, 0), (3, 5), (7, 7)]),
    ("mixkvq_14b", [(0, 0), (15, 7)]),
    ("kvquant_nuq3", [(0, 17)]),
    ("llama3_8b_wht", [(0, 0), (7, 7)]),
]


def _host(x, like):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=like.device, dtype=like.dtype)


def _oracle_slab(cfg, of, K, V, qwin, luts):
    """The oracle's cache of one slab (B = H = 1) built from that slab's host values."""
    ns, tq, tr = synth.split_tokens(cfg)
    g = of.group_tokens
    c = ocache.Cache(of, 1, 1, -(-tq // g) * g, k_lut=luts[0], v_lut=luts[1])
    K64, V64 = K.astype(np.float64), V.astype(np.float64)
    if of.k_scheme == MIXED:
        for gi in range(-(-tq // g)):
            t0, ln = gi * g, min(g, tq - gi * g)
            c["k_order"][0, 0, gi] = osal.key_salience(qwin[:, t0:t0 + ln],
                                                       K64[ns + t0:ns + t0 + ln])[1]
    ocache.quantize(of, c, KEYS, K64[None, None, ns:ns + tq], 0, tq)
    ocache.quantize(of, c, VALUES, V64[None, None, ns:ns + tq], 0, tq)
    if ns:
        c["sink_k"][0, 0] = ocache.raw_encode(K64[:ns], of.src_dtype)
        c["sink_v"][0, 0] = ocache.raw_encode(V64[:ns], of.src_dtype)
    if tr:
        c["res_k"][0, 0, :tr] = ocache.raw_encode(K64[ns + tq:], of.src_dtype)
        c["res_v"][0, 0, :tr] = ocache.raw_encode(V64[ns + tq:], of.src_dtype)
    return c


@pytest.mark.timeout(1800)
@pytest.mark.parametrize("name,slabs", CASES, ids=[c[0] for c in CASES])
def test_full_size_workload(name, slabs):
    cfg = synth.CONFIGS[name]
    fd = cfg["fmt"]
    of = Format(**fd)
    fmt = kvq.make_format(fd)
    B, Hq, H, D, g = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["D"], fd["group_tokens"]
    G = Hq // H
    ns, tq, tr = synth.split_tokens(cfg)
    C = -(-tq // g) * g
    luts = (LUT["k"], LUT["v"]) if fd["k_scheme"] == NUQ else (None, None)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    K = synth.device_kv(cfg, "k")
    V = synth.device_kv(cfg, "v")
    host = {}
    for b, h in slabs:
        hk, hv = synth.kv_slab(cfg, b, h, which="k"), synth.kv_slab(cfg, b, h, which="v")
        K[b, h] = _host(hk, K)
        V[b, h] = _host(hv, V)
        host[(b, h)] = [hk, hv, None]

    cache = kvq.Cache(fmt, B, H, C, k_lut=luts[0], v_lut=luts[1])
    if fd["k_scheme"] == MIXED:
        # salience windows: the query rows at the group's positions
        gen = torch.Generator(device="cuda")
        gen.manual_seed(cfg["seed"] * 1000 + 44)
        mu = torch.exp(torch.empty((1, Hq, 1, D), device="cuda").uniform_(
            np.log(0.1), np.log(5.0), generator=gen))
        Qw = (torch.randn((B, Hq, tq, D), device="cuda", generator=gen) * mu).to(K.dtype)
        for b, h in slabs:
            qw = np.stack([np.concatenate([synth.query_window(cfg, b, hq, t0, min(g, tq - t0))
                                           for t0 in range(0, tq, g)])
                           for hq in range(h * G, (h + 1) * G)])
            Qw[b, h * G:(h + 1) * G] = _host(qw, Qw)
            host[(b, h)][2] = qw
        order = cache.array("k_order")
        ng = C // g
        for gi in range(-(-tq // g)):
            t0, ln = gi * g, min(g, tq - gi * g)
            kvq.key_salience(fmt, Qw[:, :, t0:t0 + ln], K[:, :, ns + t0:ns + t0 + ln], order[gi * D:],
                             H * ng * D, ng * D, status=status)
        del Qw

    # bulk build, then the step's own quantize launch over its tokens
    kvq.quantize_keys(fmt, cache, K[:, :, ns:ns + tq], 0, tq, status=status)
    kvq.quantize_values(fmt, cache, V[:, :, ns:ns + tq], 0, tq, status=status)
    n_app = cfg.get("append", g)
    a0 = (tq // g) * g - n_app
    kvq.quantize_keys(fmt, cache, K[:, :, ns + a0:ns + a0 + n_app].contiguous(), a0, n_app, status=status)
    kvq.quantize_values(fmt, cache, V[:, :, ns + a0:ns + a0 + n_app].contiguous(), a0, n_app,
                        status=status)
    if ns:
        cache.array("sink_k").copy_(K[:, :, :ns].contiguous().view(-1).view(torch.uint8))
        cache.array("sink_v").copy_(V[:, :, :ns].contiguous().view(-1).view(torch.uint8))
    if tr:
        cache.array("res_k").copy_(K[:, :, ns + tq:].contiguous().view(-1).view(torch.uint8))
        cache.array("res_v").copy_(V[:, :, ns + tq:].contiguous().view(-1).view(torch.uint8))
    del K, V

    q = synth.device_queries(cfg)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(16, kvq.decode_workspace_bytes(fmt, B, Hq, H, tq, tr)), dtype=torch.uint8,
                     device="cuda")
    scale = 1.0 / float(np.sqrt(D))
    kvq.decode_partial(fmt, cache, q, tq, tr, scale, ws, status=status)
    kvq.decode_combine(fmt, B, Hq, H, tq, tr, ws, out)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got_out = out.cpu().numpy()

    for (b, h), (hk, hv, qw) in host.items():
        c = _oracle_slab(cfg, of, hk, hv, qw, luts)
        for n, arr in c.arrays.items():
            if n in ("k_lut", "v_lut"):
                continue
            got = cache.array(n).view(B * H, -1)[b * H + h].cpu().numpy()
            want = np.ascontiguousarray(arr).reshape(-1).view(np.uint8)
            if not np.array_equal(got, want):
                bad = np.nonzero(got != want)[0]
                raise AssertionError(f"{name} slab {(b, h)} {n}: {bad.size} bytes differ, first at {bad[:8]}")
        qh = np.stack([synth.query(cfg, b, hq) for hq in range(h * G, (h + 1) * G)])
        ref = oatt.decode_attention(of, c, qh[None].astype(np.float64), tq, tr)[0]
        err = rel_l2(got_out[b, h * G:(h + 1) * G], ref)
        worst = rel_l2_rows(got_out[b, h * G:(h + 1) * G], ref)
        assert err <= tolerance(F32) and worst <= tolerance(F32), (name, (b, h), err, worst)
