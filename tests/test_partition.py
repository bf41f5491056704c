"""Host logic of the tensor-core decode plan, on CPU (no GPU: the library plans for the
148 SMs of the part when no device is visible).

An independent model of the item partition -- each KV head a row of positions (two
per raw item of 8 tokens, one per packed half group), the rows cut into one equal
contiguous range per warp, 12 warps per CTA -- is checked exhaustively for what the
kernel and the combine rely on:
  * every position belongs to exactly one warp, and no range touches more than two heads;
  * the slots a head's combine reads (slot 0 when a range crosses out of the head, then
    one per CTA whose warps end inside the head) are each written by exactly one writer,
    and every state the kernel writes is read;
and the slot count the library plans (kvq_decode_partial_slots) equals the model's."""
import math

import pytest

import synth
from quantized_decode_attention_quantize_b200 import kvq

KCW = 12
SMS = 148


def positions_per_head(tq, nraw, esz):
    rt = 2048 // (128 * esz)
    nrp = 2 * math.ceil(nraw / rt)
    ngv = math.ceil(tq / 128)
    rem = tq - (ngv - 1) * 128
    return nrp + 2 * (ngv - 1) + (2 if rem > 64 else 1)


def model(heads, U, max_ctas):
    I = heads * U
    cap = min(SMS, max_ctas) if max_ctas > 0 else SMS
    grid = max(min(cap, math.ceil(I / KCW)), math.ceil(heads / KCW), 1)
    W = grid * KCW
    start = [gw * I // W for gw in range(W + 1)]
    writes = {}                       # (head, slot) -> writer
    owner = [None] * I
    for gw in range(W):
        i0, i1 = start[gw], start[gw + 1]
        assert i1 - i0 <= U
        for i in range(i0, i1):
            assert owner[i] is None
            owner[i] = gw
        hs = sorted({i // U for i in range(i0, i1)})
        assert len(hs) <= 2
        if len(hs) == 2:              # the state of the first head leaves through slot 0
            assert (hs[0], 0) not in writes
            writes[(hs[0], 0)] = ("warp", gw)
        last = (i1 - 1) // U if i1 > 0 else -1
        if last >= 0:                 # merged per CTA into slot 1 + CTA - first CTA ending in the head
            first_end = min(w for w in range(W) if start[w + 1] >= last * U + 1)
            slot = 1 + gw // KCW - first_end // KCW
            prev = writes.setdefault((last, slot), ("cta", gw // KCW))
            assert prev == ("cta", gw // KCW)
    assert all(o is not None for o in owner)
    # what the combine reads
    span = 1
    for h in range(heads):
        ending = [w for w in range(W) if h * U + 1 <= start[w + 1] <= (h + 1) * U]
        ca, cb = ending[0] // KCW, ending[-1] // KCW
        span = max(span, cb - ca + 1)
        holder = max(w for w in range(W) if start[w] <= (h + 1) * U - 1)
        crossing = start[holder + 1] > (h + 1) * U
        read = ([0] if crossing else []) + list(range(1, 2 + cb - ca))
        for s in read:
            assert (h, s) in writes, (h, s)
        written = sorted(s for (hh, s) in writes if hh == h)
        assert written == read, (h, written, read)
    return 1 + span


SHAPES = [
    # B, Hkv, G, tq, n_sink, tr, num_splits, src
    (8, 8, 4, 32639, 1, 128, 0, synth.BF16),
    (1, 32, 1, 4096, 0, 0, 0, synth.F16),
    (2, 3, 4, 2 * 128 + 40, 1, 21, 0, synth.BF16),
    (3, 5, 2, 2 * 128 + 1, 2, 3, 13, synth.BF16),
    (2, 3, 8, 5, 1, 0, 4, synth.BF16),
    (1, 7, 4, 9 * 128, 0, 100, 0, synth.BF16),
    (2, 2, 4, 300, 1, 20, 0, synth.F32),
    (5, 3, 2, 7 * 128 + 64, 1, 100, 1, synth.BF16),
    (2, 3, 4, 64, 1, 13, 0, synth.BF16),
    (2, 3, 4, 65, 1, 13, 3, synth.BF16),
    (1, 1, 1, 1, 0, 0, 0, synth.F16),
    (16, 120, 2, 70, 1, 3, 0, synth.BF16),
]


MIXED_SHAPES = [
    # MixKVQ tiers (8 / 24 / 96) on bf16: the tensor-core plan too
    (16, 8, 5, 16384, 0, 0, 0, synth.BF16),
    (1, 2, 5, 4096, 0, 0, 1, synth.BF16),
    (2, 3, 4, 3 * 128 + 45, 1, 29, 3, synth.BF16),
]


def flag_bytes(B, Hkv):
    """The tensor-core path's workspace ends with 32 flags (4 bytes each) per KV head, 16-byte
    aligned, for the append that its split kernel can take over."""
    return (B * Hkv * 32 * 4 + 15) // 16 * 16


@pytest.mark.parametrize("B,Hkv,G,tq,ns,tr,splits,src", MIXED_SHAPES)
def test_mixed_tiers_plan_like_k4v2(B, Hkv, G, tq, ns, tr, splits, src):
    # every host planning helper sees the tiers: the slot count, the workspace of the
    # split kernel and the combine agree with the tensor-core partition
    fd = synth._fmt(src_dtype=src, k_scheme=synth.MIXED, k_bits=0, mixed_hi=8, mixed_mid=24,
                    n_sink=ns, residual_cap=max(tr, 1))
    f = kvq.make_format(fd)
    U = positions_per_head(tq, ns + tr, 2)
    want = model(B * Hkv, U, splits)
    assert kvq.decode_partial_slots(f, B, G * Hkv, Hkv, tq, tr, splits) == want
    rows = B * G * Hkv * want
    assert kvq.decode_workspace_bytes(f, B, G * Hkv, Hkv, tq, tr, splits) == \
        2 * ((rows * 4 + 15) // 16 * 16) + rows * 128 * 4 + flag_bytes(B, Hkv)


@pytest.mark.parametrize("B,Hkv,G,tq,ns,tr,splits,src", SHAPES)
def test_planned_slots_match_the_partition_model(B, Hkv, G, tq, ns, tr, splits, src):
    fd = synth._fmt(src_dtype=src, n_sink=ns, residual_cap=max(tr, 1))
    f = kvq.make_format(fd)
    esz = 4 if src == synth.F32 else 2
    U = positions_per_head(tq, ns + tr, esz)
    want = model(B * Hkv, U, splits)
    assert kvq.decode_partial_slots(f, B, G * Hkv, Hkv, tq, tr, splits) == want
    rows = B * G * Hkv * want
    assert kvq.decode_workspace_bytes(f, B, G * Hkv, Hkv, tq, tr, splits) == \
        2 * ((rows * 4 + 15) // 16 * 16) + rows * 128 * 4 + flag_bytes(B, Hkv)
