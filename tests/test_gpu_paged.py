"""GPU parity of the paged cache with per-sequence lengths (kvq_quantize_kv_paged,
kvq_decode_attention_paged) against oracle.paged: every pool byte the appends write
equals the oracle's, and every sequence's decode output matches the float64 attention
over that sequence's own tokens.  Lengths hit ragged groups, single tokens, sequences of
sink tokens only, and (without a sink) sequences with no tokens at all."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import paged as opaged
from oracle.formats import BF16, F16, F32, KEYS, VALUES, Format
from quantized_decode_attention_quantize_b200 import kvq
from tests.gpu_util import TORCH, assert_attn, dev, raw_bits, tolerance

pytestmark = pytest.mark.gpu
D, g = 128, 128


def fmt(**kw):
    return synth._fmt(**kw)


def vals(rng, shape, dt, scale=1.0, heavy=False, outlier_cols=()):
    """Exact source values: scaled, outlier channels x10, then rounded to the source type."""
    x = (rng.standard_t(4, shape) if heavy else rng.standard_normal(shape)) * scale
    x[..., list(outlier_cols)] *= 10.0
    return synth.to_dtype_values(x.astype(np.float32), dt)


def build(fd, H, t_quant, t_res, num_blocks, seed):
    """Both paged caches filled group by group, each sequence's groups in shuffled blocks."""
    rng = np.random.default_rng(seed)
    S = len(t_quant)
    dt = fd["src_dtype"]
    max_blocks = max(1, max(-(-t // g) for t in t_quant))
    f = kvq.make_format(fd)
    gpu = kvq.PagedCache(f, H, num_blocks, S, max_blocks)
    ora = opaged.PagedCache(Format(**fd), H, num_blocks, S, max_blocks)
    free = list(rng.permutation(num_blocks))
    table = np.full((S, max_blocks), -1, np.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for s in range(S):
        for gi in range(-(-t_quant[s] // g)):
            n = min(g, t_quant[s] - gi * g)
            blk = int(free.pop())
            table[s, gi] = blk
            K = vals(rng, (H, n, D), dt, heavy=True, outlier_cols=rng.choice(D, 3, replace=False))
            V = vals(rng, (H, n, D), dt)
            # one sequence's append: a one-sequence view of the same pool
            view = kvq.kvq_paged_cache(pool=gpu.pool.struct, num_seqs=1, max_blocks=max_blocks,
                                       block_table=gpu.block_table.data_ptr())
            kt, vt = dev(K[None], dt), dev(V[None], dt)
            st = kvq.lib().kvq_quantize_kv_paged(ctypes.byref(f), ctypes.byref(view), kvq._ptr(kt), kvq._ptr(vt),
                                                 kt.stride(0), kt.stride(1), kt.stride(2),
                                                 kvq._ptr(torch.tensor([blk], dtype=torch.int32, device="cuda")), n,
                                                 kvq._ptr(status), None)
            assert st == kvq.KVQ_OK
            opaged.quantize_group(ora, KEYS, K, blk, n)
            opaged.quantize_group(ora, VALUES, V, blk, n)
    gpu.block_table.copy_(torch.from_numpy(table))
    ora.block_table[...] = table
    for name, rows in (("sink_k", fd["n_sink"]), ("sink_v", fd["n_sink"]),
                       ("res_k", fd["residual_cap"]), ("res_v", fd["residual_cap"])):
        if rows:
            x = vals(rng, (S, H, rows, D), dt, heavy=name == "res_k")
            bits = raw_bits(x, dt)
            ora.raw[name][...] = bits
            gpu.raw[name].copy_(torch.from_numpy(np.ascontiguousarray(bits).reshape(-1).view(np.uint8)).cuda())
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return gpu, ora, table


def check_pool(gpu, ora, table):
    # every written block's bytes, array by array
    used = sorted({int(b) for b in table.reshape(-1) if b >= 0})
    for name in ("k_codes", "k_scale", "k_zero", "v_codes", "v_scale", "v_zero"):
        got = gpu.pool.tensors[name].view(gpu.num_blocks, -1).cpu().numpy()
        want = np.ascontiguousarray(ora.pool[name]).reshape(ora.num_blocks, -1).view(np.uint8)
        for b in used:
            if not np.array_equal(got[b], want[b]):
                bad = np.nonzero(got[b] != want[b])[0]
                raise AssertionError(f"{name} block {b}: {bad.size} bytes differ, first at {bad[:8]}")


def run(gpu, ora, fd, t_quant, t_res, G, q_dtype, out_dtype, seed):
    rng = np.random.default_rng(seed + 1)
    S, H = len(t_quant), gpu.H
    q = vals(rng, (S, G * H, D), q_dtype)
    tq = torch.tensor(t_quant, dtype=torch.int32, device="cuda")
    tr = torch.tensor(t_res, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.decode_attention_paged(gpu.fmt, gpu, tq, tr, max(t_quant), max(t_res), dev(q, q_dtype),
                                     1.0 / np.sqrt(D), out_dtype, status=status)
    torch.cuda.synchronize()
    ref = opaged.decode_attention(ora, q.astype(np.float64), t_quant, t_res)
    return out.float().cpu().numpy(), ref, int(status.item())


@pytest.mark.parametrize("G,src,out_dtype", [(4, BF16, F32), (1, F16, BF16), (2, BF16, F32)])
def test_paged_mixed_lengths(G, src, out_dtype):
    fd = fmt(src_dtype=src, n_sink=1, residual_cap=64)
    t_quant = [1000, 1, 0, 64, 65, 128, 129, 3 * 128 + 7]
    t_res = [5, 0, 0, 64, 1, 63, 0, 17]
    H = 2
    gpu, ora, table = build(fd, H, t_quant, t_res, num_blocks=40, seed=200 + G)
    check_pool(gpu, ora, table)
    out, ref, st = run(gpu, ora, fd, t_quant, t_res, G, src, out_dtype, 300 + G)
    assert st == 0
    for s in range(len(t_quant)):   # each sequence on its own
        assert_attn(out[s], ref[s], tolerance(out_dtype), out_dtype)


def test_paged_without_sink_and_empty_sequences():
    fd = fmt(src_dtype=BF16, n_sink=0, residual_cap=16)
    t_quant = [0, 200, 0, 7]
    t_res = [0, 3, 9, 0]          # sequence 0 has no tokens at all
    gpu, ora, table = build(fd, 3, t_quant, t_res, num_blocks=8, seed=210)
    out, ref, st = run(gpu, ora, fd, t_quant, t_res, 4, BF16, F32, 310)
    assert st == 0
    assert np.all(out[0] == 0.0) and np.all(ref[0] == 0.0)
    for s in range(1, 4):
        assert_attn(out[s], ref[s], tolerance(F32))


def test_paged_rotated_keys():
    fd = fmt(src_dtype=BF16, n_sink=1, residual_cap=32, k_rotate=1)
    t_quant = [500, 130, 3]
    t_res = [31, 0, 2]
    gpu, ora, table = build(fd, 2, t_quant, t_res, num_blocks=9, seed=220)
    check_pool(gpu, ora, table)
    out, ref, st = run(gpu, ora, fd, t_quant, t_res, 4, BF16, F32, 320)
    assert st == 0
    for s in range(3):
        assert_attn(out[s], ref[s], tolerance(F32))


def test_paged_long_sequence_spans_chunks():
    # a sequence of many groups next to short ones: several chunks of one sequence merged
    fd = fmt(src_dtype=BF16, n_sink=1, residual_cap=128)
    t_quant = [40 * 128 + 33, 2, 260]
    t_res = [128, 1, 0]
    gpu, ora, table = build(fd, 2, t_quant, t_res, num_blocks=48, seed=230)
    out, ref, st = run(gpu, ora, fd, t_quant, t_res, 4, BF16, F32, 330)
    assert st == 0
    for s in range(3):
        assert_attn(out[s], ref[s], tolerance(F32))


@pytest.mark.parametrize("S,H,tq_max,seed", [(300, 8, 200, 250), (20, 2, 10, 260)])
def test_paged_many_short_sequences(S, H, tq_max, seed):
    # many short rows next to one of the longest: most chunks past a sequence's end are
    # empty, and (20 sequences of a few tokens) most sequences take a single chunk
    rng = np.random.default_rng(seed)
    fd = fmt(src_dtype=BF16, n_sink=1, residual_cap=16)
    t_quant = [int(x) for x in rng.integers(0, tq_max + 1, S)]
    t_res = [int(x) for x in rng.integers(0, 17, S)]
    t_quant[0], t_res[0] = tq_max, 16
    gpu, ora, table = build(fd, H, t_quant, t_res, num_blocks=sum(-(-t // g) for t in t_quant) + 2, seed=seed)
    out, ref, st = run(gpu, ora, fd, t_quant, t_res, 4, BF16, F32, seed + 1)
    assert st == 0
    for s in range(S):
        assert_attn(out[s], ref[s], tolerance(F32))


def test_paged_bounds_are_flagged_not_followed():
    # a block id outside the pool and a length past its bound: KVQ_DEV_BOUNDS, no fault;
    # the other sequences' outputs are unaffected
    fd = fmt(src_dtype=BF16, n_sink=1, residual_cap=16)
    t_quant = [300, 100]
    t_res = [3, 2]
    gpu, ora, table = build(fd, 2, t_quant, t_res, num_blocks=6, seed=240)
    bad = table.copy()
    bad[1, 0] = 1000                      # out of range: read from block 0 and flagged
    gpu.block_table.copy_(torch.from_numpy(bad))
    out, ref, st = run(gpu, ora, fd, t_quant, t_res, 4, BF16, F32, 340)
    assert st & kvq.KVQ_DEV_BOUNDS
    assert_attn(out[0], ref[0], tolerance(F32))
    gpu.block_table.copy_(torch.from_numpy(table))
    # a device length above the bound the launch was sized for: clamped and flagged
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = dev(vals(np.random.default_rng(5), (2, 8, D), BF16), BF16)
    tq = torch.tensor([300, 100], dtype=torch.int32, device="cuda")
    tr = torch.tensor([3, 99], dtype=torch.int32, device="cuda")   # 99 > max_t_res = 3
    kvq.decode_attention_paged(gpu.fmt, gpu, tq, tr, 300, 3, q, 0.1, F32, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & kvq.KVQ_DEV_BOUNDS
    # an append to a block id outside the pool: flagged, nothing written
    before = gpu.pool.tensors["k_codes"].clone()
    src = dev(vals(np.random.default_rng(6), (2, 2, 16, D), BF16), BF16)
    status.zero_()
    kvq.quantize_kv_paged(gpu.fmt, gpu, src, src, torch.tensor([-1, 7], dtype=torch.int32, device="cuda"), 16,
                          status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & kvq.KVQ_DEV_BOUNDS
    assert torch.equal(before, gpu.pool.tensors["k_codes"])
