"""Host-side checks of libkvq.so that need no GPU: it loads, exports every function
include/kvq.h declares, sizes cache arrays exactly as the oracle's independent byte
accounting does, and rejects bad arguments before anything is launched."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
from oracle import formats as of
from quantized_decode_attention_quantize_b200 import kvq


def torch_cuda_available():
    import torch
    return torch.cuda.is_available()

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    names = _declared_functions()
    assert len(names) >= 9
    lib = kvq.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert lib.kvq_version() == (0 << 16) | 2


def test_status_strings():
    for s in range(5):
        assert kvq.status_string(s)
    assert kvq.status_string(99) == "unknown status"


# (KQV array sizes are checked in test_kqv_host.py: oracle.formats states the other schemes)
ALL_FORMATS = [c["fmt"] for c in synth.CONFIGS.values() if c["fmt"]["k_scheme"] != synth.KQV] + [
    synth.toy_format(s, t, N) for s in ("tensor", "token", "hybrid")
    for t in ("both", "k_only", "v_only") for N in (64, 256)]


@pytest.mark.parametrize("fd", ALL_FORMATS)
def test_array_bytes_match_oracle(fd):
    f = kvq.make_format(fd)
    assert kvq.format_check(f) == kvq.KVQ_OK
    o = of.Format(**fd)
    for B, H, C in ((1, 1, fd["group_tokens"]), (2, 3, 4 * fd["group_tokens"])):
        for i, name in enumerate(kvq.ARRAYS):
            assert kvq.cache_array_bytes(f, B, H, C, i) == of.array_bytes(o, B, H, C, name), name


def test_page_byte_table_through_the_library():
    # [AXES] "Scales occupy bytes too", N = 64 / 256, D = 32
    for N, want in ((64, (4104, 4608, 4480)), (256, (16392, 18432, 17536))):
        for scheme, w in zip(("tensor", "token", "hybrid"), want):
            f = kvq.make_format(synth.toy_format(scheme, "both", N))
            tot = sum(kvq.cache_array_bytes(f, 1, 1, N, i) for i in range(len(kvq.ARRAYS)))
            assert tot == w


def _fmt(**kw):
    d = dict(synth.CONFIGS["llama2_7b"]["fmt"])
    d.update(kw)
    return kvq.make_format(d)


@pytest.mark.parametrize("kw,want", [
    (dict(head_dim=96), kvq.KVQ_ERR_INVALID),
    (dict(group_tokens=24), kvq.KVQ_ERR_INVALID),
    (dict(group_tokens=512), kvq.KVQ_ERR_INVALID),
    (dict(src_dtype=7), kvq.KVQ_ERR_INVALID),
    (dict(k_bits=3), kvq.KVQ_ERR_INVALID),
    (dict(k_axis=kvq.TOKEN), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(v_axis=kvq.CHANNEL), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(v_scheme=kvq.MIXED), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(k_scheme=kvq.MIXED, mixed_hi=4, mixed_mid=24), kvq.KVQ_ERR_INVALID),
    (dict(k_scheme=kvq.NUQ, k_bits=3, k_outliers=9), kvq.KVQ_ERR_INVALID),
    (dict(rope=1, rope_base=0.5), kvq.KVQ_ERR_INVALID),
    (dict(head_dim=32, group_tokens=64, rope=1), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(k_rotate=2), kvq.KVQ_ERR_INVALID),
    (dict(k_rotate=1, rope=1), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(k_rotate=1, k_scheme=kvq.MIXED, mixed_hi=8, mixed_mid=24), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(k_rotate=1, k_scheme=kvq.NONE, k_bits=0), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(k_rotate=1), kvq.KVQ_OK),
    (dict(k_rotate=1, k_scheme=kvq.NUQ, k_bits=3, k_outliers=2), kvq.KVQ_OK),
    (dict(k_rotate=1, k_scheme=kvq.SYM8, k_bits=8, k_axis=kvq.TOKEN), kvq.KVQ_OK),
    (dict(), kvq.KVQ_OK),
])
def test_format_check(kw, want):
    assert kvq.format_check(_fmt(**kw)) == want


class _FakeCache:
    """A cache struct with well-aligned dummy addresses (never dereferenced: every
    call below fails validation on the host)."""

    def __init__(self, B=1, H=1, C=128):
        self.struct = kvq.kvq_cache(batch=B, kv_heads=H, capacity=C)
        for i, n in enumerate(kvq.ARRAYS):
            setattr(self.struct, n, 0x10000 * (i + 1))

    def ref(self):
        return ctypes.byref(self.struct)


# The tests below hand made-up device addresses to launching entry points, relying on
# the host checks to refuse them before any launch.  They run where no GPU is present;
# on a GPU machine a regressed check would launch kernels on those addresses.
fake_pointers = pytest.mark.skipif(torch_cuda_available(), reason="made-up device addresses; CPU only")


@fake_pointers
def test_host_validation_rejects_before_launch():
    L = kvq.lib()
    f = _fmt()
    c = _FakeCache()
    src = ctypes.c_void_p(0x100000)
    # t0 not a multiple of the group, n past capacity, misaligned source, bad strides
    assert L.kvq_quantize_keys(ctypes.byref(f), c.ref(), src, 0, 0, 128, 64, 8, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_quantize_keys(ctypes.byref(f), c.ref(), src, 0, 0, 128, 0, 129, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_quantize_keys(ctypes.byref(f), c.ref(), ctypes.c_void_p(0x100002), 0, 0, 128, 0, 8, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_quantize_keys(ctypes.byref(f), c.ref(), src, 0, 0, 100, 0, 8, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_quantize_values(ctypes.byref(f), c.ref(), None, 0, 0, 128, 0, 8, None, None) == kvq.KVQ_ERR_INVALID
    # zero tokens is a no-op
    assert L.kvq_quantize_values(ctypes.byref(f), c.ref(), src, 0, 0, 128, 0, 0, None, None) == kvq.KVQ_OK
    # capacity not a multiple of the group
    bad = _FakeCache(C=100)
    assert L.kvq_quantize_keys(ctypes.byref(f), bad.ref(), src, 0, 0, 128, 0, 8, None, None) == kvq.KVQ_ERR_INVALID
    # a missing array
    nul = _FakeCache()
    nul.struct.k_scale = None
    assert L.kvq_quantize_keys(ctypes.byref(f), nul.ref(), src, 0, 0, 128, 0, 8, None, None) == kvq.KVQ_ERR_INVALID
    # dequantize: bad which, range, dtype
    out = ctypes.c_void_p(0x200000)
    assert L.kvq_dequantize(ctypes.byref(f), c.ref(), 2, 0, 8, out, kvq.F32, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_dequantize(ctypes.byref(f), c.ref(), 0, 120, 9, out, kvq.F32, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_dequantize(ctypes.byref(f), c.ref(), 0, 0, 8, out, 5, None, None) == kvq.KVQ_ERR_INVALID
    # decode: heads not a multiple, too many residual tokens, empty cache, tiny workspace
    q = ctypes.c_void_p(0x300000)
    ws = ctypes.c_void_p(0x400000)
    c = _FakeCache(H=2)
    assert L.kvq_decode_attention(ctypes.byref(f), c.ref(), q, kvq.F16, 3, 64, 0, 0.1, out, kvq.F32, ws, 1 << 20, 0, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_decode_attention(ctypes.byref(f), c.ref(), q, kvq.F16, 2, 64, 1, 0.1, out, kvq.F32, ws, 1 << 20, 0, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_decode_attention(ctypes.byref(f), c.ref(), q, kvq.F16, 2, 0, 0, 0.1, out, kvq.F32, ws, 1 << 20, 0, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_decode_attention(ctypes.byref(f), c.ref(), q, kvq.F16, 2, 64, 0, 0.1, out, kvq.F32, ws, 4, 2, None, None) == kvq.KVQ_ERR_WORKSPACE
    assert L.kvq_decode_attention(ctypes.byref(f), c.ref(), q, kvq.F16, 2, 200, 0, 0.1, out, kvq.F32, ws, 1 << 20, 2, None, None) == kvq.KVQ_ERR_INVALID
    # salience: heads not a multiple
    assert L.kvq_key_salience(ctypes.byref(f), q, 0, 0, 128, q, 0, 0, 128, 1, 3, 2, 4, None, out, 0, 0, None, None) == kvq.KVQ_ERR_INVALID


def test_workspace_bytes_with_explicit_splits():
    f = _fmt(k_bits=8)   # 8-bit keys: the generic split-per-group-run path
    # slots: 4 packed splits, no raw tokens -> B*Hq*4 * (2 + D) floats (16-byte padded)
    n = kvq.decode_workspace_bytes(f, 1, 32, 32, 4096, 0, 4)
    rows = 32 * 4
    assert n == 2 * ((rows * 4 + 15) // 16 * 16) + rows * 128 * 4


@fake_pointers
def test_sequence_split_entry_points_validate_on_the_host():
    # nothing is launched: every call below fails validation before touching memory
    L = kvq.lib()
    f = _fmt()
    ws = ctypes.c_void_p(0x400000)
    out = ctypes.c_void_p(0x200000)
    lse = ctypes.c_void_p(0x500000)
    # combine_lse: missing or misaligned lse, too small a workspace
    assert L.kvq_decode_combine_lse(ctypes.byref(f), 1, 4, 1, 256, 0, 0, ws, 1 << 20, out, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_decode_combine_lse(ctypes.byref(f), 1, 4, 1, 256, 0, 0, ws, 1 << 20, out,
                                    ctypes.c_void_p(0x500004), None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_decode_combine_lse(ctypes.byref(f), 1, 4, 1, 256, 0, 0, ws, 4, out, lse, None) == kvq.KVQ_ERR_WORKSPACE
    # merge: part count, rows, head dim, dtype, alignment
    outs = ctypes.c_void_p(0x600000)
    lses = ctypes.c_void_p(0x700000)
    assert L.kvq_merge_states(0, 8, 128, outs, lses, out, kvq.F32, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_merge_states(5000, 8, 128, outs, lses, out, kvq.F32, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_merge_states(2, 0, 128, outs, lses, out, kvq.F32, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_merge_states(2, 8, 96, outs, lses, out, kvq.F32, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_merge_states(2, 8, 128, outs, lses, out, 9, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_merge_states(2, 8, 128, ctypes.c_void_p(0x600008), lses, out, kvq.F32, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_merge_states(2, 8, 128, outs, None, out, kvq.F32, None, None) == kvq.KVQ_ERR_INVALID


def test_noalloc_rejects_oversized_requests():
    # A workspace need above the library's fixed scratch is refused before anything runs.
    # Every cache array and the q / out pointers are null: the size check comes first, and
    # should it ever regress, the null pointers fail the host validation that follows
    # (KVQ_ERR_INVALID) instead of reaching a launch.
    fd = dict(head_dim=128, group_tokens=128, src_dtype=of.BF16, k_scheme=of.ASYM, k_bits=4,
              k_axis=of.CHANNEL, k_outliers=0, v_scheme=of.ASYM, v_bits=2, v_axis=of.TOKEN,
              v_outliers=0, mixed_hi=0, mixed_mid=0, n_sink=0, residual_cap=0, rope=1,
              rope_base=10000.0, k_rotate=0)
    f = kvq.make_format(fd)              # RoPE keys: the generic path, 64 splits per head as asked
    B, Hq, Hkv, tq = 64, 64, 64, 131072
    need = kvq.decode_workspace_bytes(f, B, Hq, Hkv, tq, 0, 64)
    assert need > kvq.NOALLOC_SCRATCH_BYTES
    cache = kvq.kvq_cache(batch=B, kv_heads=Hkv, capacity=tq)
    st = kvq.lib().kvq_decode_attention_noalloc(ctypes.byref(f), ctypes.byref(cache), None, kvq.BF16, Hq,
                                                tq, 0, 0.1, None, kvq.F32, 64, None, None)
    assert st == kvq.KVQ_ERR_WORKSPACE


def test_paged_entry_points_validate_on_the_host():
    # null pools, tables and lengths are refused before anything runs (all pointers null)
    L = kvq.lib()
    f = _fmt(k_bits=4, v_bits=2)
    pc = kvq.kvq_paged_cache()
    pc.pool = kvq.kvq_cache(batch=4, kv_heads=2, capacity=128)
    pc.num_seqs, pc.max_blocks = 2, 3
    assert L.kvq_decode_attention_paged(ctypes.byref(f), ctypes.byref(pc), None, None, 256, 0, None, kvq.BF16, 8,
                                        0.1, None, kvq.F32, None, 0, None, None) == kvq.KVQ_ERR_INVALID
    assert L.kvq_quantize_kv_paged(ctypes.byref(f), ctypes.byref(pc), None, None, 0, 0, 128, None, 16, None,
                                   None) == kvq.KVQ_ERR_INVALID
    # workspace sizing: unsupported head groups and formats give 0
    assert L.kvq_decode_paged_workspace_bytes(ctypes.byref(f), 2, 16, 2, 256, 0) == 0     # G = 8
    assert L.kvq_decode_paged_workspace_bytes(ctypes.byref(f), 2, 8, 2, 256, 0) > 0
    f8 = _fmt(k_bits=8)
    assert L.kvq_decode_paged_workspace_bytes(ctypes.byref(f8), 2, 8, 2, 256, 0) == 0
