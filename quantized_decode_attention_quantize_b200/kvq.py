"""ctypes binding of libkvq.so (include/kvq.h).

Argument marshalling only: every entry point forwards to the C ABI with the same
name; device memory and streams come from PyTorch.  There is no fallback: when the
shared library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

# enums of include/kvq.h
KVQ_OK, KVQ_ERR_INVALID, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CUDA, KVQ_ERR_WORKSPACE = range(5)
KVQ_DEV_NONFINITE, KVQ_DEV_RANGE, KVQ_DEV_TIMEOUT, KVQ_DEV_BOUNDS = 1, 2, 4, 8
F32, F16, BF16 = 0, 1, 2
NONE, SYM8, ASYM, NUQ, MIXED, KQV = range(6)
TENSOR, TOKEN, CHANNEL = range(3)
KEYS, VALUES = 0, 1

ARRAYS = [
    "k_codes", "k_scale", "k_zero", "k_order",
    "k_out_rowptr", "k_out_col", "k_out_val",
    "v_codes", "v_scale", "v_zero",
    "v_out_col", "v_out_val",
    "k_lut", "v_lut",
    "sink_k", "sink_v", "res_k", "res_v",
    "v_sketch",
]

TORCH_DTYPE = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}
KVQ_DTYPE = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}


class kvq_format(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "head_dim", "group_tokens", "src_dtype",
        "k_scheme", "k_bits", "k_axis", "k_outliers",
        "v_scheme", "v_bits", "v_axis", "v_outliers",
        "mixed_hi", "mixed_mid", "n_sink", "residual_cap", "rope")] + [("rope_base", ctypes.c_float),
                                                                ("k_rotate", ctypes.c_int32)]


class kvq_cache(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("kv_heads", ctypes.c_int32),
                ("capacity", ctypes.c_int64)] + [(n, ctypes.c_void_p) for n in ARRAYS]


class kvq_paged_cache(ctypes.Structure):
    _fields_ = [("pool", kvq_cache), ("num_seqs", ctypes.c_int32), ("max_blocks", ctypes.c_int32),
                ("block_table", ctypes.c_void_p), ("sink_k", ctypes.c_void_p), ("sink_v", ctypes.c_void_p),
                ("res_k", ctypes.c_void_p), ("res_v", ctypes.c_void_p)]


class KvqError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn}: {status_string(status)} ({status})")
        self.status = status


_lib = None


def lib():
    """The loaded libkvq.so (raises when it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} not built; run python -m quantized_decode_attention_quantize_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        FP, CP = ctypes.POINTER(kvq_format), ctypes.POINTER(kvq_cache)
        PP = ctypes.POINTER(kvq_paged_cache)
        sig = {
            "kvq_version": (I32, []),
            "kvq_status_string": (ctypes.c_char_p, [I32]),
            "kvq_format_check": (I32, [FP]),
            "kvq_cache_array_bytes": (SZ, [FP, I32, I32, I64, I32]),
            "kvq_kqv_codebook": (I32, [I32, I32, ctypes.POINTER(ctypes.c_float)]),
            "kvq_quantize_keys": (I32, [FP, CP, P, I64, I64, I64, I64, I64, P, P]),
            "kvq_quantize_values": (I32, [FP, CP, P, I64, I64, I64, I64, I64, P, P]),
            "kvq_quantize_kv": (I32, [FP, CP, P, P, I64, I64, I64, I64, I64, P, P]),
            "kvq_dequantize": (I32, [FP, CP, I32, I64, I64, P, I32, P, P]),
            "kvq_key_salience": (I32, [FP, P, I64, I64, I64, P, I64, I64, I64, I32, I32, I32, I32,
                                       P, P, I64, I64, P, P]),
            "kvq_decode_workspace_bytes": (SZ, [FP, I32, I32, I32, I64, I32, I32]),
            "kvq_decode_attention": (I32, [FP, CP, P, I32, I32, I64, I32, ctypes.c_float, P, I32,
                                           P, SZ, I32, P, P]),
            "kvq_append_decode_attention": (I32, [FP, CP, P, P, I64, I64, I64, I64, I64, P, I32, I32, I64, I32,
                                                  ctypes.c_float, P, I32, P, SZ, I32, P, P]),
            "kvq_decode_partial_slots": (I32, [FP, I32, I32, I32, I64, I32, I32]),
            "kvq_decode_partial": (I32, [FP, CP, P, I32, I32, I64, I32, ctypes.c_float, P, SZ, I32,
                                         P, P]),
            "kvq_decode_combine": (I32, [FP, I32, I32, I32, I64, I32, I32, P, SZ, P, I32, P]),
            "kvq_decode_combine_lse": (I32, [FP, I32, I32, I32, I64, I32, I32, P, SZ, P, P, P]),
            "kvq_merge_states": (I32, [I32, I64, I32, P, P, P, I32, P, P]),
            "kvq_decode_attention_noalloc": (I32, [FP, CP, P, I32, I32, I64, I32, ctypes.c_float,
                                                   P, I32, I32, P, P]),
            "kvq_quantize_kv_paged": (I32, [FP, PP, P, P, I64, I64, I64, P, I64, P, P]),
            "kvq_decode_paged_workspace_bytes": (SZ, [FP, I32, I32, I32, I64, I32]),
            "kvq_decode_attention_paged": (I32, [FP, PP, P, P, I64, I32, P, I32, I32, ctypes.c_float, P,
                                                 I32, P, SZ, P, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(st):
    return lib().kvq_status_string(int(st)).decode()


def _check(fn, st):
    if st != KVQ_OK:
        raise KvqError(fn, st)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_format(d: dict) -> kvq_format:
    f = kvq_format()
    for name, _ in kvq_format._fields_:
        setattr(f, name, d.get(name, 0) if name == "k_rotate" else d[name])
    return f


def format_check(fmt: kvq_format) -> int:
    return lib().kvq_format_check(ctypes.byref(fmt))


def cache_array_bytes(fmt: kvq_format, B, H, C, array_id) -> int:
    return lib().kvq_cache_array_bytes(ctypes.byref(fmt), B, H, C, array_id)


def kqv_codebook(bits: int, head_dim: int):
    """kvq_kqv_codebook: the 2^bits fp32 Lloyd-Max centroids (a list of floats)."""
    out = (ctypes.c_float * (1 << bits))()
    _check("kvq_kqv_codebook", lib().kvq_kqv_codebook(bits, head_dim, out))
    return list(out)


class Cache:
    """Device arrays of a packed cache (torch uint8 tensors), owned by this object.
    k_lut / v_lut: the codebooks (NUQ: stored as fp16, KQV: fp32); sketch: the KQV sketch
    matrix [D][D] (stored as fp32)."""

    def __init__(self, fmt: kvq_format, B: int, H: int, C: int, device="cuda", k_lut=None,
                 v_lut=None, sketch=None):
        self.fmt, self.B, self.H, self.C = fmt, B, H, C
        self.tensors = {}
        self.struct = kvq_cache(batch=B, kv_heads=H, capacity=C)
        for i, name in enumerate(ARRAYS):
            n = cache_array_bytes(fmt, B, H, C, i)
            if n:
                t = torch.zeros(n, dtype=torch.uint8, device=device)
                self.tensors[name] = t
                setattr(self.struct, name, t.data_ptr())
        for name, lut, scheme in (("k_lut", k_lut, fmt.k_scheme), ("v_lut", v_lut, fmt.v_scheme)):
            if name in self.tensors and lut is not None:
                dt = torch.float32 if scheme == KQV else torch.float16
                self.tensors[name].copy_(torch.tensor(lut, dtype=dt).reshape(-1).view(torch.uint8))
        if "v_sketch" in self.tensors and sketch is not None:
            self.tensors["v_sketch"].copy_(torch.as_tensor(sketch, dtype=torch.float32).reshape(-1).view(torch.uint8))

    def array(self, name):
        return self.tensors[name]

    def ref(self):
        return ctypes.byref(self.struct)


def quantize_keys(fmt, cache: Cache, src: torch.Tensor, t0: int, n: int, status=None, stream=None):
    """src [B, H, n, D] (strided over the first three dims, channels contiguous)."""
    st = lib().kvq_quantize_keys(ctypes.byref(fmt), cache.ref(), _ptr(src), src.stride(0),
                                 src.stride(1), src.stride(2), t0, n, _ptr(status), _stream(stream))
    _check("kvq_quantize_keys", st)


def quantize_values(fmt, cache: Cache, src: torch.Tensor, t0: int, n: int, status=None,
                    stream=None):
    st = lib().kvq_quantize_values(ctypes.byref(fmt), cache.ref(), _ptr(src), src.stride(0),
                                   src.stride(1), src.stride(2), t0, n, _ptr(status),
                                   _stream(stream))
    _check("kvq_quantize_values", st)


def quantize_kv(fmt, cache: Cache, k_src: torch.Tensor, v_src: torch.Tensor, t0: int, n: int,
                status=None, stream=None):
    """Keys and values of one append (same strides), one launch where the kernels allow."""
    if k_src.stride() != v_src.stride():
        raise ValueError("k_src and v_src must have the same strides")
    st = lib().kvq_quantize_kv(ctypes.byref(fmt), cache.ref(), _ptr(k_src), _ptr(v_src),
                               k_src.stride(0), k_src.stride(1), k_src.stride(2), t0, n,
                               _ptr(status), _stream(stream))
    _check("kvq_quantize_kv", st)


def dequantize(fmt, cache: Cache, which: int, t0: int, n: int, out_dtype=F32, out=None,
               status=None, stream=None):
    if out is None:
        out = torch.empty((cache.B, cache.H, n, fmt.head_dim), dtype=TORCH_DTYPE[out_dtype],
                          device="cuda")
    st = lib().kvq_dequantize(ctypes.byref(fmt), cache.ref(), which, t0, n, _ptr(out), out_dtype,
                              _ptr(status), _stream(stream))
    _check("kvq_dequantize", st)
    return out


def key_salience(fmt, q: torch.Tensor, k: torch.Tensor, order_out: torch.Tensor,
                 order_stride_b: int, order_stride_h: int, salience_out=None, status=None,
                 stream=None):
    """q [B, Hq, R, D], k [B, Hkv, R, D]; order_out is a uint8 tensor whose element
    (b, h, slot) sits at b * order_stride_b + h * order_stride_h + slot."""
    B, Hq, R, D = q.shape
    Hkv = k.shape[1]
    st = lib().kvq_key_salience(ctypes.byref(fmt), _ptr(q), q.stride(0), q.stride(1), q.stride(2),
                                _ptr(k), k.stride(0), k.stride(1), k.stride(2), B, Hq, Hkv, R,
                                _ptr(salience_out), _ptr(order_out), order_stride_b,
                                order_stride_h, _ptr(status), _stream(stream))
    _check("kvq_key_salience", st)


def decode_workspace_bytes(fmt, B, Hq, Hkv, t_quant, t_res, num_splits=0) -> int:
    return lib().kvq_decode_workspace_bytes(ctypes.byref(fmt), B, Hq, Hkv, t_quant, t_res,
                                            num_splits)


def decode_attention(fmt, cache: Cache, q: torch.Tensor, t_quant: int, t_res: int, scale: float,
                     out_dtype=F32, out=None, workspace=None, num_splits=0, status=None,
                     stream=None):
    """q [B, Hq, D] contiguous -> out [B, Hq, D]."""
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=TORCH_DTYPE[out_dtype], device=q.device)
    need = decode_workspace_bytes(fmt, B, Hq, cache.H, t_quant, t_res, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib().kvq_decode_attention(ctypes.byref(fmt), cache.ref(), _ptr(q), KVQ_DTYPE[q.dtype],
                                    Hq, t_quant, t_res, scale, _ptr(out), out_dtype,
                                    _ptr(workspace), workspace.numel(), num_splits, _ptr(status),
                                    _stream(stream))
    _check("kvq_decode_attention", st)
    return out


def append_decode_attention(fmt, cache: Cache, k_src: torch.Tensor, v_src: torch.Tensor, t0: int, n: int,
                            q: torch.Tensor, t_quant: int, t_res: int, scale: float, out_dtype=F32, out=None,
                            workspace=None, num_splits=0, status=None, stream=None):
    """kvq_append_decode_attention: quantize_kv(k_src, v_src, t0, n) then decode_attention(q)."""
    if k_src.stride() != v_src.stride():
        raise ValueError("k_src and v_src must have the same strides")
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=TORCH_DTYPE[out_dtype], device=q.device)
    need = decode_workspace_bytes(fmt, B, Hq, cache.H, t_quant, t_res, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib().kvq_append_decode_attention(ctypes.byref(fmt), cache.ref(), _ptr(k_src), _ptr(v_src),
                                           k_src.stride(0), k_src.stride(1), k_src.stride(2), t0, n,
                                           _ptr(q), KVQ_DTYPE[q.dtype], Hq, t_quant, t_res, scale, _ptr(out),
                                           out_dtype, _ptr(workspace), workspace.numel(), num_splits,
                                           _ptr(status), _stream(stream))
    _check("kvq_append_decode_attention", st)
    return out


def decode_partial_slots(fmt, B, Hq, Hkv, t_quant, t_res, num_splits=0) -> int:
    return lib().kvq_decode_partial_slots(ctypes.byref(fmt), B, Hq, Hkv, t_quant, t_res, num_splits)


def decode_partial(fmt, cache: Cache, q: torch.Tensor, t_quant: int, t_res: int, scale: float,
                   workspace: torch.Tensor, num_splits=0, status=None, stream=None):
    B, Hq, D = q.shape
    st = lib().kvq_decode_partial(ctypes.byref(fmt), cache.ref(), _ptr(q), KVQ_DTYPE[q.dtype], Hq,
                                  t_quant, t_res, scale, _ptr(workspace), workspace.numel(),
                                  num_splits, _ptr(status), _stream(stream))
    _check("kvq_decode_partial", st)


def decode_combine(fmt, B, Hq, Hkv, t_quant, t_res, workspace: torch.Tensor, out: torch.Tensor,
                   num_splits=0, stream=None):
    st = lib().kvq_decode_combine(ctypes.byref(fmt), B, Hq, Hkv, t_quant, t_res, num_splits,
                                  _ptr(workspace), workspace.numel(), _ptr(out),
                                  KVQ_DTYPE[out.dtype], _stream(stream))
    _check("kvq_decode_combine", st)
    return out


def decode_combine_lse(fmt, B, Hq, Hkv, t_quant, t_res, workspace: torch.Tensor, out: torch.Tensor,
                       lse: torch.Tensor, num_splits=0, stream=None):
    """kvq_decode_combine_lse: out [B, Hq, D] fp32 and lse [B, Hq] fp32 of one part."""
    st = lib().kvq_decode_combine_lse(ctypes.byref(fmt), B, Hq, Hkv, t_quant, t_res, num_splits,
                                      _ptr(workspace), workspace.numel(), _ptr(out), _ptr(lse),
                                      _stream(stream))
    _check("kvq_decode_combine_lse", st)
    return out, lse


def merge_states(outs: torch.Tensor, lses: torch.Tensor, out_dtype=F32, out=None, lse_out=None,
                 stream=None):
    """kvq_merge_states: outs [n, rows..., D] fp32, lses [n, rows...] fp32 -> out [rows..., D]."""
    n, D = outs.shape[0], outs.shape[-1]
    rows = lses[0].numel()
    if out is None:
        out = torch.empty(outs.shape[1:], dtype=TORCH_DTYPE[out_dtype], device=outs.device)
    st = lib().kvq_merge_states(n, rows, D, _ptr(outs), _ptr(lses), _ptr(out), KVQ_DTYPE[out.dtype],
                                _ptr(lse_out), _stream(stream))
    _check("kvq_merge_states", st)
    return out


NOALLOC_SCRATCH_BYTES = 16 << 20


def decode_attention_noalloc(fmt, cache: Cache, q: torch.Tensor, t_quant: int, t_res: int,
                             scale: float, out_dtype=F32, out=None, num_splits=0, status=None,
                             stream=None):
    """kvq_decode_attention_noalloc: no workspace argument (the library's own scratch)."""
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=TORCH_DTYPE[out_dtype], device=q.device)
    st = lib().kvq_decode_attention_noalloc(ctypes.byref(fmt), cache.ref(), _ptr(q),
                                            KVQ_DTYPE[q.dtype], Hq, t_quant, t_res, scale,
                                            _ptr(out), out_dtype, num_splits, _ptr(status),
                                            _stream(stream))
    _check("kvq_decode_attention_noalloc", st)
    return out


class PagedCache:
    """A paged cache: a pool of num_blocks blocks (one token group of every KV head each,
    the layout of a Cache with batch = num_blocks and capacity = group_tokens), per-sequence
    sink / residual arrays and a device block table [num_seqs][max_blocks] (int32, -1)."""

    def __init__(self, fmt: kvq_format, kv_heads: int, num_blocks: int, num_seqs: int, max_blocks: int,
                 device="cuda"):
        self.fmt, self.H, self.num_blocks = fmt, kv_heads, num_blocks
        self.num_seqs, self.max_blocks = num_seqs, max_blocks
        self.pool = Cache(fmt, num_blocks, kv_heads, fmt.group_tokens, device=device)
        raw = Cache(fmt, num_seqs, kv_heads, fmt.group_tokens, device=device)
        self.raw = {n: raw.tensors[n] for n in ("sink_k", "sink_v", "res_k", "res_v") if n in raw.tensors}
        self.block_table = torch.full((num_seqs, max_blocks), -1, dtype=torch.int32, device=device)
        self.struct = kvq_paged_cache(pool=self.pool.struct, num_seqs=num_seqs, max_blocks=max_blocks,
                                      block_table=self.block_table.data_ptr())
        for n, t in self.raw.items():
            setattr(self.struct, n, t.data_ptr())

    def array(self, name):
        return self.raw[name] if name in self.raw else self.pool.tensors[name]

    def ref(self):
        return ctypes.byref(self.struct)


def quantize_kv_paged(fmt, cache: PagedCache, k_src: torch.Tensor, v_src: torch.Tensor, blocks: torch.Tensor,
                      n: int, status=None, stream=None):
    """kvq_quantize_kv_paged: k_src, v_src [num_seqs, H, n, D]; blocks int32 [num_seqs] (device)."""
    if k_src.stride() != v_src.stride():
        raise ValueError("k_src and v_src must have the same strides")
    st = lib().kvq_quantize_kv_paged(ctypes.byref(fmt), cache.ref(), _ptr(k_src), _ptr(v_src), k_src.stride(0),
                                     k_src.stride(1), k_src.stride(2), _ptr(blocks), n, _ptr(status),
                                     _stream(stream))
    _check("kvq_quantize_kv_paged", st)


def decode_paged_workspace_bytes(fmt, num_seqs, Hq, Hkv, max_t_quant, max_t_res) -> int:
    return lib().kvq_decode_paged_workspace_bytes(ctypes.byref(fmt), num_seqs, Hq, Hkv, max_t_quant, max_t_res)


def decode_attention_paged(fmt, cache: PagedCache, t_quant: torch.Tensor, t_res: torch.Tensor, max_t_quant: int,
                           max_t_res: int, q: torch.Tensor, scale: float, out_dtype=F32, out=None, workspace=None,
                           status=None, stream=None):
    """kvq_decode_attention_paged: t_quant, t_res int32 [num_seqs] (device); q [num_seqs, Hq, D]."""
    S, Hq, D = q.shape
    if out is None:
        out = torch.empty((S, Hq, D), dtype=TORCH_DTYPE[out_dtype], device=q.device)
    need = decode_paged_workspace_bytes(fmt, S, Hq, cache.H, max_t_quant, max_t_res)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib().kvq_decode_attention_paged(ctypes.byref(fmt), cache.ref(), _ptr(t_quant), _ptr(t_res), max_t_quant,
                                          max_t_res, _ptr(q), KVQ_DTYPE[q.dtype], Hq, scale, _ptr(out), out_dtype,
                                          _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream))
    _check("kvq_decode_attention_paged", st)
    return out
