"""Shared helpers of the GPU parity tests: one seeded input, two caches (the
library's on the device, the oracle's in numpy), compared array by array."""
import numpy as np
import torch

from oracle import fp
from oracle import cache as ocache
from oracle.formats import BF16, F16, F32, KEYS, VALUES, Format
from quantized_decode_attention_quantize_b200 import kvq

TORCH = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}


def dev(x, dtype):
    """float32 numpy values (exact in dtype) -> device tensor of that dtype."""
    return torch.tensor(np.asarray(x, np.float32), device="cuda").to(TORCH[dtype])


def raw_bits(x, dtype):
    return ocache.raw_encode(np.asarray(x, np.float64), dtype)


class Pair:
    """The same cache built by the library and by the oracle."""

    def __init__(self, fd, B, H, C, k_lut=None, v_lut=None):
        self.fd = dict(fd)
        self.fmt = kvq.make_format(self.fd)
        self.of = Format(**self.fd)
        self.B, self.H, self.C = B, H, C
        self.gpu = kvq.Cache(self.fmt, B, H, C, k_lut=k_lut, v_lut=v_lut)
        self.ora = ocache.Cache(self.of, B, H, C, k_lut=k_lut, v_lut=v_lut)
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def quantize(self, which, src, t0, n, strided=False):
        """src: float32 numpy values [B, H, n, D] exact in the source dtype."""
        dt = self.fd["src_dtype"]
        t = dev(src, dt)
        if strided:   # give the source non-trivial strides: [B, n, H, D] transposed
            t = t.transpose(1, 2).contiguous().transpose(1, 2)
        f = kvq.quantize_keys if which == KEYS else kvq.quantize_values
        f(self.fmt, self.gpu, t, t0, n, status=self.status)
        ocache.quantize(self.of, self.ora, which, np.asarray(src, np.float64), t0, n)

    def set_raw(self, name, values):
        """Fill a raw (sink / residual) array on both sides."""
        dt = self.fd["src_dtype"]
        bits = raw_bits(values, dt)
        self.ora[name][...] = bits
        self.gpu.array(name).copy_(torch.from_numpy(np.ascontiguousarray(bits).reshape(-1).view(np.uint8)).cuda())

    def set_order(self, order):
        """MIXED: slot -> channel orders [B, H, ngroups, D] on both sides."""
        self.ora["k_order"][...] = order
        self.gpu.array("k_order").copy_(torch.from_numpy(np.ascontiguousarray(order, np.uint8).reshape(-1)).cuda())

    def assert_arrays_equal(self, names=None):
        torch.cuda.synchronize()
        names = names or [n for n in self.ora.arrays if n in self.gpu.tensors]
        for n in names:
            got = self.gpu.array(n).cpu().numpy()
            want = np.ascontiguousarray(self.ora[n]).reshape(-1).view(np.uint8)
            if not np.array_equal(got, want):
                bad = np.nonzero(got != want)[0]
                raise AssertionError(f"{n}: {bad.size} bytes differ, first at {bad[:8]}")

    def status_bits(self):
        torch.cuda.synchronize()
        return int(self.status.item())


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def rel_l2_rows(a, b):
    """Largest relative L2 error over the query rows (the last axis is the head dimension)."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    a = a.reshape(-1, a.shape[-1])
    b = b.reshape(-1, b.shape[-1])
    return float(np.max(np.linalg.norm(a - b, axis=1) / np.linalg.norm(b, axis=1)))


# Unit roundoff of the output types: the largest relative error of rounding one value.
UNIT_ROUNDOFF = {F32: 0.0, F16: 2.0 ** -11, BF16: 2.0 ** -8}


def assert_attn(out, ref, tol, out_dtype=F32):
    """Attention parity: the whole tensor's relative L2 within `tol`, and every query row's
    relative L2 within `tol` plus the output type's unit roundoff u, so that one bad row
    cannot hide among good ones.  Rounding each element of a row to the output type alone
    moves the row by at most u in relative L2 (every element by at most u relative), and
    the rows of a 16-bit output scatter around the whole-tensor figure by up to that much;
    for fp32 output the two bars are the same."""
    whole, worst = rel_l2(out, ref), rel_l2_rows(out, ref)
    row_bar = tol + UNIT_ROUNDOFF[out_dtype]
    assert whole <= tol and worst <= row_bar, \
        f"relative L2 {whole:.3e} (bar {tol:.1e}), worst row {worst:.3e} (bar {row_bar:.2e})"


def tolerance(out_dtype):
    """Attention parity bar against the float64 oracle: relative L2 <= 1e-3 for fp32
    output, <= 2e-3 when the output is fp16 / bf16."""
    return 1e-3 if out_dtype == F32 else 2e-3
