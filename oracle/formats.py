"""Cache format description and byte accounting.

`Format` mirrors the fields of the library's format struct (the packed-cache
contract).  `array_bytes` restates, independently of the library, how many bytes
each cache array takes; with symmetric INT8 it reproduces the byte table of [AXES]
"Scales occupy bytes too" (pinned in tests/test_oracle_toy.py), and the K4V2 /
K4V4 code-byte ratio of [K4V2] "Key Contributions" (25 % less KV memory).
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

F32, F16, BF16 = 0, 1, 2
NONE, SYM8, ASYM, NUQ, MIXED = 0, 1, 2, 3, 4
TENSOR, TOKEN, CHANNEL = 0, 1, 2
KEYS, VALUES = 0, 1

DTYPE_BYTES = {F32: 4, F16: 2, BF16: 2}

ARRAYS = [
    "k_codes", "k_scale", "k_zero", "k_order",
    "k_out_rowptr", "k_out_col", "k_out_val",
    "v_codes", "v_scale", "v_zero",
    "v_out_col", "v_out_val",
    "k_lut", "v_lut",
    "sink_k", "sink_v", "res_k", "res_v",
]


@dataclass
class Format:
    head_dim: int = 128
    group_tokens: int = 128
    src_dtype: int = F16
    k_scheme: int = ASYM
    k_bits: int = 4
    k_axis: int = CHANNEL
    k_outliers: int = 0
    v_scheme: int = ASYM
    v_bits: int = 2
    v_axis: int = TOKEN
    v_outliers: int = 0
    mixed_hi: int = 0
    mixed_mid: int = 0
    n_sink: int = 0
    residual_cap: int = 0
    rope: int = 0
    rope_base: float = 10000.0
    k_rotate: int = 0     # keys rotated by the normalised Walsh-Hadamard transform (oracle.rotate)

    def as_dict(self):
        return asdict(self)

    @property
    def mixed_lo(self):
        return self.head_dim - self.mixed_hi - self.mixed_mid


def side(fmt: Format, which: int):
    """(scheme, bits, axis, n_outliers) of keys or values."""
    if which == KEYS:
        return fmt.k_scheme, fmt.k_bits, fmt.k_axis, fmt.k_outliers
    return fmt.v_scheme, fmt.v_bits, fmt.v_axis, fmt.v_outliers


def code_row_bytes(fmt: Format, which: int) -> int:
    """Bytes of packed codes per token row (MIXED: per row of all three planes)."""
    scheme, bits, _, _ = side(fmt, which)
    D = fmt.head_dim
    if scheme == NONE:
        return D * DTYPE_BYTES[fmt.src_dtype]
    if scheme == SYM8:
        return D
    if scheme == ASYM:
        return D * bits // 8
    if scheme == NUQ:
        return 3 * D // 8
    if scheme == MIXED:
        return 2 * fmt.mixed_hi + fmt.mixed_mid // 2 + fmt.mixed_lo // 4
    raise ValueError(scheme)


def array_bytes(fmt: Format, B: int, H: int, C: int, name: str) -> int:
    """Bytes of one cache array for B x H slabs of capacity C tokens."""
    D, g = fmt.head_dim, fmt.group_tokens
    ng = C // g
    slabs = B * H
    raw = DTYPE_BYTES[fmt.src_dtype]

    def meta(which):
        scheme, _, axis, _ = side(fmt, which)
        if scheme == SYM8:
            n = {TENSOR: ng, TOKEN: C, CHANNEL: ng * D}[axis]
            return n * 4, 0
        if scheme in (ASYM, NUQ):
            n = ng * D if axis == CHANNEL else C
            return n * 2, n * 2
        if scheme == MIXED:
            n = ng * (D - fmt.mixed_hi)
            return n * 2, n * 2
        return 0, 0

    if name == "k_codes":
        return slabs * C * code_row_bytes(fmt, KEYS)
    if name == "v_codes":
        return slabs * C * code_row_bytes(fmt, VALUES)
    if name in ("k_scale", "k_zero"):
        s, z = meta(KEYS)
        return slabs * (s if name == "k_scale" else z)
    if name in ("v_scale", "v_zero"):
        s, z = meta(VALUES)
        return slabs * (s if name == "v_scale" else z)
    if name == "k_order":
        return slabs * ng * D if fmt.k_scheme == MIXED else 0
    k_out = fmt.k_scheme == NUQ and fmt.k_outliers > 0
    v_out = fmt.v_scheme == NUQ and fmt.v_outliers > 0
    if name == "k_out_rowptr":
        return slabs * ng * (g + 1) * 4 if k_out else 0
    if name == "k_out_col":
        return slabs * ng * D * fmt.k_outliers if k_out else 0
    if name == "k_out_val":
        return slabs * ng * D * fmt.k_outliers * 2 if k_out else 0
    if name == "v_out_col":
        return slabs * C * fmt.v_outliers if v_out else 0
    if name == "v_out_val":
        return slabs * C * fmt.v_outliers * 2 if v_out else 0
    if name == "k_lut":
        return 16 if fmt.k_scheme == NUQ else 0
    if name == "v_lut":
        return 16 if fmt.v_scheme == NUQ else 0
    if name in ("sink_k", "sink_v"):
        return slabs * fmt.n_sink * D * raw
    if name in ("res_k", "res_v"):
        return slabs * fmt.residual_cap * D * raw
    if name == "v_sketch":
        return 0   # the KQV scheme's sketch matrix (oracle.kqv); none of these formats has one
    raise KeyError(name)


def payload_bytes(fmt: Format, B: int, H: int, C: int) -> int:
    """Numeric KV payload: codes + metadata + side lists + raw tokens.

    This is the quantity of [AXES] "Scales occupy bytes too" (numeric payload incl.
    fp32 scales, no headers or workspaces)."""
    return sum(array_bytes(fmt, B, H, C, a) for a in ARRAYS if a not in ("k_lut", "v_lut"))
