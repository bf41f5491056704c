"""Seeded synthetic inputs shaped like the pages' workloads.

This module draws random numbers, scales them and rounds them to the source dtype.
It contains none of the quantization or attention arithmetic; both the CUDA library
(through the tests and bench.py) and the oracle consume exactly the arrays it
returns.  Every slab (one batch entry x one head) comes from its own PCG64 stream
seeded with (seed, tag, b, h), so any slab can be regenerated alone.

Workloads (sizes from the pages' models):
  toy          [AXES] INT8 experiment: K, V, Q float32 N(0, 1), N in {64, 256},
               D = 32, 8 query rows, seeds 7, 19, 41.
  llama2_7b    B 1, 32 heads (MHA), D 128, T 4096; K, V, q fp16 N(0, 1); 4 of the
               128 key channels of every head scaled x15.  K 4-bit per channel
               (group 128), V 2-bit per token.
  llama3_8b    B 8, 32 query / 8 KV heads, D 128, T 32768; bf16 K, V i.i.d.
               Student-t(4) with round(2 % * 128) = 3 key channels per KV head x10;
               q bf16 N(0, 1).  Token 0 kept raw (sink), the last 128 tokens raw
               (residual window); K 4-bit per channel, V 2-bit per token.
  kvquant_nuq3 B 1, 32 heads, D 128, T 131072; fp16 pre-RoPE K = N(0, 1) * sigma_d,
               sigma_d log-uniform in [0.1, 10] per (head, channel); V, q N(0, 1);
               nuq3 K per channel and V per token with the top-2 (1 % of 128,
               rounded up) magnitudes per vector as fp16 outliers; RoPE base 10000.
  mixkvq_14b   B 16, 40 query / 8 KV heads, D 128, T 16384; bf16 K = N(0, 1) *
               sigma_d (log-uniform [0.1, 20] per KV-head channel), Q rows =
               N(0, 1) * mu_d (log-uniform [0.1, 5] per query-head channel), V
               N(0, 1); keys: 8 raw + 24 4-bit + 96 2-bit channels per group by
               salience; V 2-bit per token; appends of 256 tokens.
"""
from __future__ import annotations

import numpy as np

F32, F16, BF16 = 0, 1, 2
NONE, SYM8, ASYM, NUQ, MIXED, KQV = 0, 1, 2, 3, 4, 5
TENSOR, TOKEN, CHANNEL = 0, 1, 2

TAGS = {"k": 1, "v": 2, "q": 3, "qwin": 4, "kchan": 5, "qchan": 6, "toy": 7}


def _fmt(**kw):
    base = dict(head_dim=128, group_tokens=128, src_dtype=F16,
                k_scheme=ASYM, k_bits=4, k_axis=CHANNEL, k_outliers=0,
                v_scheme=ASYM, v_bits=2, v_axis=TOKEN, v_outliers=0,
                mixed_hi=0, mixed_mid=0, n_sink=0, residual_cap=0,
                rope=0, rope_base=10000.0, k_rotate=0)
    base.update(kw)
    return base


CONFIGS = {
    "llama2_7b": dict(name="llama2_7b", B=1, Hq=32, Hkv=32, D=128, T=4096, seed=7,
                      q_dtype=F16, fmt=_fmt(src_dtype=F16)),
    "llama3_8b": dict(name="llama3_8b", B=8, Hq=32, Hkv=8, D=128, T=32768, seed=7,
                      q_dtype=BF16,
                      fmt=_fmt(src_dtype=BF16, n_sink=1, residual_cap=128)),
    # the Llama-3-8B workload with key-only Walsh-Hadamard rotation (same data recipe)
    "llama3_8b_wht": dict(name="llama3_8b_wht", recipe="llama3_8b", B=8, Hq=32, Hkv=8, D=128,
                          T=32768, seed=7, q_dtype=BF16,
                          fmt=_fmt(src_dtype=BF16, n_sink=1, residual_cap=128, k_rotate=1)),
    # the Llama-3-8B workload under KQV at a 4-bit budget (same data recipe): K 4-bit scalar
    # codes, V 3-bit codes plus the one-bit sketch, both after the Walsh-Hadamard rotation
    "llama3_8b_kqv": dict(name="llama3_8b_kqv", recipe="llama3_8b", B=8, Hq=32, Hkv=8, D=128,
                          T=32768, seed=7, q_dtype=BF16,
                          fmt=_fmt(src_dtype=BF16, n_sink=1, residual_cap=128, k_scheme=KQV, k_bits=4,
                                   k_axis=TOKEN, v_scheme=KQV, v_bits=4, v_axis=TOKEN)),
    # the Llama-3-8B format as a paged cache with a length mix: 8 sequences of 32k, 28k, ...,
    # 4k tokens (sink 1, residual windows of 128, 112, ..., 16 tokens), their groups in
    # blocks of a shared pool in shuffled order
    "llama3_8b_paged": dict(name="llama3_8b_paged", recipe="llama3_8b", B=8, Hq=32, Hkv=8, D=128,
                            T=32768, seed=7, q_dtype=BF16, paged=True,
                            fmt=_fmt(src_dtype=BF16, n_sink=1, residual_cap=128)),
    "kvquant_nuq3": dict(name="kvquant_nuq3", B=1, Hq=32, Hkv=32, D=128, T=131072, seed=7,
                         q_dtype=F16,
                         fmt=_fmt(src_dtype=F16, k_scheme=NUQ, k_bits=3, k_outliers=2,
                                  v_scheme=NUQ, v_bits=3, v_outliers=2, rope=1)),
    "mixkvq_14b": dict(name="mixkvq_14b", B=16, Hq=40, Hkv=8, D=128, T=16384, seed=7,
                       q_dtype=BF16, append=256,
                       fmt=_fmt(src_dtype=BF16, k_scheme=MIXED, k_bits=0,
                                mixed_hi=8, mixed_mid=24)),
}


def split_tokens(cfg, T=None):
    """(n_sink, t_quant, t_residual) of a workload of T tokens."""
    T = cfg["T"] if T is None else T
    f = cfg["fmt"]
    ns, nr = f["n_sink"], f["residual_cap"]
    return ns, T - ns - nr, nr


def rng(seed, tag, *idx):
    return np.random.default_rng([int(seed), TAGS[tag]] + [int(i) for i in idx])


def to_bf16_values(x32):
    """float32 (finite, below the bf16 overflow threshold) -> nearest-even bf16,
    returned as float32 values."""
    u = np.array(x32, np.float32, copy=True).view(np.uint32)
    u += np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    u &= np.uint32(0xFFFF0000)
    return u.view(np.float32)


def to_dtype_values(x, dtype):
    """Round generated values to the source dtype; returned as float32 values."""
    x = np.asarray(x, np.float32)
    if dtype == F32:
        return x
    if dtype == F16:
        return x.astype(np.float16).astype(np.float32)
    return to_bf16_values(x)


def student_t4(r, shape):
    """Student-t with 4 degrees of freedom: N / sqrt(chi2_4 / 4), chi2_4 the sum of
    four squared standard normals."""
    n = r.standard_normal(shape, dtype=np.float32)
    chi = np.zeros(shape, np.float32)
    for _ in range(4):
        z = r.standard_normal(shape, dtype=np.float32)
        chi += z * z
    return n / np.sqrt(chi * np.float32(0.25))


def log_uniform(r, lo, hi, shape):
    return np.exp(r.uniform(np.log(lo), np.log(hi), size=shape)).astype(np.float32)


def kv_slab(cfg, b, h, T=None, which="k"):
    """Keys or values of one (b, kv-head) slab: float32 values [T, D] in src dtype."""
    T = cfg["T"] if T is None else T
    D = cfg["D"]
    name = cfg.get("recipe", cfg["name"])
    seed = cfg["seed"]
    dt = cfg["fmt"]["src_dtype"]
    r = rng(seed, which, b, h)
    if name == "llama2_7b":
        x = r.standard_normal((T, D), dtype=np.float32)
        if which == "k":
            ch = rng(seed, "kchan", b, h).choice(D, 4, replace=False)
            x[:, ch] *= np.float32(15)
    elif name == "llama3_8b":
        x = student_t4(r, (T, D))
        if which == "k":
            n_out = int(round(0.02 * D))
            ch = rng(seed, "kchan", b, h).choice(D, n_out, replace=False)
            x[:, ch] *= np.float32(10)
    elif name == "kvquant_nuq3":
        x = r.standard_normal((T, D), dtype=np.float32)
        if which == "k":
            x *= log_uniform(rng(seed, "kchan", b, h), 0.1, 10.0, (1, D))
    elif name == "mixkvq_14b":
        x = r.standard_normal((T, D), dtype=np.float32)
        if which == "k":
            x *= log_uniform(rng(seed, "kchan", b, h), 0.1, 20.0, (1, D))
    else:
        raise KeyError(name)
    return to_dtype_values(x, dt)


def query(cfg, b, hq):
    """Decode query of one query head: float32 values [D] in q dtype."""
    r = rng(cfg["seed"], "q", b, hq)
    q = r.standard_normal(cfg["D"], dtype=np.float32)
    if cfg.get("recipe", cfg["name"]) == "mixkvq_14b":
        q *= log_uniform(rng(cfg["seed"], "qchan", b, hq), 0.1, 5.0, (cfg["D"],))
    return to_dtype_values(q, cfg["q_dtype"])


def query_window(cfg, b, hq, t0, R):
    """Query rows of positions [t0, t0 + R) of one query head (salience windows):
    float32 values [R, D] in src dtype."""
    r = rng(cfg["seed"], "qwin", b, hq, t0)
    x = r.standard_normal((R, cfg["D"]), dtype=np.float32)
    x *= log_uniform(rng(cfg["seed"], "qchan", b, hq), 0.1, 5.0, (1, cfg["D"]))
    return to_dtype_values(x, cfg["fmt"]["src_dtype"])


def queries(cfg, B=None, Hq=None):
    B = cfg["B"] if B is None else B
    Hq = cfg["Hq"] if Hq is None else Hq
    return np.stack([np.stack([query(cfg, b, h) for h in range(Hq)]) for b in range(B)])


def toy(seed, N, D=32, n_q=8):
    """[AXES] toy inputs: (Q [n_q, D], K [N, D], V [N, D]) float32 N(0, 1)."""
    r = rng(seed, "toy", N)
    K = r.standard_normal((N, D), dtype=np.float32)
    V = r.standard_normal((N, D), dtype=np.float32)
    Q = r.standard_normal((n_q, D), dtype=np.float32)
    return Q, K, V


def toy_format(scheme, target, N, D=32):
    """Library format of one [AXES] toy case (g = N so that per-channel and tensor
    scales span all N tokens, as on the page)."""
    ka = {"tensor": TENSOR, "token": TOKEN, "hybrid": CHANNEL}[scheme]
    va = {"tensor": TENSOR, "token": TOKEN, "hybrid": TOKEN}[scheme]
    return _fmt(head_dim=D, group_tokens=N, src_dtype=F32,
                k_scheme=SYM8 if target in ("both", "k_only") else NONE, k_bits=8, k_axis=ka,
                v_scheme=SYM8 if target in ("both", "v_only") else NONE, v_bits=8, v_axis=va)


def random_slab(seed, shape, dtype, scale=1.0, tag="k", idx=()):
    """Plain N(0, scale^2) values in a dtype (small parity cases)."""
    r = rng(seed, tag, *idx)
    return to_dtype_values(r.standard_normal(shape, dtype=np.float32) * np.float32(scale), dtype)


# ---- device-side generation of bulk data ------------------------------------------------
# The same recipes drawn with torch's generator on the device, for full-size caches
# whose every slab need not be regenerated on the host (timing runs, and the slabs a
# full-size parity test does not sample).  Values differ from the host streams; the
# distributions and structure are the same.

def device_kv(cfg, which, T=None, B=None, H=None, device="cuda", seed_offset=0):
    """[B, Hkv, T, D] tensor of keys or values in the source dtype, on the device."""
    import torch
    T = cfg["T"] if T is None else T
    B = cfg["B"] if B is None else B
    H = cfg["Hkv"] if H is None else H
    D = cfg["D"]
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg["seed"] * 1000 + TAGS[which] * 10 + seed_offset)
    tdt = {F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}[cfg["fmt"]["src_dtype"]]
    shape = (B, H, T, D)
    name = cfg.get("recipe", cfg["name"])
    cpu = torch.Generator()
    cpu.manual_seed(cfg["seed"] * 1000 + TAGS[which] * 10 + seed_offset + 7)
    out = torch.empty(shape, dtype=tdt, device=device)
    for b in range(B):
        for h in range(H):
            if name == "llama3_8b":
                n = torch.randn((T, D), generator=gen, device=device)
                chi = torch.zeros((T, D), device=device)
                for _ in range(4):
                    z = torch.randn((T, D), generator=gen, device=device)
                    chi += z * z
                x = n / torch.sqrt(chi * 0.25)
                if which == "k":
                    ch = torch.randperm(D, generator=cpu)[: int(round(0.02 * D))]
                    x[:, ch] *= 10.0
            else:
                x = torch.randn((T, D), generator=gen, device=device)
                if which == "k":
                    if name == "llama2_7b":
                        ch = torch.randperm(D, generator=cpu)[:4]
                        x[:, ch] *= 15.0
                    elif name in ("kvquant_nuq3", "mixkvq_14b"):
                        hi = 10.0 if name == "kvquant_nuq3" else 20.0
                        u = torch.rand(D, generator=cpu)
                        x *= torch.exp(np.log(0.1) + u * (np.log(hi) - np.log(0.1))).to(device)
            out[b, h] = x.to(tdt)
    return out


def device_queries(cfg, B=None, Hq=None, device="cuda"):
    """[B, Hq, D] decode queries in the query dtype, on the device."""
    import torch
    B = cfg["B"] if B is None else B
    Hq = cfg["Hq"] if Hq is None else Hq
    q = torch.tensor(queries(cfg, B, Hq), device=device)
    return q.to({F32: torch.float32, F16: torch.float16, BF16: torch.bfloat16}[cfg["q_dtype"]])


def paged_lengths(cfg):
    """(t_quant, t_residual) per sequence of a paged workload: T (8 - s) / 8 tokens for
    sequence s, sink n_sink, residual window 128 - 16 s."""
    ns = cfg["fmt"]["n_sink"]
    tqs, trs = [], []
    for s in range(cfg["B"]):
        T = cfg["T"] * (cfg["B"] - s) // cfg["B"]
        tr = 128 - 16 * s
        tqs.append(T - ns - tr)
        trs.append(tr)
    return tqs, trs
