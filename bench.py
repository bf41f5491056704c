#!/usr/bin/env python
"""Benchmark of the hot path: append-time quantization of one token group plus
decode attention over the packed cache, on synthetic data shaped like the workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config llama3_8b]

One step = kvq_append_decode_attention: the append (kvq_quantize_kv, keys and values)
of one 128-token group (the flush of the raw window into the packed cache), then the
split kernel and the combine over all T tokens.  Every step is timed with CUDA events on
the launching stream, one pair around each step; the per-kernel breakdown comes from a
separate pass of separate calls with an event between every two launches; the L2 is flushed between steps, outside the events, by a 512 MiB write and
then a 512 MiB read of another buffer (so that no dirty line of the flush is left
for the step to write back).  `value` is the effective HBM throughput of the whole step: the format's
algorithmic bytes (codes, scales, zero-points, raw sink / residual tokens, the new
group's source and packed output, q and out) over the step time.  One JSON line is
printed by rank 0.  Under torchrun every rank runs its own replica (weak scaling:
the per-GPU work is fixed), the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "Decode-attn effective HBM GB/s over packed KV (% of 8 TB/s); quantize GB/s"
L2_FLUSH_BYTES = 512 << 20
LAUNCHES_PER_STEP = 3   # quantize K+V (one launch on the K4/V2 path), split kernel, combine
PATH_DTYPE = {
    "decode_k4v2_kernel": "f16 tensor-core operands (codes as exact f16 subnormals, probabilities as f16 "
                          "hi + lo pairs), f32 accumulation",
    "decode_kqv_kernel": "f32 on CUDA cores (fp32 centroids, sketch signs)",
    "decode_mma_kernel": "f16 tensor-core operands (codes as exact f16 subnormals), f32 accumulation",
    "decode_cc_kernel": "f32 on CUDA cores (codes reconstructed to f32)",
    "decode_generic_kernel": "f32 on CUDA cores (codes reconstructed to f32)",
}


def decode_path(cfg):
    """The split kernel the library plans for this workload (same rules as its planner)."""
    f = cfg["fmt"]
    G = cfg["Hq"] // cfg["Hkv"]
    mix = f["k_scheme"] == synth.MIXED and f["mixed_hi"] == 8 and f["mixed_mid"] == 24 and \
        f["src_dtype"] == synth.BF16 and f["v_scheme"] == synth.ASYM and f["v_bits"] == 2 and not f["rope"]
    if f["k_scheme"] == synth.KQV:
        return "decode_kqv_kernel"
    if is_k4v2(cfg) and f["head_dim"] == 128 and f["group_tokens"] == 128 and 1 <= G <= 4:
        return "decode_k4v2_kernel"
    if (is_k4v2(cfg) or mix) and f["head_dim"] == 128 and f["group_tokens"] == 128 and 1 <= G <= 8:
        return "decode_mma_kernel"
    k_ok = (f["k_scheme"] == synth.NUQ) or (f["k_scheme"] == synth.ASYM and f["k_bits"] in (2, 4)) or \
        (f["k_scheme"] == synth.MIXED and not f["rope"])
    v_ok = (f["v_scheme"] == synth.NUQ) or (f["v_scheme"] == synth.ASYM and f["v_bits"] in (2, 4))
    if f["head_dim"] == 128 and G <= 8 and f["group_tokens"] % 32 == 0 and k_ok and v_ok:
        return "decode_cc_kernel"
    return "decode_generic_kernel"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="llama3_8b",
                    choices=list(synth.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


# ---- algorithmic byte counts ---------------------------------------------------------------

def fmt_bytes(cfg):
    """Per-token / per-group byte counts of the K4V2 format (D = 128, g = 128)."""
    D, g = cfg["D"], cfg["fmt"]["group_tokens"]
    kb, vb = cfg["fmt"]["k_bits"], cfg["fmt"]["v_bits"]
    raw = 2 if cfg["fmt"]["src_dtype"] != synth.F32 else 4
    return dict(k_code=D * kb // 8, v_code=D * vb // 8, v_meta=4, k_meta_group=4 * D,
                raw_token=2 * D * raw, g=g, D=D, raw=raw)


def decode_kernel_bytes(cfg, tq, tr):
    """Bytes the decode split kernel must read: packed rows, their metadata, raw
    sink / residual tokens and the queries."""
    f = fmt_bytes(cfg)
    ns = cfg["fmt"]["n_sink"]
    ngv = -(-tq // f["g"])
    per_head = tq * (f["k_code"] + f["v_code"] + f["v_meta"]) + ngv * f["k_meta_group"] + \
        (ns + tr) * f["raw_token"]
    q = cfg["B"] * cfg["Hq"] * cfg["D"] * 2
    return cfg["B"] * cfg["Hkv"] * per_head + q


def decode_call_bytes(cfg, tq, tr):
    return decode_kernel_bytes(cfg, tq, tr) + cfg["B"] * cfg["Hq"] * cfg["D"] * 4   # fp32 out


K4V2 = dict(k_scheme=synth.ASYM, k_bits=4, k_axis=synth.CHANNEL, v_scheme=synth.ASYM, v_bits=2,
            v_axis=synth.TOKEN, k_outliers=0, v_outliers=0, rope=0)


def is_k4v2(cfg):
    return all(cfg["fmt"][k] == v for k, v in K4V2.items())


def fused_kv(cfg):
    """kvq_quantize_kv is one launch for K4/V2 (with rotated keys too, at D = 128, g <= 128)."""
    f = cfg["fmt"]
    return is_k4v2(cfg) and (not f.get("k_rotate", 0) or (f["head_dim"] == 128 and f["group_tokens"] <= 128))


def step_launches(cfg, n_app):
    """Kernels one timed step launches: the split kernel appends a single group of a
    K4/V2 cache itself (unrotated keys, 16-bit sources, G <= 4), else the append is one
    launch (two for separate key and value kernels, one more per MixKVQ salience window)."""
    f = cfg["fmt"]
    g = f["group_tokens"]
    if (is_k4v2(cfg) and not f.get("k_rotate", 0) and f["src_dtype"] in (synth.F16, synth.BF16)
            and cfg["Hq"] // cfg["Hkv"] <= 4 and n_app <= g):
        return 2
    mixed = f["k_scheme"] == synth.MIXED
    return LAUNCHES_PER_STEP + (0 if fused_kv(cfg) else 1) + (n_app // g if mixed else 0)


def cache_read_bytes(cache, cfg, tq, tr):
    """Algorithmic decode bytes of any format: every cache array the decode reads (codes,
    metadata, slot order, outliers: sized for the packed capacity, i.e. t_quant rounded up
    to whole groups; raw sink / residual tokens: the ones in use), plus q and the fp32 out."""
    raw = {"sink_k", "sink_v", "res_k", "res_v"}
    n = sum(t.numel() for name, t in cache.tensors.items() if name not in raw | {"k_lut", "v_lut"})
    esz = 4 if cfg["fmt"]["src_dtype"] == synth.F32 else 2
    n += cfg["B"] * cfg["Hkv"] * (cfg["fmt"]["n_sink"] + tr) * 2 * cfg["D"] * esz
    return n + cfg["B"] * cfg["Hq"] * cfg["D"] * (2 + 4)


def quant_bytes(cfg, n):
    """One append of n tokens: 16-bit K and V read, codes and metadata written."""
    f = fmt_bytes(cfg)
    heads = cfg["B"] * cfg["Hkv"]
    read = heads * n * f["D"] * f["raw"] * 2
    write = heads * (n * (f["k_code"] + f["v_code"] + f["v_meta"]) + -(-n // f["g"]) * f["k_meta_group"])
    return read + write


# ---- clocks -----------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index):
        self.dev = dev_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---- the oracle as a CPU baseline ------------------------------------------------------------

class OracleSample:
    """The float64 oracle on a bounded sample of the workload: the flush quantize of
    one group of one KV head plus decode attention of that head's G query heads over
    `groups` packed groups and its raw tokens.  Setup (data, cache) is not timed."""

    def __init__(self, cfg, groups, head=0):
        from oracle import cache as ocache
        from oracle import fp
        from oracle.formats import KEYS, VALUES, Format
        self.cfg = cfg
        of = Format(**cfg["fmt"])
        g = of.group_tokens
        self.G = cfg["Hq"] // cfg["Hkv"]
        ns, tq_full, tr = synth.split_tokens(cfg)
        tq = min(tq_full, groups * g)
        T = ns + tq + tr
        self.head = head % cfg["Hkv"]
        K = synth.kv_slab(cfg, 0, self.head, T, "k")[None, None].astype(np.float64)
        V = synth.kv_slab(cfg, 0, self.head, T, "v")[None, None].astype(np.float64)
        luts = (None, None)
        if of.k_scheme == synth.NUQ:
            cb = json.load(open(os.path.join(ROOT, "tests", "golden", "nuq3_codebook.json")))
            luts = (cb["k"], cb["v"])
        c = ocache.Cache(of, 1, 1, -(-tq // g) * g, k_lut=luts[0], v_lut=luts[1])
        if of.k_scheme == synth.MIXED:   # a valid slot order (salience is not timed here)
            c["k_order"][...] = np.arange(of.head_dim, dtype=np.uint8)
        ocache.quantize(of, c, KEYS, K[:, :, ns:ns + tq], 0, tq)
        ocache.quantize(of, c, VALUES, V[:, :, ns:ns + tq], 0, tq)
        enc = fp.bf16_bits if of.src_dtype == synth.BF16 else fp.f16_bits
        if ns:
            c["sink_k"][...] = enc(K[:, :, :ns])
            c["sink_v"][...] = enc(V[:, :, :ns])
        if tr:
            c["res_k"][...] = enc(K[:, :, ns + tq:])
            c["res_v"][...] = enc(V[:, :, ns + tq:])
        self.q = np.stack([synth.query(cfg, 0, self.head * self.G + h)
                           for h in range(self.G)])[None].astype(np.float64)
        self.newk, self.newv = K[:, :, ns:ns + g], V[:, :, ns:ns + g]
        self.of, self.c, self.tq, self.tr, self.g, self.ns = of, c, tq, tr, g, ns
        one_head = dict(cfg, B=1, Hkv=1, Hq=self.G)
        if is_k4v2(cfg):
            self.nbytes = decode_call_bytes(one_head, tq, tr) + quant_bytes(one_head, g)
        else:   # the packed arrays it reads, its raw tokens, q and out, one group's input
            packed = sum(a.nbytes for n, a in c.arrays.items()
                         if n not in ("sink_k", "sink_v", "res_k", "res_v", "k_lut", "v_lut"))
            esz = 4 if of.src_dtype == synth.F32 else 2
            self.nbytes = packed + (ns + tr) * 2 * of.head_dim * esz + self.G * of.head_dim * 6 + \
                2 * g * of.head_dim * esz

    def run(self):
        return sum(self.run_split())

    def run_split(self):
        """(quantize seconds, decode seconds) of one pass over the sample."""
        from oracle import cache as ocache
        from oracle import attention as oatt
        from oracle.formats import KEYS, VALUES
        t0 = time.perf_counter()
        ocache.quantize(self.of, self.c, KEYS, self.newk, 0, self.g)
        ocache.quantize(self.of, self.c, VALUES, self.newv, 0, self.g)
        t1 = time.perf_counter()
        oatt.decode_attention(self.of, self.c, self.q, self.tq, self.tr)
        return t1 - t0, time.perf_counter() - t1

    def describe(self):
        return (f"oracle (numpy, float64) on one KV head of {self.cfg['name']}: quantize of one "
                f"{self.g}-token group (K and V) + decode of its {self.G} query heads over "
                f"{self.tq} packed rows + {self.ns + self.tr} raw tokens")


def single_thread():
    """Limits the BLAS pools of this process to one thread (the oracle is then one thread)."""
    from threadpoolctl import threadpool_limits
    return threadpool_limits(1)


def oracle_sized(cfg, budget_s):
    """An OracleSample whose run() takes about budget_s seconds on one thread."""
    with single_thread():
        probe = OracleSample(cfg, 4)
        probe.run()
        per_group = probe.run() / 4
    groups = int(max(1, budget_s / max(per_group, 1e-6)))
    return OracleSample(cfg, groups)


def _oracle_worker(job):
    """One process of the all-cores baseline: its own KV head of the sample, one thread."""
    name, groups, head, reps = job
    with single_thread():
        smp = OracleSample(synth.CONFIGS[name], groups, head)
        smp.run()
        t = [smp.run_split() for _ in range(reps)]
    return smp.nbytes, t


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def cpu_baseline(cfg, budget_s=4.0, reps=3):
    """The float64 oracle timed on this host: one thread in this process, then one process
    per available core (spawned, each on its own KV head of the workload, one thread each,
    at most 32), with quantize and decode seconds reported apart."""
    import multiprocessing as mp
    smp = oracle_sized(cfg, budget_s)
    with single_thread():
        smp.run()
        one = [smp.run_split() for _ in range(reps)]
    q1 = statistics.mean(t[0] for t in one)
    d1 = statistics.mean(t[1] for t in one)
    procs = max(1, min(32, cpu_cores()))
    jobs = [(cfg["name"], smp.tq // smp.g, h, reps) for h in range(procs)]
    with mp.get_context("spawn").Pool(procs) as pool:
        pool.map(_oracle_worker, jobs[:procs], chunksize=1)   # imports and setup, untimed
        t0 = time.perf_counter()
        res = pool.map(_oracle_worker, jobs, chunksize=1)
        wall = time.perf_counter() - t0
    # the processes run side by side: the aggregate rate is the sum of their own rates over
    # the passes each timed (each process's setup is outside its timed passes)
    rate = sum(n * len(t) / sum(a + b for a, b in t) for n, t in res)
    qa = statistics.mean(statistics.mean(a for a, _ in t) for _, t in res)
    da = statistics.mean(statistics.mean(b for _, b in t) for _, t in res)
    return {
        "value": rate / 1e9, "unit": "GB/s", "cores": procs, "kind": "oracle",
        "sample": smp.describe() + f"; {procs} spawned processes side by side, one thread each, "
                  f"each on its own KV head, {reps} timed passes per process, rates summed",
        "nproc": os.cpu_count(), "available_cores": cpu_cores(),
        "single_thread": {"value": smp.nbytes / (q1 + d1) / 1e9, "unit": "GB/s", "cores": 1,
                          "quantize_s": q1, "decode_s": d1},
        "all_cores": {"quantize_s": qa, "decode_s": da, "wall_s": wall},
    }


# ---- main --------------------------------------------------------------------------------------

def setup_dist(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank timings over the process group (any backend: the
    tensor lives on `device`, CPU for gloo); identity without a group of size > 1."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def run_reference(args, world, rank):
    cfg = synth.CONFIGS[args.config]
    if rank != 0:
        return
    if cfg["fmt"]["k_scheme"] == synth.KQV or cfg.get("paged"):
        print(json.dumps({"impl": "reference", "unavailable": "the oracle's timed sample covers the "
                          "contiguous cache schemes of oracle.cache"}), flush=True)
        return
    per_step = max(0.02, 120.0 / max(1, args.steps + args.warmup))
    smp = oracle_sized(cfg, per_step)
    with single_thread():
        for _ in range(args.warmup):
            smp.run()
        times = [smp.run() for _ in range(args.steps)]
    sec = statistics.mean(times)
    gbs = smp.nbytes / sec / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sec,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(cfg),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": smp.describe() + " per step, one thread", "nproc": os.cpu_count()},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(cfg):
    ns, tq, tr = synth.split_tokens(cfg)
    f = cfg["fmt"]
    names = {synth.NONE: "raw", synth.SYM8: "INT8 sym", synth.ASYM: "asym", synth.NUQ: "nuq", synth.MIXED: "mixed"}
    names[synth.KQV] = "KQV"
    kdesc = (f"mixed {f['mixed_hi']} raw / {f['mixed_mid']} 4-bit / rest 2-bit by salience"
             if f["k_scheme"] == synth.MIXED else
             f"KQV {f['k_bits']}-bit Lloyd-Max codes of the rotated direction per token"
             if f["k_scheme"] == synth.KQV else f"{names[f['k_scheme']]}{f['k_bits']} per-channel")
    if f.get("k_rotate"):
        kdesc += " after a Walsh-Hadamard rotation of each key"
    extra = []
    if f["k_outliers"] or f["v_outliers"]:
        extra.append(f"top-{max(f['k_outliers'], f['v_outliers'])} fp16 outliers per vector")
    if f["rope"]:
        extra.append(f"RoPE base {f['rope_base']:g} on keys")
    n_app = cfg.get("append", f["group_tokens"])
    return {"workload": f"{cfg['name']}: B={cfg['B']} Hq={cfg['Hq']} Hkv={cfg['Hkv']} D={cfg['D']} "
                        f"T={cfg['T']} (sink {ns}, packed {tq}, residual {tr}); K {kdesc} "
                        + (f"+ V KQV {f['v_bits'] - 1}-bit codes + 1-bit sketch per token"
                           if f["v_scheme"] == synth.KQV else
                           f"g{f['group_tokens']} + V {names[f['v_scheme']]}{f['v_bits']} per-token")
                        + ("; " + ", ".join(extra) if extra else ""),
            "B": cfg["B"], "Hq": cfg["Hq"], "Hkv": cfg["Hkv"], "D": cfg["D"], "T": cfg["T"],
            "step": f"append of {n_app} tokens (quantize K, V" +
                    (", salience" if f["k_scheme"] == synth.MIXED else "") + ") + decode attention over T",
            "l2": "flushed between steps outside the timed events (512 MiB write, then 512 MiB read)",
            "parallelism": "replicas (one independent cache per GPU)"}


def main_paged(args, cfg, world, rank, dev):
    """The paged cache with per-sequence lengths: one step = the flush of one group per
    sequence into its block (kvq_quantize_kv_paged) + kvq_decode_attention_paged over every
    sequence's own tokens."""
    import torch
    from quantized_decode_attention_quantize_b200 import kvq
    fd = cfg["fmt"]
    fmt = kvq.make_format(fd)
    S, Hq, Hkv, D, g = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["D"], fd["group_tokens"]
    ns = fd["n_sink"]
    tqs, trs = synth.paged_lengths(cfg)
    ngs = [-(-t // g) for t in tqs]
    nblocks = sum(ngs)
    max_blocks = max(ngs)
    scale = 1.0 / float(np.sqrt(D))
    cache = kvq.PagedCache(fmt, Hkv, nblocks, S, max_blocks, device=dev)
    # every block's group drawn with the workload's recipe, quantized into the pool at once
    K = synth.device_kv(cfg, "k", T=g, B=nblocks, device=dev, seed_offset=rank)
    V = synth.device_kv(cfg, "v", T=g, B=nblocks, device=dev, seed_offset=rank)
    kvq.quantize_kv(fmt, cache.pool, K, V, 0, g)
    del K, V
    gen = torch.Generator(device="cpu")
    gen.manual_seed(cfg["seed"] * 1000 + 66 + rank)
    perm = torch.randperm(nblocks, generator=gen)
    table = torch.full((S, max_blocks), -1, dtype=torch.int32)
    o = 0
    for s_, n in enumerate(ngs):
        table[s_, :n] = perm[o:o + n].to(torch.int32)
        o += n
    cache.block_table.copy_(table)
    for name in ("sink_k", "sink_v", "res_k", "res_v"):
        t = cache.array(name)
        t.copy_(torch.randn(t.numel() // 2, device=dev, generator=torch.Generator(device=dev).manual_seed(5))
                .to(torch.bfloat16).view(torch.uint8))
    tq_d = torch.tensor(tqs, dtype=torch.int32, device=dev)
    tr_d = torch.tensor(trs, dtype=torch.int32, device=dev)
    # the step's flush: the last full group of each sequence, rewritten from new values
    last = torch.tensor([int(table[s_, tqs[s_] // g - 1]) for s_ in range(S)], dtype=torch.int32, device=dev)
    newk = synth.device_kv(cfg, "k", T=g, B=S, device=dev, seed_offset=rank + 1)
    newv = synth.device_kv(cfg, "v", T=g, B=S, device=dev, seed_offset=rank + 1)
    q = synth.device_queries(cfg, B=S, device=dev)
    out = torch.empty((S, Hq, D), dtype=torch.float32, device=dev)
    ws = torch.empty(kvq.decode_paged_workspace_bytes(fmt, S, Hq, Hkv, max(tqs), max(trs)), dtype=torch.uint8,
                     device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def flush_l2(i):
        flush.fill_(i & 0xFF)
        flush_r.sum()

    def append():
        kvq.quantize_kv_paged(fmt, cache, newk, newv, last, g, status=status, stream=stream)

    def decode():
        kvq.decode_attention_paged(fmt, cache, tq_d, tr_d, max(tqs), max(trs), q, scale, kvq.F32, out=out,
                                   workspace=ws, status=status, stream=stream)

    for i in range(args.warmup):
        flush_l2(i)
        append()
        decode()
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    sampler = ClockSampler(f"GPU-{uuid}" if uuid is not None else str(dev.index))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.15)
    for i in range(args.steps):
        flush_l2(i)
        evs[i][0].record(stream)
        append()
        evs[i][1].record(stream)
        decode()
        evs[i][2].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    ms_step = statistics.mean([e[0].elapsed_time(e[2]) for e in evs])
    ms_app = statistics.mean([e[0].elapsed_time(e[1]) for e in evs])
    ms_dec = statistics.mean([e[1].elapsed_time(e[2]) for e in evs])
    ms_step, ms_app, ms_dec = max_over_ranks([ms_step, ms_app, ms_dec], dev)
    assert int(status.item()) == 0 and bool(torch.isfinite(out).all())
    # algorithmic bytes: per sequence its packed rows (64 + 32 + 4 B per token and KV head),
    # the key scale / zero-point of its groups (512 B each), its raw tokens (2 D bf16 K and
    # V), q and the fp32 out; the append reads the bf16 group and writes its codes
    dec_bytes = sum(Hkv * (t * 100 + n * 512 + (ns + r) * 2 * D * 2) for t, n, r in zip(tqs, ngs, trs))
    dec_bytes += S * Hq * D * (2 + 4)
    app_bytes = S * Hkv * (g * D * 2 * 2 + g * 100 + 512)
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except OSError:
        pass
    peak = peaks.get("hbm_gbs", 6650.0)
    achieved = dec_bytes / (ms_dec * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": world * (dec_bytes + app_bytes) / (ms_step * 1e-3) / 1e9, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": PATH_DTYPE["decode_k4v2_kernel"], "data": "synthetic (device-drawn, recipe of synth/)",
        "config": {"workload": f"{cfg['name']}: paged pool of {nblocks} blocks (one 128-token group of "
                               f"{Hkv} KV heads each, shuffled), {S} sequences of {tqs} packed + 1 sink + "
                               f"{trs} residual tokens, Hq={Hq}, D={D}; K asym4 per-channel g128 + V asym2 "
                               "per-token",
                   "step": "flush of one group per sequence into its block + paged decode attention",
                   "l2": "flushed between steps outside the timed events",
                   "parallelism": "replicas (one independent cache per GPU)"},
        "ms_breakdown": {"append": ms_app, "decode": ms_dec},
        "roofline": {"kernel": "decode_paged_kernel + combine_paged_kernel (kvq_decode_attention_paged)",
                     "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": None, "algorithmic_bytes": dec_bytes,
                     "peak_source": "MEASURED_PEAKS.json hbm_gbs (measured)" if peaks else "fallback"},
        "e2e": None, "gpu_launches": 3 * args.steps, "clocks": clocks, "cpu_baseline": None,
    }
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    import torch
    world, rank, local = setup_dist(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    from quantized_decode_attention_quantize_b200 import kvq
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = synth.CONFIGS[args.config]
    if cfg.get("paged"):
        main_paged(args, cfg, world, rank, dev)
        return
    fd = cfg["fmt"]
    fmt = kvq.make_format(fd)
    B, Hq, Hkv, D, g = cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["D"], fd["group_tokens"]
    ns, tq, tr = synth.split_tokens(cfg)
    C = -(-tq // g) * g
    scale = 1.0 / float(np.sqrt(D))

    # ---- build the cache on the device (data drawn on the device, same recipe)
    K = synth.device_kv(cfg, "k", device=dev, seed_offset=rank)
    V = synth.device_kv(cfg, "v", device=dev, seed_offset=rank)
    luts, sketch = (None, None), None
    if fd["k_scheme"] == synth.NUQ:
        cb = json.load(open(os.path.join(ROOT, "tests", "golden", "nuq3_codebook.json")))
        luts = (cb["k"], cb["v"])
    if fd["k_scheme"] == synth.KQV:   # the library's Lloyd-Max codebooks, a seeded N(0, 1) sketch
        luts = (kvq.kqv_codebook(fd["k_bits"], D), kvq.kqv_codebook(fd["v_bits"] - 1, D))
        gen = torch.Generator(device=dev)
        gen.manual_seed(cfg["seed"] * 1000 + 55)
        sketch = torch.randn((D, D), device=dev, generator=gen)
    cache = kvq.Cache(fmt, B, Hkv, C, device=dev, k_lut=luts[0], v_lut=luts[1], sketch=sketch)
    mixed = fd["k_scheme"] == synth.MIXED
    qwin = None
    if mixed:   # salience windows: query rows at every packed position (device-drawn)
        gen = torch.Generator(device=dev)
        gen.manual_seed(cfg["seed"] * 1000 + 44 + rank)
        mu = torch.exp(torch.empty((1, Hq, 1, D), device=dev).uniform_(np.log(0.1), np.log(5.0), generator=gen))
        qwin = (torch.randn((B, Hq, tq, D), device=dev, generator=gen) * mu).to(K.dtype)
        order = cache.array("k_order")
        for gi in range(-(-tq // g)):
            t0, ln = gi * g, min(g, tq - gi * g)
            kvq.key_salience(fmt, qwin[:, :, t0:t0 + ln], K[:, :, ns + t0:ns + t0 + ln], order[gi * D:],
                             Hkv * (C // g) * D, (C // g) * D)
    kvq.quantize_keys(fmt, cache, K[:, :, ns:ns + tq], 0, tq)
    kvq.quantize_values(fmt, cache, V[:, :, ns:ns + tq], 0, tq)
    # full-cache quantize rate (keys + values of all packed tokens in one call, timed
    # again after the build above)
    fq_ms = []
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        kvq.quantize_kv(fmt, cache, K[:, :, ns:ns + tq], V[:, :, ns:ns + tq], 0, tq)
        e1.record()
        e1.synchronize()
        fq_ms.append(e0.elapsed_time(e1))
    fq_read = 2 * B * Hkv * tq * D * K.element_size()
    fq_written = sum(t.numel() for name, t in cache.tensors.items()
                     if name not in ("sink_k", "sink_v", "res_k", "res_v", "k_lut", "v_lut"))
    full_quant = {"ms": min(fq_ms), "gbs": (fq_read + fq_written) / (min(fq_ms) * 1e-3) / 1e9,
                  "bytes": fq_read + fq_written, "tokens": tq}
    if ns:
        cache.array("sink_k").copy_(K[:, :, :ns].contiguous().view(-1).view(torch.uint8))
        cache.array("sink_v").copy_(V[:, :, :ns].contiguous().view(-1).view(torch.uint8))
    if tr:
        cache.array("res_k").copy_(K[:, :, ns + tq:].contiguous().view(-1).view(torch.uint8))
        cache.array("res_v").copy_(V[:, :, ns + tq:].contiguous().view(-1).view(torch.uint8))
    # the append: rewrite the last n_app packed tokens (whole groups) from their own
    # values -- one group (the flush of the residual window), or the workload's append
    n_app = cfg.get("append", g)
    a0 = (tq // g) * g - n_app
    gi_f = a0 // g
    newk = K[:, :, ns + a0: ns + a0 + n_app].contiguous()
    newv = V[:, :, ns + a0: ns + a0 + n_app].contiguous()
    neww = qwin[:, :, a0:a0 + n_app].contiguous() if mixed else None
    del K, V, qwin
    q = synth.device_queries(cfg, device=dev)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    ws = torch.empty(kvq.decode_workspace_bytes(fmt, B, Hq, Hkv, tq, tr), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)

    def flush_l2(i):
        flush.fill_(i & 0xFF)
        flush_r.sum()

    order = cache.array("k_order") if mixed else None

    def salience(k_src, w_src):
        if mixed:
            for j in range(n_app // g):
                kvq.key_salience(fmt, w_src[:, :, j * g:(j + 1) * g], k_src[:, :, j * g:(j + 1) * g],
                                 order[(gi_f + j) * D:], Hkv * (C // g) * D, (C // g) * D,
                                 status=status, stream=stream)

    def fused(k_src, v_src, w_src, qq):
        # the public one-call step: append then decode (kvq_append_decode_attention)
        salience(k_src, w_src)
        kvq.append_decode_attention(fmt, cache, k_src, v_src, a0, n_app, qq, tq, tr, scale, kvq.F32, out=out,
                                    workspace=ws, status=status, stream=stream)

    def step(evs=None):
        if not evs:
            fused(newk, newv, neww, q)
            return
        # the same work as separate calls, an event between every two
        evs[0].record(stream)
        salience(newk, neww)
        kvq.quantize_kv(fmt, cache, newk, newv, a0, n_app, status=status, stream=stream)
        evs[1].record(stream)
        kvq.decode_partial(fmt, cache, q, tq, tr, scale, ws, status=status, stream=stream)
        evs[2].record(stream)
        kvq.decode_combine(fmt, B, Hq, Hkv, tq, tr, ws, out, stream=stream)
        evs[3].record(stream)

    for i in range(args.warmup):
        flush_l2(i)
        step()
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0, f"device status {int(status.item())}"

    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    sampler = ClockSampler(f"GPU-{uuid}" if uuid is not None else str(local))
    # the timed steps: one event pair around each step (events between the launches
    # would stop each kernel from starting while its predecessor drains)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.15)
    for i in range(args.steps):
        flush_l2(i)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    ms_step = statistics.mean([e[0].elapsed_time(e[1]) for e in evs])
    # the breakdown: a separate pass with an event between every two launches
    nb = min(args.steps, 50)
    bevs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nb)]
    for i in range(nb):
        flush_l2(i)
        step(bevs[i])
    torch.cuda.synchronize(dev)
    ms_quant = statistics.mean([e[0].elapsed_time(e[1]) for e in bevs])
    ms_part = statistics.mean([e[1].elapsed_time(e[2]) for e in bevs])
    ms_comb = statistics.mean([e[2].elapsed_time(e[3]) for e in bevs])
    ms_step, ms_part, ms_comb, ms_quant = max_over_ranks([ms_step, ms_part, ms_comb, ms_quant], dev)

    # ---- end to end through the public API with host buffers: every step copies its new
    # K/V group and q from pinned host memory, calls kvq_append_decode_attention and reads the
    # output back.  Serial: one step at a time, timed alone.  Pipelined (the reported figure):
    # step i + 1's host-to-device copies run on a copy stream while step i computes, into a
    # second set of device buffers; the cache (larger than L2) is not flushed between steps.
    e2e_steps = max(10, args.steps // 10)
    # the step's inputs (new K, new V, q and, for MixKVQ, the query window) packed in one
    # pinned host buffer and copied with one host-to-device copy per step into one of two
    # device buffers; the tensors the call takes are views of it
    parts = [newk, newv, q] + ([neww] if mixed else [])
    sizes = [t.numel() * t.element_size() for t in parts]
    offs = [0]
    for n in sizes:
        offs.append(offs[-1] + (n + 255) // 256 * 256)
    hbuf = torch.empty(offs[-1], dtype=torch.uint8, device="cpu").pin_memory()
    for t, o, n in zip(parts, offs, sizes):
        hbuf[o:o + n].copy_(t.contiguous().view(-1).view(torch.uint8).cpu())
    dbuf = [torch.empty(offs[-1], dtype=torch.uint8, device=dev) for _ in range(2)]

    def views(sl):
        return [dbuf[sl][o:o + n].view(t.dtype).view(t.shape) for t, o, n in zip(parts, offs, sizes)]

    dviews = [views(0), views(1)]
    dk = [v[0] for v in dviews]
    dv = [v[1] for v in dviews]
    dq = [v[2] for v in dviews]
    dw = [v[3] if mixed else None for v in dviews]
    hout = [torch.empty_like(out, device="cpu").pin_memory() for _ in range(2)]

    def h2d(sl):
        dbuf[sl].copy_(hbuf, non_blocking=True)

    e2e_t = []
    for i in range(e2e_steps + 3):
        flush_l2(i)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        h2d(0)
        fused(dk[0], dv[0], dw[0], dq[0])
        hout[0].copy_(out, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if i >= 3:
            e2e_t.append(e0.elapsed_time(e1))
    ms_e2e_serial = max_over_ranks([statistics.mean(e2e_t)], dev)[0]

    copy_stream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]

    def pipelined(n):
        for i in range(n):
            sl = i & 1
            with torch.cuda.stream(copy_stream):
                if i >= 2:
                    copy_stream.wait_event(done[sl])   # step i - 2 has finished with these buffers
                h2d(sl)
                copied[sl].record(copy_stream)
            stream.wait_event(copied[sl])
            fused(dk[sl], dv[sl], dw[sl], dq[sl])
            hout[sl].copy_(out, non_blocking=True)
            done[sl].record(stream)

    pipelined(3)
    torch.cuda.synchronize(dev)
    p0 = torch.cuda.Event(enable_timing=True)
    p1 = torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    copy_stream.wait_event(p0)
    pipelined(e2e_steps)
    p1.record(stream)
    torch.cuda.synchronize(dev)
    ms_e2e = max_over_ranks([p0.elapsed_time(p1) / e2e_steps], dev)[0]
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    assert torch.isfinite(out).all()

    path = decode_path(cfg)
    if is_k4v2(cfg):
        call_bytes = decode_call_bytes(cfg, tq, tr)
        kern_bytes = decode_kernel_bytes(cfg, tq, tr)
        q_bytes = quant_bytes(cfg, n_app)
    else:
        call_bytes = cache_read_bytes(cache, cfg, tq, tr)
        kern_bytes = call_bytes - B * Hq * D * 4
        esz = 4 if fd["src_dtype"] == synth.F32 else 2
        packed = sum(t.numel() for name, t in cache.tensors.items()
                     if name not in ("sink_k", "sink_v", "res_k", "res_v", "k_lut", "v_lut"))
        q_bytes = B * Hkv * n_app * D * esz * 2 + packed * n_app // C
        if mixed:
            q_bytes += B * Hq * n_app * D * esz
    step_bytes = call_bytes + q_bytes
    value = world * step_bytes / (ms_step * 1e-3) / 1e9
    decode_gbs = call_bytes / ((ms_part + ms_comb) * 1e-3) / 1e9
    quant_gbs = q_bytes / (ms_quant * 1e-3) / 1e9
    achieved = kern_bytes / (ms_part * 1e-3) / 1e9
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except OSError:
        pass
    peak = peaks.get("hbm_gbs", 6650.0)
    traffic = None
    prof = os.path.join(ROOT, "profiles", "decode_k4v2_llama3_8b.json")
    if os.path.exists(prof):
        try:
            pj = json.load(open(prof))
            if pj.get("kernel_hash") == kernel_hash() and cfg["name"] == pj.get("config", "llama3_8b"):
                traffic = pj.get("dram_bytes_per_launch")
        except (OSError, ValueError):
            pass
    h2d_bytes = offs[-1]   # the packed input buffer copied each step
    d2h_bytes = out.numel() * out.element_size()
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": PATH_DTYPE[path] + ("; raw key slots bf16" if fd["k_scheme"] == synth.MIXED and
                                     path == "decode_mma_kernel" else ""),
        "data": "synthetic (device-drawn, recipe of synth/)",
        "config": workload_config(cfg),
        "pct_of_8tbs": 100.0 * value / world / 8000.0,
        "decode_gbs": decode_gbs, "quantize_gbs": quant_gbs,
        "tokens_heads_per_s": world * B * Hq * cfg["T"] / ((ms_part + ms_comb) * 1e-3),
        "ms_breakdown": {"quantize": ms_quant, "decode_split": ms_part, "combine": ms_comb,
                         "note": "a separate pass with an event between every two launches"},
        "full_cache_quantize": full_quant,
        "roofline": {"kernel": f"{path} (kvq_decode_partial)", "bound": "hbm",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "algorithmic_bytes": kern_bytes,
                     "peak_source": "MEASURED_PEAKS.json hbm_gbs (measured)" if peaks else "fallback"},
        "e2e": {"value": world * step_bytes / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                "ms_per_step": ms_e2e, "steps": e2e_steps,
                "mode": "pipelined: step i+1's host-to-device copies on a copy stream overlap step i",
                "serial": {"value": world * step_bytes / (ms_e2e_serial * 1e-3) / 1e9,
                           "ms_per_step": ms_e2e_serial}},
        "gpu_launches": step_launches(cfg, n_app) * args.steps,
        "clocks": clocks,
    }
    if path not in ("decode_mma_kernel", "decode_k4v2_kernel"):
        line["roofline"]["traffic"] = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if fd["k_scheme"] == synth.KQV:   # the oracle times the cache schemes of oracle.cache only
            line["cpu_baseline"] = None
        else:
            line["cpu_baseline"] = cpu_baseline(cfg)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def kernel_hash():
    import hashlib
    p = os.path.join(ROOT, "quantized_decode_attention_quantize_b200", "csrc", "decode_mma.cu")
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


if __name__ == "__main__":
    main()
