"""The algorithmic byte counts behind the benchmark's roofline, recomputed from the
packed format's own byte accounting (oracle.formats) on CPU: a K4/V2 token costs 64 B of
key codes, 32 B of value codes and 4 B of value scale / zero-point per KV head, a key
group 512 B of per-channel metadata, a raw token 2 x 128 x 2 B, and the queries are read
once."""
import sys
import os

import pytest

import synth
from oracle import formats

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("name", ["llama3_8b", "llama2_7b", "llama3_8b_wht"])
def test_decode_bytes_follow_the_format(name):
    cfg = synth.CONFIGS[name]
    f = formats.Format(**cfg["fmt"])
    ns, tq, tr = synth.split_tokens(cfg)
    g, D = f.group_tokens, f.head_dim
    ngv = -(-tq // g)
    per_token = formats.code_row_bytes(f, formats.KEYS) + formats.code_row_bytes(f, formats.VALUES) + 4
    per_group = 2 * 2 * D                      # fp16 key scale and zero-point per channel
    raw = 2 * D * formats.DTYPE_BYTES[f.src_dtype]
    per_head = tq * per_token + ngv * per_group + (ns + tr) * raw
    q = cfg["B"] * cfg["Hq"] * D * formats.DTYPE_BYTES[cfg["q_dtype"]]
    assert per_token == 100
    assert bench.decode_kernel_bytes(cfg, tq, tr) == cfg["B"] * cfg["Hkv"] * per_head + q
    assert bench.decode_call_bytes(cfg, tq, tr) == bench.decode_kernel_bytes(cfg, tq, tr) + \
        cfg["B"] * cfg["Hq"] * D * 4


def test_headline_figures():
    cfg = synth.CONFIGS["llama3_8b"]
    ns, tq, tr = synth.split_tokens(cfg)
    assert (ns, tq, tr) == (1, 32639, 128)
    assert bench.decode_kernel_bytes(cfg, tq, tr) == 221538048
    # one 128-token append: bf16 K and V read, codes and metadata written
    assert bench.quant_bytes(cfg, 128) == 64 * (128 * 128 * 2 * 2 + 128 * 100 + 512)


def test_decode_path_matches_the_planner_rules():
    assert bench.decode_path(synth.CONFIGS["llama3_8b"]) == "decode_k4v2_kernel"
    assert bench.decode_path(synth.CONFIGS["llama3_8b_kqv"]) == "decode_kqv_kernel"
    assert bench.decode_path(synth.CONFIGS["mixkvq_14b"]) == "decode_mma_kernel"
    assert bench.decode_path(synth.CONFIGS["kvquant_nuq3"]) == "decode_cc_kernel"
    assert bench.fused_kv(synth.CONFIGS["llama3_8b_wht"])
    assert not bench.fused_kv(synth.CONFIGS["mixkvq_14b"])
