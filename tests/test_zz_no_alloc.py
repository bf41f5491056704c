"""GPU test of kvq_decode_attention_noalloc, the decode entry point for callers that
cannot allocate device memory (it uses a scratch array inside the library instead of
a caller workspace).  Collected last on purpose: a run that stops at the first failure
has run every other test before this one.  Checks the output of two calls in a row
against kvq_decode_attention on the same inputs, within the decode tolerance."""
import numpy as np
import pytest
import torch

import synth
from oracle.formats import BF16, F16, F32
from quantized_decode_attention_quantize_b200 import kvq
from tests.gpu_util import dev, rel_l2, tolerance
from tests.test_gpu_decode import build, fmt, vals

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("G,src,out_dtype", [(4, BF16, F32), (1, F16, BF16), (5, BF16, F32)])
def test_noalloc_matches_workspace_entry_point(G, src, out_dtype):
    B, H, tq, tr = 2, 3, 5 * 128 + 19, 21
    fd = fmt(src_dtype=src, n_sink=1, residual_cap=32)
    p = build(fd, B, H, G * H, tq, tr, seed=70 + G)
    q = dev(vals(80 + G, (B, G * H, 128), src), src)
    scale = 1.0 / np.sqrt(128.0)
    want = kvq.decode_attention(p.fmt, p.gpu, q, tq, tr, scale, out_dtype)
    outs = []
    for _ in range(2):   # the scratch keeps the previous call's contents
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        outs.append(kvq.decode_attention_noalloc(p.fmt, p.gpu, q, tq, tr, scale, out_dtype,
                                                 status=status))
        torch.cuda.synchronize()
        assert int(status.item()) == 0
    ref = want.float().cpu().numpy()
    for o in outs:
        assert rel_l2(o.float().cpu().numpy(), ref) <= tolerance(out_dtype)


def test_noalloc_rejects_oversized_requests():
    # a workspace need above the scratch size is refused before anything runs
    fd = fmt(src_dtype=BF16, rope=1)        # the generic path: 64 splits per head as asked
    f = kvq.make_format(fd)
    B, Hq, Hkv, tq = 64, 64, 64, 131072
    need = kvq.decode_workspace_bytes(f, B, Hq, Hkv, tq, 0, 64)
    assert need > kvq.NOALLOC_SCRATCH_BYTES
    cache = kvq.kvq_cache(batch=B, kv_heads=Hkv, capacity=tq)
    for i, n in enumerate(kvq.ARRAYS):
        setattr(cache, n, 0x10000 * (i + 1))
    import ctypes
    st = kvq.lib().kvq_decode_attention_noalloc(ctypes.byref(f), ctypes.byref(cache), ctypes.c_void_p(0x100000),
                                                kvq.BF16, Hq, tq, 0, 0.1, ctypes.c_void_p(0x200000), kvq.F32,
                                                64, None, None)
    assert st == kvq.KVQ_ERR_WORKSPACE
