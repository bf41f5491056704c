"""GPU test of kvq_decode_attention_noalloc, the decode entry point for callers that
cannot allocate device memory (it uses a scratch array inside the library instead of
a caller workspace).  Collected last on purpose: a run that stops at the first failure
has run every other test before this one.  Checks the output of two calls in a row
against kvq_decode_attention on the same inputs: both run the same kernels on the same
inputs, so the outputs are equal bit for bit."""
import numpy as np
import pytest
import torch

from oracle.formats import BF16, F16, F32
from quantized_decode_attention_quantize_b200 import kvq
from tests.gpu_util import dev
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
    for o in outs:
        assert torch.equal(o, want)

