"""The collective of the sequence-split decode on CPU: two gloo ranks gather their
(out, lse) parts in rank order with one all-gather each, and the gathered parts merge
(by the oracle's merge of disjoint token sets) to the attention over the union of the
ranks' tokens.  The merge kernel itself runs in the GPU tests."""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _parts():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((3, 16))
    K = rng.standard_normal((2, 40, 16))   # rank r holds tokens 40 r .. 40 r + 39
    V = rng.standard_normal((2, 40, 16))
    return q, K, V


def _rank(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    from datetime import timedelta

    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    from oracle.attention import attention_lse
    from quantized_decode_attention_quantize_b200 import seqsplit
    q, K, V = _parts()
    o, l = attention_lse(q, K[rank], V[rank], 0.25)
    outs, lses = seqsplit.gather_states(torch.tensor(o, dtype=torch.float32),
                                        torch.tensor(l, dtype=torch.float32))
    dist.destroy_process_group()
    out_q.put((rank, outs.numpy(), lses.numpy()))


def test_gather_states_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out_q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in procs:
        r, outs, lses = out_q.get(timeout=120)
        got[r] = (outs, lses)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    from oracle.attention import attention_lse, merge_parts
    q, K, V = _parts()
    # both ranks hold the same gathered parts, in rank order
    np.testing.assert_array_equal(got[0][0], got[1][0])
    np.testing.assert_array_equal(got[0][1], got[1][1])
    for r in range(2):
        o, l = attention_lse(q, K[r], V[r], 0.25)
        np.testing.assert_allclose(got[0][0][r], o, rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(got[0][1][r], l, rtol=1e-6, atol=1e-6)
    merged, lse = merge_parts(got[0][0], got[0][1])
    whole, whole_lse = attention_lse(q, K.reshape(80, 16), V.reshape(80, 16), 0.25)
    np.testing.assert_allclose(merged, whole, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(lse, whole_lse, rtol=1e-6, atol=1e-6)
