"""Sequence-split decode over ranks ([KVQ] "Approach": contexts too long for one GPU are
spread over several).

Each rank holds the cache of its own disjoint range of tokens (rank 0 the attention sink,
the last rank the residual window, every rank a run of packed groups) and runs the
split kernel and the combine over it, which yields its part of the output and the log
of its softmax denominator.  One all-gather of those (head_dim + 1) fp32 values per
query row crosses NVLink (NCCL), and every rank merges the parts with the library's
merge kernel.  Keys must not take RoPE here: a rank's cache positions are its own.

Argument marshalling and the collective only; every step of the arithmetic runs in
libkvq.so.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import kvq


def gather_states(out: torch.Tensor, lse: torch.Tensor, group=None):
    """All-gather (out [..., D], lse [...]) of every rank, in rank order, as one packed
    buffer per rank: returns outs [world, ..., D] and lses [world, ...]."""
    world = dist.get_world_size(group)
    packed = torch.cat([out.reshape(-1).float(), lse.reshape(-1).float()])
    parts = [torch.empty_like(packed) for _ in range(world)]
    dist.all_gather(parts, packed, group=group)
    allp = torch.stack(parts)
    n = out.numel()
    return allp[:, :n].reshape(world, *out.shape), allp[:, n:].reshape(world, *lse.shape)


def decode_local(fmt, cache: kvq.Cache, q: torch.Tensor, t_quant: int, t_res: int, scale: float,
                 num_splits=0, status=None, stream=None):
    """This rank's part: out [B, Hq, D] fp32 and lse [B, Hq] fp32 over its own tokens."""
    B, Hq, D = q.shape
    need = kvq.decode_workspace_bytes(fmt, B, Hq, cache.H, t_quant, t_res, num_splits)
    # the buffers belong to the stream the kernels run on, so that the caching allocator
    # does not hand them out again while those kernels may still use them
    with torch.cuda.stream(stream if stream is not None else torch.cuda.current_stream(q.device)):
        ws = torch.empty(max(16, need), dtype=torch.uint8, device=q.device)
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=q.device)
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    kvq.decode_partial(fmt, cache, q, t_quant, t_res, scale, ws, num_splits=num_splits, status=status,
                       stream=stream)
    kvq.decode_combine_lse(fmt, B, Hq, cache.H, t_quant, t_res, ws, out, lse, num_splits=num_splits,
                           stream=stream)
    return out, lse


def decode_sequence_split(fmt, cache: kvq.Cache, q: torch.Tensor, t_quant: int, t_res: int,
                          scale: float, out_dtype=kvq.F32, group=None, num_splits=0, status=None,
                          stream=None):
    """Decode attention over the union of every rank's tokens; the same result on every rank."""
    if fmt.rope:
        raise ValueError("sequence split needs keys without RoPE (positions are per rank)")
    out, lse = decode_local(fmt, cache, q, t_quant, t_res, scale, num_splits, status, stream)
    outs, lses = gather_states(out, lse, group)
    return kvq.merge_states(outs.contiguous(), lses.contiguous(), out_dtype, stream=stream)
