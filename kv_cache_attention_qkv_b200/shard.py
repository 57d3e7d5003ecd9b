"""Sequence sharding of a packed batch across ranks.

A Flash-Cache step touches, for sequence b, only its own query rows and its
own cache rows (W_qkv is shared and read-only), so a batch splits across GPUs
by whole sequences with no data exchange.  ``shard_batch`` cuts a packed batch
into the rank's contiguous block of sequences and re-bases the length arrays;
``max_over_ranks`` is the timing reduction (the slowest rank sets the time).
"""
from __future__ import annotations

import dataclasses

import numpy as np


def shard_bounds(batch: int, rank: int, world: int):
    """[first, last) sequence indices of ``rank`` (block split, sizes differ by <= 1)."""
    base, extra = divmod(batch, world)
    first = rank * base + min(rank, extra)
    return first, first + base + (1 if rank < extra else 0)


def shard_batch(inp, rank: int, world: int):
    """The rank's sequences of a packed StepInputs, with re-based cu_seqlens."""
    b0, b1 = shard_bounds(inp.batch, rank, world)
    q0, q1 = int(inp.cu_seqlens_q[b0]), int(inp.cu_seqlens_q[b1])
    k0, k1 = int(inp.cu_seqlens_k[b0]), int(inp.cu_seqlens_k[b1])
    return dataclasses.replace(
        inp,
        x=inp.x[q0:q1], q_pos=inp.q_pos[q0:q1],
        k_cache=inp.k_cache[k0:k1], v_cache=inp.v_cache[k0:k1],
        cu_seqlens_q=(inp.cu_seqlens_q[b0:b1 + 1] - q0).astype(np.int32),
        cu_seqlens_k=(inp.cu_seqlens_k[b0:b1 + 1] - k0).astype(np.int32),
        cand_lo=inp.cand_lo[b0:b1], cand_hi=inp.cand_hi[b0:b1], topk=inp.topk[b0:b1],
        window_start=inp.window_start[b0:b1], window_len=inp.window_len[b0:b1],
    )


def max_over_ranks(value, device=None):
    """All-reduce MAX over the default process group of a scalar (returns a
    float) or of a sequence of scalars (returns a list, element-wise)."""
    import torch
    import torch.distributed as dist

    many = isinstance(value, (list, tuple))
    vals = [float(v) for v in value] if many else [float(value)]
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    out = [float(v) for v in t.tolist()]
    return out if many else out[0]
