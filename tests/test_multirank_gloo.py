"""Multi-rank host logic on CPU with the gloo backend (world size 2).

Each rank takes its block of sequences of a packed batch, runs the oracle on
it, and the gathered per-rank results must equal the unsharded step exactly
(sequences are independent, so sharding needs no collective on the data path).
The timing reduction (max over ranks) is checked too.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from kv_cache_attention_qkv_b200 import shard, workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_q):
    import torch.distributed as dist

    import oracle

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = workloads.generate("small_varlen")
        mine = shard.shard_batch(inp, rank, world)
        res = oracle.flashcache_step(mine.x, mine.w_qkv, mine.q_pos, mine.cu_seqlens_q,
                                     mine.cu_seqlens_k, mine.k_cache, mine.v_cache,
                                     mine.n_heads, mine.head_dim, mine.rope_theta, mine.dtype)
        tracked = oracle.topk_tracked(res["importance"], mine.cu_seqlens_k, mine.cand_lo,
                                      mine.cand_hi, mine.topk, int(inp.topk.max()))
        gathered = [None] * world
        dist.all_gather_object(gathered, (res["out"], res["importance"], tracked))
        slowest = shard.max_over_ranks(10.0 + rank)
        pair = shard.max_over_ranks([5.0 - rank, 7.0 + 2 * rank])
        if rank == 0:
            out_q.put((gathered, (slowest, pair)))
    finally:
        dist.destroy_process_group()


def test_sharded_oracle_matches_unsharded():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    gathered, (slowest, pair) = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    import oracle

    inp = workloads.generate("small_varlen")
    full = oracle.flashcache_step(inp.x, inp.w_qkv, inp.q_pos, inp.cu_seqlens_q, inp.cu_seqlens_k,
                                  inp.k_cache, inp.v_cache, inp.n_heads, inp.head_dim,
                                  inp.rope_theta, inp.dtype)
    tracked = oracle.topk_tracked(full["importance"], inp.cu_seqlens_k, inp.cand_lo, inp.cand_hi,
                                  inp.topk, int(inp.topk.max()))
    np.testing.assert_array_equal(np.concatenate([g[0] for g in gathered]), full["out"])
    np.testing.assert_array_equal(np.concatenate([g[1] for g in gathered]), full["importance"])
    np.testing.assert_array_equal(np.concatenate([g[2] for g in gathered]), tracked)
    assert slowest == 11.0
    assert pair == [5.0, 9.0]  # element-wise over the ranks


@pytest.mark.parametrize("batch,world", [(32, 8), (3, 2), (5, 4), (1, 1)])
def test_shard_bounds_cover_the_batch(batch, world):
    spans = [shard.shard_bounds(batch, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == batch
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1
