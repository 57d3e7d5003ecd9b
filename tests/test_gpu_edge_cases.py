"""GPU parity on edge cases of the packed layout and of the reselection.

* Packed batches that contain empty sequences: a sequence with a cache but no
  query rows, and one with neither (zero-length cache, no candidates).  Nothing
  is written for them, their keys get zero importance and their tracked rows
  are the lowest candidates (all tie at zero) or all -1.
* Top-k over candidate ranges longer than the kernel's shared-memory stage
  (8192 keys), at the largest supported k (1024), with many planted ties.
"""
import numpy as np
import pytest
import torch

import oracle

from kv_cache_attention_qkv_b200 import workloads
import fc_testlib as tl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu(cuda_ok):
    return cuda_ok


def _drop_rows_of(inp, b, drop_cache):
    """small_varlen with sequence b's query rows (and, if asked, its cache) removed."""
    qs, ks = inp.seq_slice_q(b), inp.seq_slice_k(b)
    keep_q = np.r_[0:qs.start, qs.stop:inp.total_q]
    inp.x, inp.q_pos = inp.x[keep_q], inp.q_pos[keep_q]
    n = np.diff(inp.cu_seqlens_q)
    n[b] = 0
    inp.cu_seqlens_q = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    if drop_cache:
        keep_k = np.r_[0:ks.start, ks.stop:inp.total_k]
        inp.k_cache, inp.v_cache = inp.k_cache[keep_k], inp.v_cache[keep_k]
        L = np.diff(inp.cu_seqlens_k)
        L[b] = 0
        inp.cu_seqlens_k = np.concatenate([[0], np.cumsum(L)]).astype(np.int32)
        inp.cand_lo[b] = inp.cand_hi[b] = 0
    return inp


@pytest.mark.parametrize("drop_cache", [False, True], ids=["no_rows", "no_rows_no_cache"])
def test_empty_sequence_inside_a_ragged_batch(drop_cache):
    inp = _drop_rows_of(workloads.generate("small_varlen"), 1, drop_cache)
    gpu = tl.run_gpu(inp)
    assert gpu["err"] == 0
    ref = tl.run_oracle(inp)
    tl.compare_step(inp, gpu, ref, range(inp.batch))
    tl.assert_unwritten_rows_unchanged(inp, gpu)
    ks = inp.seq_slice_k(1)
    assert (gpu["importance"][ks] == 0.0).all()
    K = int(inp.topk[1])
    want = [-1] * K if drop_cache else list(range(int(inp.cand_lo[1]), int(inp.cand_lo[1]) + K))
    assert gpu["tracked"][1][:K].tolist() == want


def test_topk_beyond_the_staged_candidates_at_the_largest_k():
    rng = np.random.default_rng(11)
    L = np.array([20000, 9000, 300], np.int64)
    cu = np.zeros(len(L) + 1, np.int32)
    cu[1:] = np.cumsum(L)
    # multiples of 1/8 below 64: every value repeats many times, so the k-th
    # score is shared by a run of candidates and ties go by position
    imp = (rng.integers(0, 512, cu[-1]) * 0.125).astype(np.float32)
    lo = np.array([100, 0, 0], np.int32)
    hi = np.array([19900, 9000, 300], np.int32)   # 19800 and 9000 candidates: not staged
    K = 1024
    kb = np.array([1024, 700, 1024], np.int32)    # the last sequence has fewer candidates than k
    inp = workloads.generate("tiny_fp32")
    dev = tl.upload(inp)
    layer = tl.make_layer(inp, dev["w"], max_topk=K, max_total_k=int(cu[-1]), max_pos=int(L.max()),
                          max_batch=len(L))
    t = lambda a: torch.from_numpy(a).cuda()
    tracked = torch.full((len(L), K), -7, dtype=torch.int32, device="cuda")
    layer.topk_tracked(t(imp), t(cu), t(lo), t(hi), K, tracked, k_per_seq=t(kb))
    assert layer.get_error() == 0
    ref = oracle.topk_tracked(imp.astype(np.float64), cu, lo, hi, kb, K)
    np.testing.assert_array_equal(tracked.cpu().numpy(), ref)
