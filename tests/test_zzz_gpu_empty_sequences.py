"""GPU parity on packed batches that contain empty sequences: a sequence with
a cache but no query rows, and one with neither (zero-length cache, no
candidates).  Nothing is written for them, their keys get zero importance and
their tracked rows are the lowest candidates (all tie at zero) or all -1."""
import numpy as np
import pytest

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
