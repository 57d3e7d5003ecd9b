"""fc_attention_noalloc: the entry point for callers that cannot allocate
device memory (and so cannot create a handle, whose workspace fc_create
allocates).  Its output must match fc_step's on the same step, on two calls in
a row: the second call checks that the shared static scratch is cleared
between calls.  Collected last so that a run stopping at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from kv_cache_attention_qkv_b200 import binding, workloads
import fc_testlib as tl

pytestmark = pytest.mark.gpu


def _rotated_q(inp):
    """Projected and rotated queries of every row (fp64 oracle -> bf16)."""
    q = np.empty((inp.total_q, inp.n_heads, inp.head_dim))
    for b in range(inp.batch):
        qs = inp.seq_slice_q(b)
        qb, _, _ = oracle.qkv_project(inp.x[qs], inp.w_qkv, inp.n_heads, inp.head_dim)
        q[qs] = oracle.rope_rotate(qb, inp.q_pos[qs], inp.rope_theta)
    return torch.from_numpy(q).to(device="cuda", dtype=torch.bfloat16)


def test_noalloc_matches_fc_step_on_two_calls(cuda_ok):
    inp = workloads.generate("small_varlen")
    ref = tl.run_gpu(inp)  # fc_step: refreshes the caches in place, out + importance
    assert ref["err"] == 0
    dev = ref["dev"]
    q = _rotated_q(inp)
    lib = binding.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    T, S, H, d, B = inp.total_q, inp.total_k, inp.n_heads, inp.head_dim, inp.batch
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    for call in range(2):
        out = torch.full((T, H, d), float("nan"), device="cuda", dtype=torch.bfloat16)
        imp = torch.full((S,), float("nan"), device="cuda")
        st = lib.fc_attention_noalloc(stream, binding.FC_DTYPE_BF16, B, H, d, p(q), p(dev["cu_q"]),
                                      p(dev["cu_k"]), T, S, p(dev["k_cache"]), p(dev["v_cache"]),
                                      p(out), p(imp))
        assert st == 0, binding.STATUS.get(st, st)
        torch.cuda.synchronize()
        tl.assert_close(out.float().cpu().numpy(), ref["out"], tl.TOL["bf16"], f"out (call {call})")
        tl.assert_close(imp.cpu().numpy(), ref["importance"], tl.TOL["bf16"],
                        f"importance (call {call})")


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_ok):
    lib = binding.load_library()
    too_many_keys = 65536 + 1  # FC_NOALLOC_MAX_KEYS + 1
    vp = ctypes.c_void_p(16)
    st = lib.fc_attention_noalloc(None, binding.FC_DTYPE_BF16, 1, 1, 128, vp, vp, vp, 1,
                                  too_many_keys, vp, vp, vp, vp)
    assert st == -2  # FC_ERR_UNSUPPORTED, nothing queued
