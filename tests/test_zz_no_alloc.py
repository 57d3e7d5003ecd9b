"""fc_attention_noalloc: the entry point for callers that cannot allocate
device memory (and so cannot create a handle, whose workspace fc_create
allocates).  Its scratch is a static device array shared by every call.

* Two calls in a row on the same step match fc_step's output and importance
  (the second call checks that the shared scratch is cleared between calls).
* Against the fp64 oracle's attention on the same queries and caches: bf16
  with head_dim 128 and 64, fp32 at the fp32 tolerance, and a ragged batch
  that holds a sequence without query rows, one with query rows but an empty
  cache (its rows are zero), a single-row cache and an odd head count.

Collected last, so that a run stopping at the first failure has already run
every other test."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from kv_cache_attention_qkv_b200 import binding, workloads
import fc_testlib as tl

pytestmark = pytest.mark.gpu


def _rotated_q(inp):
    """Projected and rotated queries of every row (fp64 oracle)."""
    q = np.empty((inp.total_q, inp.n_heads, inp.head_dim))
    for b in range(inp.batch):
        qs = inp.seq_slice_q(b)
        qb, _, _ = oracle.qkv_project(inp.x[qs], inp.w_qkv, inp.n_heads, inp.head_dim)
        q[qs] = oracle.rope_rotate(qb, inp.q_pos[qs], inp.rope_theta)
    return q


def _call(lib, dtype, q, cu_q, cu_k, kc, vc, H, d):
    """One fc_attention_noalloc call on device tensors; returns (out, importance)."""
    T, S, B = q.shape[0], kc.shape[0], cu_q.shape[0] - 1
    out = torch.full((T, H, d), float("nan"), device="cuda", dtype=q.dtype)
    imp = torch.full((S,), float("nan"), device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.fc_attention_noalloc(stream, dtype, B, H, d, p(q), p(cu_q), p(cu_k), T, S, p(kc),
                                  p(vc), p(out), p(imp))
    assert st == 0, binding.STATUS.get(st, st)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), imp.cpu().numpy().astype(np.float64)


def _oracle(q, k, v, cu_q, cu_k):
    """The oracle's attention and importance per sequence (inputs as fp64);
    rows of a sequence without cache rows are zero (an empty sum)."""
    T, H, d = q.shape
    out = np.zeros((T, H, d))
    imp = np.zeros(k.shape[0])
    for b in range(len(cu_q) - 1):
        qs, ks = slice(cu_q[b], cu_q[b + 1]), slice(cu_k[b], cu_k[b + 1])
        if qs.stop == qs.start or ks.stop == ks.start:
            continue
        o, P = oracle.attend_sequence(q[qs], k[ks], v[ks])
        out[qs] = o
        imp[ks] = P.sum(axis=(0, 1))
    return out, imp


def _check_against_oracle(q, k, v, cu_q, cu_k, dtype, tol):
    """Upload (bf16 or fp32), run the entry point, compare per sequence."""
    dt = torch.bfloat16 if dtype == binding.FC_DTYPE_BF16 else torch.float32
    dv = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to("cuda", dtype=dt)
    qd, kd, vd = dv(q), dv(k), dv(v)
    f64 = lambda t: t.float().cpu().numpy().astype(np.float64)  # the values the kernel sees
    ref_o, ref_i = _oracle(f64(qd), f64(kd), f64(vd), cu_q, cu_k)
    i32 = lambda a: torch.from_numpy(np.asarray(a, np.int32)).cuda()
    H, d = q.shape[1], q.shape[2]
    out, imp = _call(binding.load_library(), dtype, qd, i32(cu_q), i32(cu_k), kd, vd, H, d)
    for b in range(len(cu_q) - 1):
        qs, ks = slice(cu_q[b], cu_q[b + 1]), slice(cu_k[b], cu_k[b + 1])
        if qs.stop > qs.start:
            if ks.stop > ks.start:
                tl.assert_close(out[qs], ref_o[qs], tol, f"out[seq {b}]")
            else:
                assert (out[qs] == 0).all(), f"seq {b}: rows without a cache must be zero"
        if ks.stop > ks.start:
            if qs.stop > qs.start:
                tl.assert_close(imp[ks], ref_i[ks], tol, f"importance[seq {b}]")
            else:
                assert (imp[ks] == 0).all(), f"seq {b}: keys without query rows"
    return out, imp


def test_noalloc_matches_fc_step_on_two_calls(cuda_ok):
    inp = workloads.generate("small_varlen")
    ref = tl.run_gpu(inp)  # fc_step: refreshes the caches in place, out + importance
    assert ref["err"] == 0
    dev = ref["dev"]
    q = torch.from_numpy(_rotated_q(inp)).to(device="cuda", dtype=torch.bfloat16)
    lib = binding.load_library()
    H, d = inp.n_heads, inp.head_dim
    for call in range(2):
        out, imp = _call(lib, binding.FC_DTYPE_BF16, q, dev["cu_q"], dev["cu_k"], dev["k_cache"],
                         dev["v_cache"], H, d)
        tl.assert_close(out, ref["out"], tl.TOL["bf16"], f"out (call {call})")
        tl.assert_close(imp, ref["importance"], tl.TOL["bf16"], f"importance (call {call})")


@pytest.mark.parametrize("name", ["small_varlen", "small_d64", "tiny_fp32"])
def test_noalloc_against_the_oracle(cuda_ok, name):
    """The workload's rotated queries over its prior caches (bf16 head_dim 128
    and 64; fp32 at the fp32 tolerance)."""
    inp = workloads.generate(name)
    dtype = binding.FC_DTYPE_BF16 if inp.dtype == "bf16" else binding.FC_DTYPE_FP32
    _check_against_oracle(_rotated_q(inp), inp.k_cache, inp.v_cache, inp.cu_seqlens_q,
                          inp.cu_seqlens_k, dtype, tl.TOL[inp.dtype])


def test_noalloc_ragged_batch_with_empty_sequences(cuda_ok):
    """Five sequences, three heads: 37 rows over 300 keys, no rows over 50 keys,
    20 rows over an empty cache, 16 rows over one key, 9 rows over 129 keys."""
    rng = np.random.default_rng(5)
    n, L, H, d = np.array([37, 0, 20, 16, 9]), np.array([300, 50, 0, 1, 129]), 3, 128
    cu_q = np.r_[0, np.cumsum(n)].astype(np.int32)
    cu_k = np.r_[0, np.cumsum(L)].astype(np.int32)
    q = rng.standard_normal((cu_q[-1], H, d))
    k = rng.standard_normal((cu_k[-1], H, d))
    v = rng.standard_normal((cu_k[-1], H, d))
    out, _ = _check_against_oracle(q, k, v, cu_q, cu_k, binding.FC_DTYPE_BF16, tl.TOL["bf16"])
    # one key: every row's output is that key's value row (bf16-rounded)
    vb = torch.from_numpy(v[cu_k[3]].astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.allclose(out[cu_q[3]:cu_q[4]], vb[None], rtol=0, atol=1e-2 * np.abs(vb).max())


def test_noalloc_skips_a_sequence_outside_the_arrays(cuda_ok):
    """A sequence whose cache range leaves [0, total_k) is skipped: its rows
    keep their prior bytes, and the keys inside the range get no importance
    from it; the other sequence is computed as usual."""
    rng = np.random.default_rng(6)
    H, d, S = 2, 128, 60
    cu_q = np.array([0, 24, 40], np.int32)
    cu_k = np.array([0, 40, 80], np.int32)  # sequence 1 claims rows 40..79 of 60
    dv = lambda a: torch.from_numpy(a.astype(np.float32)).to("cuda", dtype=torch.bfloat16)
    q, k, v = (dv(rng.standard_normal(s)) for s in ((40, H, d), (80, H, d), (80, H, d)))
    out = torch.full((40, H, d), float("nan"), device="cuda", dtype=torch.bfloat16)
    imp = torch.full((S,), float("nan"), device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    cq, ck = torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda()  # kept alive
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = binding.load_library().fc_attention_noalloc(
        stream, binding.FC_DTYPE_BF16, 2, H, d, p(q), p(cq), p(ck), 40, S, p(k), p(v), p(out),
        p(imp))
    assert st == 0
    torch.cuda.synchronize()
    o = out.float().cpu().numpy()
    im = imp.cpu().numpy().astype(np.float64)
    assert np.isnan(o[24:]).all()
    assert (im[40:] == 0).all()
    f64 = lambda t: t.float().cpu().numpy().astype(np.float64)
    ro, P = oracle.attend_sequence(f64(q)[:24], f64(k)[:40], f64(v)[:40])
    tl.assert_close(o[:24], ro, tl.TOL["bf16"], "out[seq 0]")
    tl.assert_close(im[:40], P.sum(axis=(0, 1)), tl.TOL["bf16"], "importance[seq 0]")
