"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against a closed form, a library routine, an
invariant the mathematics fixes, or brute force; they are chosen so that a
dropped term, a wrong sign or index, or a transposed operand fails one.
CPU only.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_attention_qkv_b200 import workloads


def _rng(seed=123):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------- bf16 rounding
def test_bf16_round_matches_torch_conversion():
    rng = _rng(1)
    vals = rng.standard_normal(200000).astype(np.float32) * np.float32(3.0)
    vals = np.concatenate([vals, (rng.standard_normal(2000) * 1e6).astype(np.float32),
                           (rng.standard_normal(2000) * 1e-6).astype(np.float32)])
    # exact halfway cases: low 16 bits = 0x8000, both parities of the kept lsb
    bits = rng.integers(0x3C000000, 0x42000000, size=4000, dtype=np.uint32)
    bits = (bits & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    vals = np.concatenate([vals, bits.view(np.float32), -bits.view(np.float32)])
    ref = torch.from_numpy(vals).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.bf16_round(vals.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_bf16_round_zero_and_signs():
    got = oracle.bf16_round(np.array([0.0, -0.0, 1.0, -1.0, 1.0 + 2.0 ** -9, 1.0 + 3 * 2.0 ** -9]))
    # 1 + 2^-9 is halfway between 1 and 1 + 2^-8: ties go to the even (1.0);
    # 1 + 3*2^-9 is halfway between 1 + 2^-8 and 1 + 2^-7: even is 1 + 2^-7.
    np.testing.assert_array_equal(got, [0.0, 0.0, 1.0, -1.0, 1.0, 1.0 + 2.0 ** -7])


# ----------------------------------------------------------------- RoPE
def test_rope_d2_closed_form():
    # d = 2: one pair, frequency theta**0 = 1, so the angle is the position.
    pos = np.array([0, 1, 5, 37], np.int64)
    u = np.tile(np.array([[[1.0, 0.0]]]), (4, 1, 1))
    r = oracle.rope_rotate(u, pos, theta=1.0e4)
    np.testing.assert_allclose(r[:, 0, 0], np.cos(pos), atol=1e-15)
    np.testing.assert_allclose(r[:, 0, 1], np.sin(pos), atol=1e-15)


def test_rope_frequency_ladder():
    d, theta = 16, 1.0e4
    a = oracle.rope_angles(np.array([1.0]), d, theta)[0]
    assert a[0] == 1.0
    np.testing.assert_allclose(a[1:] / a[:-1], theta ** (-2.0 / d), rtol=1e-14)
    assert a.shape == (d // 2,)


def test_rope_identity_at_position_zero():
    u = _rng(2).standard_normal((5, 3, 8))
    np.testing.assert_array_equal(oracle.rope_rotate(u, np.zeros(5, np.int64), 500000.0), u)


def test_rope_preserves_norm():
    u = _rng(3).standard_normal((64, 4, 128))
    pos = _rng(4).integers(0, 4096, 64)
    r = oracle.rope_rotate(u, pos, 500000.0)
    np.testing.assert_allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(u, axis=-1), rtol=1e-13)


def test_rope_dot_product_depends_only_on_offset():
    rng = _rng(5)
    q = rng.standard_normal((1, 2, 32))
    k = rng.standard_normal((1, 2, 32))
    for p, pk, c in [(3, 10, 7), (100, 2, 1000), (0, 0, 12345)]:
        a = (oracle.rope_rotate(q, np.array([p]), 1e4) * oracle.rope_rotate(k, np.array([pk]), 1e4)).sum(-1)
        b = (oracle.rope_rotate(q, np.array([p + c]), 1e4) * oracle.rope_rotate(k, np.array([pk + c]), 1e4)).sum(-1)
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-10)


def test_rope_complex_restatement():
    # Rotate-half RoPE is multiplication of z_i = u_i + i*u_{i+d/2} by exp(i*a_i).
    rng = _rng(6)
    d, theta = 64, 5.0e5
    u = rng.standard_normal((9, 2, d))
    pos = rng.integers(0, 3000, 9)
    z = u[..., : d // 2] + 1j * u[..., d // 2:]
    freq = np.power(theta, -np.arange(0, d, 2) / d)
    z = z * np.exp(1j * np.outer(pos, freq))[:, None, :]
    ref = np.concatenate([z.real, z.imag], axis=-1)
    np.testing.assert_allclose(oracle.rope_rotate(u, pos, theta), ref, atol=1e-12)


# ----------------------------------------------------------------- attention
def _torch_sdpa(q, k, v):
    """Library bidirectional attention in fp64: q [n,H,d], k/v [L,H,d]."""
    tq = torch.from_numpy(q).permute(1, 0, 2)[None]
    tk = torch.from_numpy(k).permute(1, 0, 2)[None]
    tv = torch.from_numpy(v).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=False)
    return o[0].permute(1, 0, 2).numpy()


def _torch_rope(u, pos, theta):
    t = torch.from_numpy(u)
    d = t.shape[-1]
    z = torch.complex(t[..., : d // 2], t[..., d // 2:])
    ang = torch.from_numpy(np.asarray(pos, np.float64))[:, None] * torch.pow(
        torch.tensor(theta, dtype=torch.float64), -torch.arange(0, d, 2, dtype=torch.float64) / d)
    z = z * torch.polar(torch.ones_like(ang), ang)[:, None, :]
    return torch.cat([z.real, z.imag], dim=-1).numpy()


@pytest.mark.parametrize("L,H,d,D", [(24, 3, 8, 20), (7, 1, 16, 5), (40, 2, 32, 48)])
def test_full_coverage_equals_uncached_attention(L, H, d, D):
    """Query covering every position == plain bidirectional attention on X."""
    rng = _rng(L * 7 + d)
    x = rng.standard_normal((L, D))
    w = rng.standard_normal((3 * H * d, D)) * 0.3
    pos = rng.permutation(L)
    stale_k = rng.standard_normal((L, H, d)) * 50.0  # must be fully overwritten
    stale_v = rng.standard_normal((L, H, d)) * 50.0
    theta = 1.0e4
    res = oracle.step_sequence(x, w, pos, stale_k, stale_v, H, d, theta, None)

    tx, tw = torch.from_numpy(x), torch.from_numpy(w)
    y = (tx @ tw.T).numpy()
    hd = H * d
    q = _torch_rope(y[:, :hd].reshape(L, H, d), pos, theta)
    k = _torch_rope(y[:, hd:2 * hd].reshape(L, H, d), pos, theta)
    v = y[:, 2 * hd:].reshape(L, H, d)
    ref = _torch_sdpa(q, k[np.argsort(pos)], v[np.argsort(pos)])
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-12)
    kc = np.empty_like(k)
    kc[pos] = k
    vc = np.empty_like(v)
    vc[pos] = v
    np.testing.assert_allclose(res["k_cache"], kc, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res["v_cache"], vc, rtol=1e-12, atol=1e-12)


def test_partial_query_matches_sdpa_over_stored_cache():
    """A partial query attends over fresh rows plus the stale rows as stored."""
    rng = _rng(11)
    L, H, d, D, n = 30, 2, 8, 12, 6
    x = rng.standard_normal((n, D))
    w = rng.standard_normal((3 * H * d, D)) * 0.4
    pos = rng.choice(L, n, replace=False)
    kc = rng.standard_normal((L, H, d))
    vc = rng.standard_normal((L, H, d))
    res = oracle.step_sequence(x, w, pos, kc, vc, H, d, 1e4, "bf16")
    y = x @ w.T
    hd = H * d
    q = _torch_rope(y[:, :hd].reshape(n, H, d), pos, 1e4)
    k = _torch_rope(y[:, hd:2 * hd].reshape(n, H, d), pos, 1e4)
    kk, vv = kc.copy(), vc.copy()
    kk[pos] = torch.from_numpy(k).to(torch.bfloat16).double().numpy()
    vv[pos] = torch.from_numpy(y[:, 2 * hd:].reshape(n, H, d)).to(torch.bfloat16).double().numpy()
    np.testing.assert_allclose(res["out"], _torch_sdpa(q, kk, vv), rtol=1e-10, atol=1e-12)
    untouched = np.setdiff1d(np.arange(L), pos)
    np.testing.assert_array_equal(res["k_cache"][untouched], kc[untouched])
    np.testing.assert_array_equal(res["v_cache"][untouched], vc[untouched])


def test_softmax_rows_sum_to_one_and_importance_total():
    rng = _rng(12)
    n, L, H, d = 5, 17, 3, 8
    q = rng.standard_normal((n, H, d)) * 4
    k = rng.standard_normal((L, H, d))
    v = rng.standard_normal((L, H, d))
    _, P = oracle.attend_sequence(q, k, v)
    np.testing.assert_allclose(P.sum(axis=2), 1.0, rtol=0, atol=1e-14)
    assert (P >= 0).all()
    res = oracle.step_sequence(rng.standard_normal((n, 10)), rng.standard_normal((3 * H * d, 10)),
                               rng.choice(L, n, replace=False), k, v, H, d, 1e4, None)
    np.testing.assert_allclose(res["importance"].sum(), H * n, rtol=1e-12)


def test_single_key_returns_value():
    rng = _rng(13)
    H, d, D = 2, 8, 6
    x = rng.standard_normal((1, D))
    w = rng.standard_normal((3 * H * d, D))
    res = oracle.step_sequence(x, w, np.array([0]), np.zeros((1, H, d)), np.zeros((1, H, d)),
                               H, d, 1e4, None)
    v = (x @ w.T)[:, 2 * H * d:].reshape(1, H, d)
    np.testing.assert_allclose(res["out"], v, rtol=1e-13)
    np.testing.assert_allclose(res["importance"], [H * 1.0], rtol=1e-14)


def test_zero_query_gives_uniform_attention():
    """x = 0 makes q = 0: every key gets probability 1/L."""
    rng = _rng(14)
    n, L, H, d, D = 4, 9, 2, 8, 5
    kc = rng.standard_normal((L, H, d))
    vc = rng.standard_normal((L, H, d))
    pos = np.array([1, 4, 6, 8])
    res = oracle.step_sequence(np.zeros((n, D)), rng.standard_normal((3 * H * d, D)), pos, kc, vc,
                               H, d, 1e4, None)
    vv = vc.copy()
    vv[pos] = 0.0  # x = 0 also makes the fresh v rows zero
    np.testing.assert_allclose(res["out"], np.broadcast_to(vv.mean(axis=0), (n, H, d)), atol=1e-14)
    np.testing.assert_allclose(res["importance"], np.full(L, H * n / L), rtol=1e-13)


def test_query_row_permutation_equivariance():
    rng = _rng(15)
    n, L, H, d, D = 7, 20, 2, 16, 9
    x = rng.standard_normal((n, D))
    w = rng.standard_normal((3 * H * d, D)) * 0.5
    pos = rng.choice(L, n, replace=False)
    kc, vc = rng.standard_normal((L, H, d)), rng.standard_normal((L, H, d))
    a = oracle.step_sequence(x, w, pos, kc, vc, H, d, 1e4, "bf16")
    perm = rng.permutation(n)
    b = oracle.step_sequence(x[perm], w, pos[perm], kc, vc, H, d, 1e4, "bf16")
    np.testing.assert_allclose(b["out"], a["out"][perm], rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(b["k_cache"], a["k_cache"])
    np.testing.assert_allclose(b["importance"], a["importance"], rtol=1e-12)


def test_sequences_are_independent():
    inp = workloads.generate("small_varlen")
    full = oracle.flashcache_step(inp.x, inp.w_qkv, inp.q_pos, inp.cu_seqlens_q, inp.cu_seqlens_k,
                                  inp.k_cache, inp.v_cache, inp.n_heads, inp.head_dim,
                                  inp.rope_theta, "bf16")
    for b in range(inp.batch):
        qs, ks = inp.seq_slice_q(b), inp.seq_slice_k(b)
        one = oracle.step_sequence(inp.x[qs], inp.w_qkv, inp.q_pos[qs], inp.k_cache[ks],
                                   inp.v_cache[ks], inp.n_heads, inp.head_dim, inp.rope_theta, "bf16")
        np.testing.assert_array_equal(full["out"][qs], one["out"])
        np.testing.assert_array_equal(full["k_cache"][ks], one["k_cache"])
        np.testing.assert_array_equal(full["importance"][ks], one["importance"])


def test_hand_worked_two_token_example():
    """H=1, d=2, identity projections; worked out by hand.

    Rows: x0 = (1, 0) at position 0 and x1 = (0, 1) at position 1, with
    W_q = W_k = W_v = I.  RoPE with d=2 turns by the position itself, so
    q0 = k0 = (1, 0) and q1 = k1 = R(1)(0, 1) = (-sin 1, cos 1); v0 = (1, 0),
    v1 = (0, 1).  The cache has 3 rows; row 2 is stale: K2 = (0, 2), V2 = (0, 3).
    For q0: scores (1, -sin 1, 0)/sqrt 2; for q1: (-sin 1, 1, 2 cos 1)/sqrt 2.
    """
    x = np.array([[1.0, 0.0], [0.0, 1.0]])
    w = np.concatenate([np.eye(2)] * 3, axis=0)
    kc = np.array([[[9.0, 9.0]], [[9.0, 9.0]], [[0.0, 2.0]]])
    vc = np.array([[[9.0, 9.0]], [[9.0, 9.0]], [[0.0, 3.0]]])
    res = oracle.step_sequence(x, w, np.array([0, 1]), kc, vc, 1, 2, 1.0e4, None)
    s1, c1 = math.sin(1.0), math.cos(1.0)
    r2 = math.sqrt(2.0)
    v_rows = [(1.0, 0.0), (0.0, 1.0), (0.0, 3.0)]

    def expect(scores):
        e = [math.exp(s / r2) for s in scores]
        z = sum(e)
        p = [t / z for t in e]
        return p, (sum(pi * v[0] for pi, v in zip(p, v_rows)), sum(pi * v[1] for pi, v in zip(p, v_rows)))

    p0, o0 = expect([1.0, -s1, 0.0])
    p1, o1 = expect([-s1, 1.0, 2.0 * c1])
    np.testing.assert_allclose(res["out"][:, 0, :], [o0, o1], rtol=1e-14)
    np.testing.assert_allclose(res["importance"], np.add(p0, p1), rtol=1e-14)
    np.testing.assert_allclose(res["k_cache"][:, 0, :], [[1.0, 0.0], [-s1, c1], [0.0, 2.0]], atol=1e-16)


def test_oracle_refuses_duplicate_or_out_of_range_positions():
    kc = np.zeros((4, 1, 2))
    with pytest.raises(AssertionError):
        oracle.write_cache(kc, np.array([1, 1]), np.zeros((2, 1, 2)), None)
    with pytest.raises(AssertionError):
        oracle.write_cache(kc, np.array([4]), np.zeros((1, 1, 2)), None)


# ----------------------------------------------------------------- top-k
def _brute_topk(scores, lo, hi, k):
    """Rank by counting: j is kept iff fewer than k candidates beat it."""
    keep = []
    for j in range(lo, hi):
        better = sum(1 for i in range(lo, hi)
                     if scores[i] > scores[j] or (scores[i] == scores[j] and i < j))
        if better < k:
            keep.append((better, j))
    return [j for _, j in sorted(keep)]


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_brute_force_with_ties(seed):
    rng = _rng(100 + seed)
    B = 4
    lens = rng.integers(1, 40, B)
    cu = np.zeros(B + 1, np.int64)
    cu[1:] = np.cumsum(lens)
    imp = rng.integers(0, 6, cu[-1]).astype(np.float64) * 0.25  # many planted ties
    lo = np.array([rng.integers(0, L) for L in lens])
    hi = np.array([rng.integers(l, L + 1) for l, L in zip(lo, lens)])
    kk = rng.integers(0, 12, B)
    width = 12
    got = oracle.topk_tracked(imp, cu, lo, hi, kk, width)
    for b in range(B):
        ref = _brute_topk(imp[cu[b]:cu[b + 1]], int(lo[b]), int(hi[b]), int(kk[b]))
        row = list(got[b])
        assert row[:len(ref)] == ref
        assert all(v == -1 for v in row[len(ref):])


def test_topk_pads_when_fewer_candidates():
    got = oracle.topk_tracked(np.array([0.5, 0.25, 1.0]), np.array([0, 3]), np.array([0]),
                              np.array([2]), np.array([4]), 4)
    assert list(got[0]) == [0, 1, -1, -1]


# ----------------------------------------------------------------- workloads
@pytest.mark.parametrize("name", ["tiny_fp32", "layer_b1", "small_varlen", "small_d64",
                                  "small_longcache"])
def test_workload_structure(name):
    inp = workloads.generate(name)
    assert inp.cu_seqlens_q[0] == 0 and inp.cu_seqlens_k[0] == 0
    assert inp.x.shape == (inp.total_q, inp.hidden)
    assert inp.k_cache.shape == (inp.total_k, inp.n_heads, inp.head_dim)
    for b in range(inp.batch):
        pos = inp.q_pos[inp.seq_slice_q(b)]
        L = inp.cu_seqlens_k[b + 1] - inp.cu_seqlens_k[b]
        assert len(np.unique(pos)) == len(pos) and pos.min() >= 0 and pos.max() < L
        ws, wl = inp.window_start[b], inp.window_len[b]
        tracked = pos[: len(pos) - wl]
        assert (tracked < ws).all() and len(tracked) == inp.topk[b]
        np.testing.assert_array_equal(pos[len(pos) - wl:], np.arange(ws, ws + wl))
        assert inp.cand_lo[b] == 0 and inp.cand_hi[b] == ws
    if inp.dtype == "bf16":
        for a in (inp.x, inp.w_qkv, inp.k_cache):
            np.testing.assert_array_equal(oracle.bf16_round(a.astype(np.float64)), a)


def test_varlen_workload_recipe():
    inp = workloads.generate("batch32_varlen")
    L = np.diff(inp.cu_seqlens_k)
    assert inp.batch == 32 and L.min() >= 600 and L.max() <= 2048
    assert set(np.unique(inp.window_len)) <= {16, 64}
    assert set(np.unique(inp.topk)) <= {48, 64, 80}
    n = np.diff(inp.cu_seqlens_q)
    assert n.min() >= 64 and n.max() <= 144
    assert (inp.window_start % inp.window_len == 0).all()
    assert (inp.window_start >= L - 512).all()
    assert (inp.window_start + inp.window_len <= L).all()


@pytest.mark.parametrize("name,B,beta,L", [("sweep_b1_m64_L768", 1, 64, 768),
                                           ("sweep_b3_m256_L600", 3, 256, 600)])
def test_sweep_workload_recipe(name, B, beta, L):
    """Sweep points: B sequences of L cache rows, beta/2 tracked + beta/2 window rows,
    the window inside the generated span (the last min(512, L/2) rows)."""
    assert workloads.parse_sweep(name) == (B, beta, L)
    inp = workloads.generate(name)
    assert inp.batch == B and (np.diff(inp.cu_seqlens_k) == L).all()
    assert (np.diff(inp.cu_seqlens_q) == beta).all()
    assert (inp.window_len == beta // 2).all() and (inp.topk == beta // 2).all()
    gen = min(512, L // 2)
    assert (inp.window_start >= L - gen).all() and (inp.window_start + beta // 2 <= L).all()
    for b in range(B):
        pos = inp.q_pos[inp.seq_slice_q(b)]
        assert len(np.unique(pos)) == beta and (pos[: beta // 2] < inp.window_start[b]).all()
    with pytest.raises(ValueError):
        workloads.parse_sweep("sweep_b1_m63_L768")
    assert workloads.parse_sweep("batch32_uniform") is None


def test_sequence_without_query_rows_contributes_nothing():
    # the importance sums over the step's query rows: with none it is an empty sum
    rng = _rng(31)
    H, d, D = 2, 8, 16
    w = rng.standard_normal((3 * H * d, D))
    for L in (0, 5):
        kc, vc = rng.standard_normal((L, H, d)), rng.standard_normal((L, H, d))
        r = oracle.step_sequence(np.zeros((0, D)), w, np.zeros(0, np.int64), kc, vc, H, d, 1e4, None)
        assert r["out"].shape == (0, H, d)
        assert r["importance"].shape == (L,) and (r["importance"] == 0).all()
        np.testing.assert_array_equal(r["k_cache"], kc)
        np.testing.assert_array_equal(r["v_cache"], vc)
