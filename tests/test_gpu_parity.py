"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle."""
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


@pytest.mark.parametrize("name", ["tiny_fp32", "small_d64", "small_varlen", "layer_b1",
                                  "small_longcache"])
def test_full_parity(name):
    """Every output element of small workloads against the oracle."""
    inp = workloads.generate(name)
    gpu = tl.run_gpu(inp)
    assert gpu["err"] == 0
    ref = tl.run_oracle(inp)
    tl.compare_step(inp, gpu, ref, range(inp.batch))
    tl.assert_unwritten_rows_unchanged(inp, gpu)
    # importance of every key of the batch, not only the sampled sequences
    tl.assert_close(gpu["importance"], ref["importance"], tl.TOL[inp.dtype], "importance")


@pytest.mark.parametrize("name", ["layer_b1", "small_varlen", "small_longcache"])
def test_both_projection_kernels(name):
    """The CTA-pair projection and the split-K cluster projection (forced, at
    several cluster sizes) all meet the parity bar on every output, and the
    default run is bit-identical to a forced run of the kernel it planned."""
    inp = workloads.generate(name)
    ref = tl.run_oracle(inp)
    outs = {}
    smax = min(8, inp.hidden // 64)
    for which, split in (("pair", 0), ("splitk", 0), ("splitk", 1), ("splitk", 2),
                         ("splitk", smax), ("auto", 0)):
        dev = tl.upload(inp)
        layer = tl.make_layer(inp, dev["w"])
        layer.set_qkv_kernel(which, split)
        plan = layer.qkv_plan(inp.total_q)
        gpu = tl.run_gpu(inp, layer=layer, dev=dev)
        assert gpu["err"] == 0, (which, split)
        tl.compare_step(inp, gpu, ref, range(inp.batch))
        tl.assert_unwritten_rows_unchanged(inp, gpu)
        outs[(which, split)] = (plan, gpu["out"], dev["k_cache"].cpu(), dev["v_cache"].cpu())
    # the default run is bit-identical to the forced run of the kernel it planned
    auto = outs[("auto", 0)]
    if auto[0]["kernel"] == "pair":
        same = outs[("pair", 0)]
    else:
        same = next(v for (w, sp), v in outs.items()
                    if w == "splitk" and v[0]["split"] == auto[0]["split"])
    assert np.array_equal(auto[1], same[1])
    assert torch.equal(auto[2], same[2]) and torch.equal(auto[3], same[3])


@pytest.mark.slow
@pytest.mark.parametrize("name,seqs", [("batch32_uniform", [0, 13, 31]),
                                       ("batch32_varlen", [0, 5, 17, 30]),
                                       # sweep extremes: two 128-row query tiles per
                                       # sequence over an 8192-row cache; 64 sequences
                                       ("sweep_b2_m256_L8192", [0, 1]),
                                       ("sweep_b64_m128_L1536", [0, 40, 63])])
def test_full_size_sampled_parity(name, seqs):
    """Full-size workloads, same launch configuration as the bench; the oracle
    recomputes sampled sequences (sequences are independent)."""
    inp = workloads.generate(name)
    gpu = tl.run_gpu(inp)
    assert gpu["err"] == 0
    ref = tl.run_oracle(inp, seqs=seqs)
    tl.compare_step(inp, gpu, ref, seqs)
    tl.assert_unwritten_rows_unchanged(inp, gpu)
    # properties that hold for every sequence at any size
    imp = gpu["importance"]
    for b in range(inp.batch):
        n = inp.cu_seqlens_q[b + 1] - inp.cu_seqlens_q[b]
        tot = imp[inp.seq_slice_k(b)].sum()
        assert abs(tot - inp.n_heads * n) <= 1e-3 * inp.n_heads * n, (b, tot)
    assert np.isfinite(gpu["out"]).all()


def test_attention_work_split():
    """Unsplit, a step with importance gives every item to the two-pass kernel
    (the column sums need each row's final normaliser) and a step without
    importance gives them to the one-pass kernel, whose ordinary scores never
    leave its exponent band.  Split (forced: its caches are short), every item
    becomes entries over runs of key tiles, all in the two-pass kernel."""
    inp = workloads.generate("small_longcache")
    n = np.diff(inp.cu_seqlens_q)
    want = inp.n_heads * int(((n + 127) // 128).sum())
    gpu = tl.run_gpu(inp, attn_split=False)
    assert gpu["layer"].last_step_work() == (want, want, 0)
    g = tl.run_gpu(inp, want_importance=False, attn_split=False)
    assert g["layer"].last_step_work() == (want, 0, 0)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert not tl.splits_attention(inp, sms) and tl.splits_attention(inp, sms, forced=True)
    entries = tl.split_entries(inp, sms, forced=True)
    assert entries > want
    for imp in (True, False):
        g = tl.run_gpu(inp, want_importance=imp, attn_split="always")
        assert g["layer"].last_step_work() == (entries, entries, 0)


@pytest.mark.parametrize("name", ["small_varlen", "small_longcache", "layer_b1"])
def test_split_attention_agrees_with_unsplit(name):
    """The small-batch split (forced here: these caches are short; two launches,
    parts of O combined by the item's last entry in entry order) against the
    oracle, with and without importance, and run to run bit-identical; the
    unsplit kernels agree within the bar."""
    inp = workloads.generate(name)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert tl.splits_attention(inp, sms, forced=True)
    ref = tl.run_oracle(inp)
    for imp in (True, False):
        a = tl.run_gpu(inp, want_importance=imp, attn_split="always")
        b = tl.run_gpu(inp, want_importance=imp, attn_split="always")
        u = tl.run_gpu(inp, want_importance=imp, attn_split=False)
        for g in (a, u):
            assert g["err"] == 0
            tl.compare_step(inp, g, ref, range(inp.batch))
        assert np.array_equal(a["out"], b["out"])
        tl.assert_close(a["out"], u["out"], tl.TOL[inp.dtype], "split vs unsplit")
        if imp:
            assert np.array_equal(a["importance"], b["importance"])
            tl.assert_close(a["importance"], ref["importance"], tl.TOL[inp.dtype], "importance")
            np.testing.assert_array_equal(a["tracked"], b["tracked"])


def test_split_attention_repeated_on_one_handle():
    """Consecutive split steps on one handle (the per-item counters of the last
    entry are reset by the step that used them) give identical results, with
    and without importance in between."""
    inp = workloads.generate("small_longcache")
    dev = tl.upload(inp)
    layer = tl.make_layer(inp, dev["w"])
    layer.set_attn_split("always")
    ref = tl.run_oracle(inp)
    first = None
    for imp in (True, False, True, True):
        g = tl.run_gpu(inp, layer=layer, dev=dev, want_importance=imp)
        assert g["err"] == 0
        tl.compare_step(inp, g, ref, range(inp.batch))
        if imp:
            if first is None:
                first = g
            else:
                assert np.array_equal(g["out"], first["out"])
                assert np.array_equal(g["importance"], first["importance"])
                np.testing.assert_array_equal(g["tracked"], first["tracked"])


@pytest.mark.slow
@pytest.mark.parametrize("name,seqs", [("sweep_b1_m128_L8192", [0]), ("sweep_b2_m128_L8192", [0, 1]),
                                       ("sweep_b1_m128_L1536", [0]), ("sweep_b2_m256_L8192", [0, 1])])
def test_split_attention_full_size(name, seqs):
    """Small batches at full size, in the launch configuration the bench uses
    (split for the long caches, not for L = 1536 nor for beta = 256 at B = 2),
    against the oracle."""
    inp = workloads.generate(name)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    gpu = tl.run_gpu(inp)
    assert gpu["err"] == 0
    if tl.splits_attention(inp, sms):
        e = tl.split_entries(inp, sms)
        assert gpu["layer"].last_step_work() == (e, e, 0)
    ref = tl.run_oracle(inp, seqs=seqs)
    tl.compare_step(inp, gpu, ref, seqs)
    tl.assert_unwritten_rows_unchanged(inp, gpu)


@pytest.mark.parametrize("name,seqs", [("small_varlen", None), ("small_longcache", None),
                                       ("layer_b1", None)])
def test_one_pass_attention_without_importance(name, seqs):
    """The one-pass kernel (steps without importance) against the oracle."""
    inp = workloads.generate(name)
    gpu = tl.run_gpu(inp, want_importance=False, attn_split=False)
    assert gpu["err"] == 0
    ref = tl.run_oracle(inp, seqs=seqs)
    tl.compare_step(inp, gpu, ref, seqs if seqs is not None else range(inp.batch))
    tl.assert_unwritten_rows_unchanged(inp, gpu)


@pytest.mark.slow
@pytest.mark.parametrize("name,seqs", [("batch32_uniform", [0, 13, 31]),
                                       ("batch32_varlen", [0, 5, 17, 30]),
                                       ("sweep_b2_m256_L8192", [0, 1])])
def test_one_pass_attention_without_importance_full_size(name, seqs):
    """Full-size workloads through the one-pass kernel, sampled sequences."""
    inp = workloads.generate(name)
    gpu = tl.run_gpu(inp, want_importance=False)
    assert gpu["err"] == 0
    ref = tl.run_oracle(inp, seqs=seqs)
    tl.compare_step(inp, gpu, ref, seqs)
    assert np.isfinite(gpu["out"]).all()


def _plant_far_key(inp, b, n_rows, seed):
    """Keep the first n_rows query rows of sequence b and plant, in a prior cache
    row of its second key tile, a key whose score against every kept row is
    +-200 (log2 units, the kernels' score domain), chosen per head as the
    least-norm solution of q_r . k = +-200 sqrt(d) / log2(e) (rotated q of the
    oracle).  Rows at +200 put all their attention on that key, far outside the
    one-pass kernel's band above the first tile's maximum (2^64); rows at -200
    ignore it.  Either way the softmax does not depend on the rounding of q,
    which a large key magnifies (the kernels keep q in bf16)."""
    qs = inp.seq_slice_q(b)
    keep = np.r_[0:qs.start + n_rows, qs.stop:inp.total_q]
    cnt = np.diff(inp.cu_seqlens_q)
    cnt[b] = n_rows
    inp.x, inp.q_pos = inp.x[keep], inp.q_pos[keep]
    inp.cu_seqlens_q = np.r_[0, np.cumsum(cnt)].astype(np.int32)
    qs, ks = inp.seq_slice_q(b), inp.seq_slice_k(b)
    H, d = inp.n_heads, inp.head_dim
    q, _, _ = oracle.qkv_project(inp.x[qs], inp.w_qkv, H, d)
    q = oracle.rope_rotate(q, inp.q_pos[qs], inp.rope_theta)
    sgn = np.random.default_rng(seed).choice([-1.0, 1.0], size=n_rows)
    target = sgn * 200.0 * np.sqrt(d) / np.log2(np.e)
    written = set(inp.q_pos[qs].tolist())
    j = next(p for p in range(128, ks.stop - ks.start) if p not in written)
    inp.k_cache = inp.k_cache.copy()
    for h in range(H):
        qh = q[:, h, :]
        inp.k_cache[ks.start + j, h] = qh.T @ np.linalg.solve(qh @ qh.T, target)
    inp.k_cache[ks.start + j] = workloads.to_bf16_exact(inp.k_cache[ks.start + j])
    return j, sgn


@pytest.mark.parametrize("seq", [0, 2])
def test_scores_out_of_the_one_pass_band_are_handed_over(seq):
    """In a step without importance, items with scores far above their first key
    tile's maximum are handed to the two-pass kernel and still match the
    oracle."""
    inp = workloads.generate("small_varlen")
    _plant_far_key(inp, seq, 64, seed=seq)
    gpu = tl.run_gpu(inp, want_importance=False, attn_split=False)
    assert gpu["err"] == 0
    items, two_pass, handed = gpu["layer"].last_step_work()
    assert two_pass == 0 and handed == inp.n_heads  # every head of that sequence
    ref = tl.run_oracle(inp)
    tl.compare_step(inp, gpu, ref, range(inp.batch))
    # with importance the same step runs in the two-pass kernel from the start
    g2 = tl.run_gpu(inp, attn_split=False)
    assert g2["layer"].last_step_work()[2] == 0
    tl.compare_step(inp, g2, ref, range(inp.batch))
    # split over the SMs (two launches), with and without importance
    for imp in (True, False):
        g3 = tl.run_gpu(inp, want_importance=imp, attn_split="always")
        assert g3["err"] == 0
        tl.compare_step(inp, g3, ref, range(inp.batch))


def test_topk_kernel_is_exact_on_gpu_importance():
    """fc_topk_tracked on the GPU's own importance equals the oracle's
    reselection of those same fp32 values, bit for bit."""
    inp = workloads.generate("small_varlen")
    gpu = tl.run_gpu(inp)
    ref_tr = oracle.topk_tracked(gpu["importance"], inp.cu_seqlens_k, inp.cand_lo, inp.cand_hi,
                                 inp.topk, int(inp.topk.max()))
    np.testing.assert_array_equal(gpu["tracked"], ref_tr)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_topk_ties_and_ragged_candidates(seed):
    """Planted ties, empty candidate ranges, k above the candidate count."""
    rng = np.random.default_rng(seed)
    B = 7
    L = rng.integers(1, 3000, B)
    L[2] = 1
    cu = np.zeros(B + 1, np.int32)
    cu[1:] = np.cumsum(L)
    imp = (rng.integers(0, 50, cu[-1]) * 0.125).astype(np.float32)
    imp[cu[3]:cu[4]] = 1.0  # one sequence made entirely of ties
    lo = np.array([rng.integers(0, l + 1) for l in L], np.int32)
    hi = np.array([rng.integers(a, l + 1) for a, l in zip(lo, L)], np.int32)
    lo[5], hi[5] = 3, 3  # empty
    K = 300
    kb = rng.integers(0, K + 1, B).astype(np.int32)
    inp = workloads.generate("tiny_fp32")
    dev = tl.upload(inp)
    layer = tl.make_layer(inp, dev["w"], max_topk=K, max_total_k=int(cu[-1]), max_pos=int(L.max()),
                          max_batch=B)
    t = lambda a: torch.from_numpy(a).cuda()
    tracked = torch.full((B, K), -7, dtype=torch.int32, device="cuda")
    layer.topk_tracked(t(imp), t(cu), t(lo), t(hi), K, tracked, k_per_seq=t(kb))
    assert layer.get_error() == 0
    ref = oracle.topk_tracked(imp.astype(np.float64), cu, lo, hi, kb, K)
    np.testing.assert_array_equal(tracked.cpu().numpy(), ref)


@pytest.mark.parametrize("seed", [0, 1])
def test_topk_small_selection_path(seed):
    """k <= 64 from at most 8192 candidates (the register-sort path) at its
    edges: 1, 63, 64, 65, 127-129, 2047-2049 and 8192 candidates (one to four
    blocks of 128 per warp), one sequence just past the path (8193, the radix
    select over unstaged keys), heavy ties, k_per_seq 0, 1, 63 and 64."""
    rng = np.random.default_rng(100 + seed)
    n_cand = np.array([1, 63, 64, 65, 127, 128, 129, 2047, 2048, 2049, 8192, 8193, 1536, 700],
                      np.int64)
    B = len(n_cand)
    L = n_cand + rng.integers(0, 40, B)
    cu = np.zeros(B + 1, np.int32)
    cu[1:] = np.cumsum(L)
    imp = (rng.integers(0, 12, cu[-1]) * 0.25).astype(np.float32)  # many equal scores
    imp[cu[13]:cu[14]] = 0.5  # one sequence of ties only
    lo = np.array([rng.integers(0, l - c + 1) for l, c in zip(L, n_cand)], np.int32)
    hi = (lo + n_cand).astype(np.int32)
    K = 64
    kb = np.array([1, 63, 64, 64, 64, 64, 64, 17, 64, 64, 64, 64, 0, 64], np.int32)
    inp = workloads.generate("tiny_fp32")
    dev = tl.upload(inp)
    layer = tl.make_layer(inp, dev["w"], max_topk=K, max_total_k=int(cu[-1]), max_pos=int(L.max()),
                          max_batch=B)
    t = lambda a: torch.from_numpy(a).cuda()
    tracked = torch.full((B, K), -7, dtype=torch.int32, device="cuda")
    layer.topk_tracked(t(imp), t(cu), t(lo), t(hi), K, tracked, k_per_seq=t(kb))
    assert layer.get_error() == 0
    ref = oracle.topk_tracked(imp.astype(np.float64), cu, lo, hi, kb, K)
    np.testing.assert_array_equal(tracked.cpu().numpy(), ref)


def test_rerun_is_bit_identical():
    """The step is deterministic: a second run from the same inputs gives the
    same bytes (importance is summed in order-independent fixed point)."""
    inp = workloads.generate("small_varlen")
    a = tl.run_gpu(inp)
    b = tl.run_gpu(inp)
    assert np.array_equal(a["out"], b["out"])
    assert np.array_equal(a["importance"], b["importance"])
    assert np.array_equal(a["tracked"], b["tracked"])
    assert torch.equal(a["dev"]["k_cache"], b["dev"]["k_cache"])


def test_step_is_idempotent_in_place():
    """Running the same step twice on the same cache leaves it as after one."""
    inp = workloads.generate("small_varlen")
    dev = tl.upload(inp)
    layer = tl.make_layer(inp, dev["w"])
    a = tl.run_gpu(inp, layer=layer, dev=dev)
    k1 = dev["k_cache"].clone()
    b = tl.run_gpu(inp, layer=layer, dev=dev)
    assert torch.equal(k1, dev["k_cache"])
    assert np.array_equal(a["out"], b["out"])


def test_accumulate_adds_importance():
    inp = workloads.generate("small_varlen")
    dev = tl.upload(inp)
    layer = tl.make_layer(inp, dev["w"])
    T, H, d = inp.total_q, inp.n_heads, inp.head_dim
    out = torch.empty((T, H, d), device="cuda", dtype=torch.bfloat16)
    imp = torch.zeros(inp.total_k, device="cuda")
    layer.step(dev["x"], dev["q_pos"], dev["cu_q"], dev["cu_k"], dev["k_cache"], dev["v_cache"], out, imp)
    one = imp.clone()
    layer.step(dev["x"], dev["q_pos"], dev["cu_q"], dev["cu_k"], dev["k_cache"], dev["v_cache"], out, imp,
               accumulate=True)
    torch.cuda.synchronize()
    assert torch.equal(imp, one + one)


def test_without_importance_and_empty_query():
    inp = workloads.generate("small_varlen")
    gpu = tl.run_gpu(inp, want_importance=False)
    ref = tl.run_oracle(inp)
    tl.assert_close(gpu["out"], ref["out"], 1e-2, "out without importance")
    # T = 0: nothing written, importance zeroed
    layer, dev = gpu["layer"], gpu["dev"]
    B = inp.batch
    cu0 = torch.zeros(B + 1, dtype=torch.int32, device="cuda")
    imp = torch.full((inp.total_k,), 5.0, device="cuda")
    before = dev["k_cache"].clone()
    layer.step(dev["x"][:0], dev["q_pos"][:0], cu0, dev["cu_k"], dev["k_cache"], dev["v_cache"],
               torch.empty((0, inp.n_heads, inp.head_dim), device="cuda", dtype=torch.bfloat16), imp)
    torch.cuda.synchronize()
    assert torch.equal(before, dev["k_cache"]) and float(imp.abs().max()) == 0.0
    assert layer.get_error() == 0


def test_single_key_sequence_returns_value():
    """L_b = 1 with a single query row at position 0: attention returns v."""
    inp = workloads.generate("small_varlen", batch=1)
    # shrink to one row attending a one-row cache
    inp.q_pos = np.array([0], np.int32)
    inp.x = inp.x[:1]
    inp.cu_seqlens_q = np.array([0, 1], np.int32)
    inp.cu_seqlens_k = np.array([0, 1], np.int32)
    inp.k_cache, inp.v_cache = inp.k_cache[:1], inp.v_cache[:1]
    inp.cand_lo, inp.cand_hi, inp.topk = (np.array([0], np.int32), np.array([1], np.int32),
                                          np.array([1], np.int32))
    gpu = tl.run_gpu(inp)
    ref = tl.run_oracle(inp)
    tl.compare_step(inp, gpu, ref, [0])
    tl.assert_close(gpu["out"][0], ref["v_cache"][0], 1e-2, "o = v")
    assert abs(gpu["importance"][0] - inp.n_heads) < 1e-3


@pytest.mark.parametrize("bad", ["range", "dup", "seqlens", "cand"])
def test_device_checks_set_error_word(bad):
    from kv_cache_attention_qkv_b200.binding import describe_error_word

    inp = workloads.generate("small_varlen")
    if bad == "range":
        inp.q_pos = inp.q_pos.copy()
        inp.q_pos[3] = 10_000
    elif bad == "dup":
        inp.q_pos = inp.q_pos.copy()
        inp.q_pos[5] = inp.q_pos[4]
    elif bad == "seqlens":
        inp.cu_seqlens_q = inp.cu_seqlens_q.copy()
        inp.cu_seqlens_q[1] = inp.cu_seqlens_q[2] + 1  # not monotone
    else:
        inp.cand_hi = inp.cand_hi.copy()
        inp.cand_hi[0] = 10 ** 6
    prior_k = inp.k_cache.copy()
    gpu = tl.run_gpu(inp)
    names = describe_error_word(gpu["err"])
    expect = {"range": "POS_RANGE", "dup": "POS_DUP", "seqlens": "SEQLENS", "cand": "CAND"}[bad]
    assert expect in names, names
    # the offending rows were not written anywhere
    if bad in ("range", "dup"):
        k_now = gpu["dev"]["k_cache"].float().cpu().numpy()
        S = inp.total_k
        assert k_now.shape[0] == S
        if bad == "dup":
            row = inp.seq_slice_k(0).start + inp.q_pos[4]
            np.testing.assert_array_equal(k_now[row], prior_k[row])
    assert tl.run_gpu(workloads.generate("small_varlen"), layer=gpu["layer"])["err"] == 0


def test_bounded_wait_times_out_and_context_stays_usable():
    """A barrier that never completes turns into FC_ERR_TIMEOUT, not a hang;
    the next step on the same handle is correct."""
    from kv_cache_attention_qkv_b200.binding import describe_error_word

    inp = workloads.generate("small_varlen")
    dev = tl.upload(inp)
    layer = tl.make_layer(inp, dev["w"])
    layer.selftest_wait_timeout(50_000)  # 50 ms
    word = layer.get_error()
    assert "TIMEOUT" in describe_error_word(word)
    gpu = tl.run_gpu(inp, layer=layer, dev=dev)
    assert gpu["err"] == 0
    tl.compare_step(inp, gpu, tl.run_oracle(inp), range(inp.batch))


@pytest.mark.parametrize("name", ["small_varlen", "tiny_fp32"])
def test_step_host_matches_device_path(name):
    """fc_step_host (host inputs and outputs, copies double-buffered against the
    kernels) gives the same bits as fc_step + fc_topk_tracked on device buffers,
    over consecutive calls with different inputs: both staging sets, then their
    reuse."""
    inp = workloads.generate(name)
    dev_a, dev_b = tl.upload(inp), tl.upload(inp)
    layer_a, layer_b = tl.make_layer(inp, dev_a["w"]), tl.make_layer(inp, dev_b["w"])
    T, S, H, d, B = inp.total_q, inp.total_k, inp.n_heads, inp.head_dim, inp.batch
    K = int(inp.topk.max())
    dt = dev_a["x"].dtype
    scales = (1.0, -0.5, 0.25, 2.0)
    want_out, want_tr = [], []
    for sc in scales:
        out = torch.empty((T, H, d), device="cuda", dtype=dt)
        imp = torch.empty((S,), device="cuda")
        tr = torch.empty((B, K), device="cuda", dtype=torch.int32)
        layer_a.step(dev_a["x"] * sc, dev_a["q_pos"], dev_a["cu_q"], dev_a["cu_k"],
                     dev_a["k_cache"], dev_a["v_cache"], out, imp)
        layer_a.topk_tracked(imp, dev_a["cu_k"], dev_a["cand_lo"], dev_a["cand_hi"], K, tr,
                             k_per_seq=dev_a["topk"])
        want_out.append(out.cpu())
        want_tr.append(tr.cpu())
    assert layer_a.get_error() == 0

    pin = lambda t: t.cpu().contiguous().pin_memory()
    xs = [pin(dev_b["x"] * sc) for sc in scales]
    small = {n: pin(dev_b[n]) for n in ("q_pos", "cu_q", "cu_k", "cand_lo", "cand_hi", "topk")}
    outs = [torch.full((T, H, d), float("nan"), dtype=dt).pin_memory() for _ in scales]
    trs = [torch.full((B, K), -7, dtype=torch.int32).pin_memory() for _ in scales]
    torch.cuda.synchronize()
    for i in range(len(scales)):
        layer_b.step_host(xs[i], small["q_pos"], small["cu_q"], small["cu_k"], dev_b["k_cache"],
                          dev_b["v_cache"], small["cand_lo"], small["cand_hi"], K, outs[i], trs[i],
                          k_per_seq=small["topk"])
    layer_b.host_sync()
    torch.cuda.synchronize()
    assert layer_b.get_error() == 0
    bits = torch.int16 if dt == torch.bfloat16 else torch.int32
    for i in range(len(scales)):
        assert torch.equal(outs[i].view(bits), want_out[i].view(bits)), f"out of call {i}"
        assert torch.equal(trs[i], want_tr[i]), f"tracked of call {i}"
    for n in ("k_cache", "v_cache"):
        assert torch.equal(dev_b[n].view(bits), dev_a[n].view(bits)), n
    layer_a.close()
    layer_b.close()
