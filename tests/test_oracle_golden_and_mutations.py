"""The oracle against its stored fixture, and the pins against planted mistakes.

The mutation tests plant a plausible mistake in the oracle (on the CPU only)
and check that at least one pin then fails, so a pin that can never fail is
noticed.
"""
import json
import os

import numpy as np
import pytest

import oracle
import oracle.flashcache_oracle as fo
from kv_cache_attention_qkv_b200 import workloads
import test_oracle_pins as pins

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_fp32_step.json")


def test_oracle_reproduces_golden_fixture():
    with open(GOLDEN) as f:
        g = json.load(f)
    inp = workloads.generate("tiny_fp32")
    res = oracle.flashcache_step(inp.x, inp.w_qkv, inp.q_pos, inp.cu_seqlens_q, inp.cu_seqlens_k,
                                 inp.k_cache, inp.v_cache, inp.n_heads, inp.head_dim,
                                 inp.rope_theta, "fp32")
    assert g["q_pos"] == inp.q_pos.tolist()
    np.testing.assert_allclose(res["out"].reshape(-1), g["out"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(res["k_cache"][inp.q_pos].reshape(-1), g["k_rows_written"], rtol=1e-12)
    np.testing.assert_allclose(res["importance"], g["importance"], rtol=1e-12)
    tr = oracle.topk_tracked(res["importance"], inp.cu_seqlens_k, inp.cand_lo, inp.cand_hi,
                             inp.topk, int(inp.topk.max()))
    assert tr.reshape(-1).tolist() == g["tracked"]


def _bad_rope_sign(u, pos, theta):
    u = np.asarray(u, np.float64)
    half = u.shape[-1] // 2
    a = fo.rope_angles(pos, u.shape[-1], theta)[:, None, :]
    lo, hi = u[..., :half], u[..., half:]
    return np.concatenate([lo * np.cos(a) + hi * np.sin(a), hi * np.cos(a) + lo * np.sin(a)], -1)


def _bad_rope_interleaved(u, pos, theta):
    u = np.asarray(u, np.float64)
    a = fo.rope_angles(pos, u.shape[-1], theta)[:, None, :]
    ev, od = u[..., 0::2], u[..., 1::2]
    out = np.empty_like(u)
    out[..., 0::2] = ev * np.cos(a) - od * np.sin(a)
    out[..., 1::2] = od * np.cos(a) + ev * np.sin(a)
    return out


def _bad_angles_freq(pos, head_dim, theta):
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.asarray(pos, np.float64)[:, None] * (float(theta) ** (-i / head_dim))[None, :]


def _bad_attend_no_scale(q, k, v):
    return _attend_with(q, k, v, scale=1.0)


def _bad_attend_kv_swapped(q, k, v):
    return _attend_with(q, v, k, scale=1.0 / np.sqrt(q.shape[-1]))


def _attend_with(q, k, v, scale):
    n, H, d = q.shape
    L = k.shape[0]
    o = np.empty((n, H, d))
    P = np.empty((H, n, L))
    for h in range(H):
        s = q[:, h] @ k[:, h].T * scale
        e = np.exp(s - s.max(1, keepdims=True))
        p = e / e.sum(1, keepdims=True)
        P[h] = p
        o[:, h] = p @ v[:, h]
    return o, P


def _bad_topk_ties_high_index(importance, cu, lo, hi, kk, width):
    importance = np.asarray(importance, np.float64)
    out = np.full((len(cu) - 1, width), -1, np.int32)
    for b in range(len(cu) - 1):
        cand = np.arange(int(lo[b]), int(hi[b]))
        order = np.lexsort((-cand, -importance[int(cu[b]) + cand]))
        kb = min(int(kk[b]), len(cand), width)
        out[b, :kb] = cand[order[:kb]]
    return out


def _bad_bf16_truncate(a):
    a = np.asarray(a, np.float64).astype(np.float32)
    return (a.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)


def _run_all_pins():
    """Run every pin; return how many failed."""
    failures = 0
    cases = [
        pins.test_bf16_round_matches_torch_conversion,
        pins.test_rope_d2_closed_form,
        pins.test_rope_frequency_ladder,
        pins.test_rope_complex_restatement,
        pins.test_hand_worked_two_token_example,
        lambda: pins.test_full_coverage_equals_uncached_attention(24, 3, 8, 20),
        pins.test_partial_query_matches_sdpa_over_stored_cache,
        lambda: [pins.test_topk_matches_brute_force_with_ties(s) for s in range(6)],
    ]
    for c in cases:
        try:
            c()
        except AssertionError:
            failures += 1
    return failures


@pytest.mark.parametrize("target,bad", [
    ("rope_rotate", _bad_rope_sign),
    ("rope_rotate", _bad_rope_interleaved),
    ("rope_angles", _bad_angles_freq),
    ("attend_sequence", _bad_attend_no_scale),
    ("attend_sequence", _bad_attend_kv_swapped),
    ("topk_tracked", _bad_topk_ties_high_index),
    ("bf16_round", _bad_bf16_truncate),
])
def test_planted_mistake_is_caught(monkeypatch, target, bad):
    monkeypatch.setattr(fo, target, bad)
    monkeypatch.setattr(oracle, target, bad)
    assert _run_all_pins() >= 1, f"no pin caught the planted mistake in {target}"


def test_pins_pass_on_the_real_oracle():
    assert _run_all_pins() == 0
