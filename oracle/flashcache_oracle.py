"""fp64 CPU oracle of one Flash-Cache step.  TEST INFRASTRUCTURE ONLY.

Nothing in the product path imports this module: only ``tests/``, the
``__graft_entry__.smoke()`` check and the CPU-baseline leg of ``bench.py`` do.
It shares no code with the CUDA library.

What one step computes (Flash-dLLM, paper-digest page, Fig. 2 caption; infernews
post "Flash-dLLM: IO-aware KV caching and parallel decoding", Flash-Cache
paragraph): a fixed-size query of beta_m positions per sequence (the tracked
positions plus the current masked window) is projected to Q/K/V, rotated by
RoPE at its absolute positions, its K/V rows are written into the sequence's
cache, and the query attends bidirectionally to the whole cache.  The attention
probabilities are summed per key ("attention importance") and the top-k decoded
positions are reselected for tracking at the next step.

Readings taken where the pages are silent (each is stated where it is used):

* importance of key j = sum over heads and over the query rows of the step of
  the normalised attention probability of j;
* RoPE pairs element i with element i + d/2 (rotate-half) and uses angle
  ``pos * theta**(-2i/d)``;
* the cache is written before the query attends, so the query sees its own
  fresh K/V; rows of the cache that were not refreshed are attended as stored;
* scores are scaled by 1/sqrt(d), there are no biases, K/V heads = Q heads;
* the candidates for reselection are the positions ``[cand_lo, cand_hi)`` of a
  sequence, ties broken by the lower position.

All arithmetic is float64.  Every function is pinned by tests under
``tests/test_oracle_*.py`` against closed forms, library routines and brute
force (see each function's docstring for its pins).
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional

import numpy as np


def bf16_round(a) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even.

    bfloat16 keeps 8 significant bits.  For a = m * 2**e with 0.5 <= |m| < 1 the
    representable values in that binade are spaced 2**(e-8) apart, so the
    nearest one is rint(m * 2**8) * 2**(e-8) (numpy's rint rounds halves to
    even).  Valid for finite values of magnitude in [2**-126, 3.39e38]: the
    bf16 subnormal range and overflow to infinity are not modelled.
    Pinned against torch's float32 -> bfloat16 conversion.
    """
    a = np.asarray(a, dtype=np.float64)
    out = np.zeros_like(a)
    nz = a != 0
    m, e = np.frexp(a[nz])
    out[nz] = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    return out


def round_for_cache(a: np.ndarray, cache_dtype: Optional[str]) -> np.ndarray:
    """Value a cache of ``cache_dtype`` stores for ``a`` (None = exact)."""
    if cache_dtype is None:
        return np.asarray(a, np.float64)
    if cache_dtype == "bf16":
        return bf16_round(a)
    if cache_dtype == "fp32":
        return np.asarray(a, np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(cache_dtype)


def qkv_project(x: np.ndarray, w_qkv: np.ndarray, n_heads: int, head_dim: int):
    """q, k, v = W_q x, W_k x, W_v x for every query row (no bias).

    ``w_qkv`` rows are ordered [Q heads | K heads | V heads], each head's
    ``head_dim`` rows contiguous.  Returns three [n, H, d] float64 arrays.
    Pinned through the full-coverage closed form (torch matmul + SDPA).
    """
    x = np.asarray(x, np.float64)
    w = np.asarray(w_qkv, np.float64)
    hd = n_heads * head_dim
    assert w.shape == (3 * hd, x.shape[1])
    y = x @ w.T
    n = x.shape[0]
    q = y[:, 0 * hd:1 * hd].reshape(n, n_heads, head_dim)
    k = y[:, 1 * hd:2 * hd].reshape(n, n_heads, head_dim)
    v = y[:, 2 * hd:3 * hd].reshape(n, n_heads, head_dim)
    return q, k, v


def rope_angles(pos: np.ndarray, head_dim: int, theta: float) -> np.ndarray:
    """Angles pos * theta**(-2i/d) for i = 0 .. d/2-1, shape [n, d/2].

    Pinned by the d=2 closed form (angle = pos) and the frequency ladder
    (ratio theta**(-2/d) between neighbouring frequencies).
    """
    assert head_dim % 2 == 0
    i = np.arange(head_dim // 2, dtype=np.float64)
    inv_freq = float(theta) ** (-2.0 * i / head_dim)
    return np.asarray(pos, np.float64)[:, None] * inv_freq[None, :]


def rope_rotate(u: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotate each head vector of u [n, H, d] by RoPE at positions pos [n].

    Pair (u_i, u_{i+d/2}) is turned by angle a_i:
    (u_i cos a_i - u_{i+d/2} sin a_i,  u_{i+d/2} cos a_i + u_i sin a_i).
    Pinned by norm preservation, relative-offset invariance of dot products,
    the identity at position 0 and a complex-multiplication restatement.
    """
    u = np.asarray(u, np.float64)
    d = u.shape[-1]
    half = d // 2
    a = rope_angles(pos, d, theta)[:, None, :]  # [n, 1, d/2]
    c, s = np.cos(a), np.sin(a)
    lo, hi = u[..., :half], u[..., half:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


def write_cache(cache_b: np.ndarray, pos: np.ndarray, rows: np.ndarray,
                cache_dtype: Optional[str]) -> None:
    """cache_b[pos[r]] <- stored value of rows[r] (in place, one sequence).

    Positions must be distinct and inside the cache: the oracle refuses
    anything else rather than choosing a winner.
    """
    pos = np.asarray(pos)
    assert pos.ndim == 1 and len(np.unique(pos)) == len(pos), "duplicate positions"
    assert pos.min(initial=0) >= 0 and pos.max(initial=-1) < cache_b.shape[0], "position out of range"
    cache_b[pos] = round_for_cache(rows, cache_dtype)


def attend_sequence(q: np.ndarray, k_cache_b: np.ndarray, v_cache_b: np.ndarray):
    """Bidirectional attention of q [n, H, d] over one sequence's whole cache.

    For each head h and row r: s_j = q_r . K_j / sqrt(d) over every cached j,
    P = softmax(s), o_r = sum_j P_j V_j.  Returns (o [n, H, d], P [H, n, L]).
    Pinned against torch's scaled_dot_product_attention in fp64, by softmax row
    sums, by L = 1 (o = V) and by row-permutation equivariance.
    """
    n, H, d = q.shape
    L = k_cache_b.shape[0]
    o = np.empty((n, H, d), np.float64)
    P = np.empty((H, n, L), np.float64)
    if n == 0:  # no query rows: nothing attends (the cache may be empty too)
        return o, P
    scale = 1.0 / np.sqrt(d)
    for h in range(H):
        s = (q[:, h, :] @ np.asarray(k_cache_b[:, h, :], np.float64).T) * scale
        s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        p = e / e.sum(axis=1, keepdims=True)
        P[h] = p
        o[:, h, :] = p @ np.asarray(v_cache_b[:, h, :], np.float64)
    return o, P


def step_sequence(x_b, w_qkv, pos_b, k_cache_b, v_cache_b, n_heads, head_dim, theta,
                  cache_dtype: Optional[str]) -> Dict[str, np.ndarray]:
    """One sequence of a Flash-Cache step; returns out, new caches, importance.

    Order (infernews post, Flash-Cache paragraph: projection, RoPE, cache
    write in one pass; paper-digest page, Fig. 2 caption: the query attends to
    the full cache): project, rotate q and k, write k and v, attend, sum P.
    """
    q, k, v = qkv_project(x_b, w_qkv, n_heads, head_dim)
    q = rope_rotate(q, pos_b, theta)
    k = rope_rotate(k, pos_b, theta)
    kc = np.array(k_cache_b, np.float64, copy=True)
    vc = np.array(v_cache_b, np.float64, copy=True)
    write_cache(kc, pos_b, k, cache_dtype)
    write_cache(vc, pos_b, v, cache_dtype)
    o, P = attend_sequence(q, kc, vc)
    importance = P.sum(axis=(0, 1))  # over heads and query rows -> [L]
    return {"out": o, "k_cache": kc, "v_cache": vc, "importance": importance}


def flashcache_step(x, w_qkv, q_pos, cu_seqlens_q, cu_seqlens_k, k_cache, v_cache,
                    n_heads, head_dim, theta, cache_dtype: Optional[str],
                    seqs: Optional[Iterable[int]] = None) -> Dict[str, object]:
    """A whole (packed, variable-length) step, sequence by sequence.

    Sequences are independent: sequence b touches only its query rows
    ``cu_seqlens_q[b]:cu_seqlens_q[b+1]`` and its cache rows
    ``cu_seqlens_k[b]:cu_seqlens_k[b+1]``.  With ``seqs`` only those sequences
    are computed and returned (keyed by b); otherwise all, assembled into
    packed arrays as well.
    """
    B = len(cu_seqlens_q) - 1
    todo = range(B) if seqs is None else list(seqs)
    per = {}
    for b in todo:
        qs = slice(int(cu_seqlens_q[b]), int(cu_seqlens_q[b + 1]))
        ks = slice(int(cu_seqlens_k[b]), int(cu_seqlens_k[b + 1]))
        per[b] = step_sequence(x[qs], w_qkv, q_pos[qs], k_cache[ks], v_cache[ks],
                               n_heads, head_dim, theta, cache_dtype)
    res: Dict[str, object] = {"per_seq": per}
    if seqs is None:
        res["out"] = np.concatenate([per[b]["out"] for b in range(B)], axis=0)
        res["k_cache"] = np.concatenate([per[b]["k_cache"] for b in range(B)], axis=0)
        res["v_cache"] = np.concatenate([per[b]["v_cache"] for b in range(B)], axis=0)
        res["importance"] = np.concatenate([per[b]["importance"] for b in range(B)], axis=0)
    return res


def topk_tracked(importance, cu_seqlens_k, cand_lo, cand_hi, k_per_seq, width: int) -> np.ndarray:
    """Reselect the tracked set of every sequence (paper-digest page, Fig. 2
    caption: tracked positions are the top-k decoded tokens by importance).

    For sequence b the candidates are positions j in [cand_lo[b], cand_hi[b]);
    they are ordered by importance descending, then by position ascending, and
    the first k_per_seq[b] are kept.  Rows are padded with -1 up to ``width``.
    Pinned against a rank-counting brute force on tiny inputs with planted ties.
    """
    importance = np.asarray(importance, np.float64)
    B = len(cu_seqlens_k) - 1
    out = np.full((B, width), -1, np.int32)
    for b in range(B):
        base = int(cu_seqlens_k[b])
        cand = np.arange(int(cand_lo[b]), int(cand_hi[b]), dtype=np.int64)
        scores = importance[base + cand]
        order = np.lexsort((cand, -scores))  # primary: -score, secondary: position
        kb = min(int(k_per_seq[b]), len(cand), width)
        out[b, :kb] = cand[order[:kb]]
    return out
