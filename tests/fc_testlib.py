"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
on a workload, run the oracle on the same inputs, and compare them with the
tolerances of the Flash-Cache parity bar:

* bf16 workloads: max|delta| <= 1e-2 * max|ref| for the attention output, the
  cache rows written and the importance;
* fp32 workloads: the same with 1e-5;
* tracked positions: identical wherever neighbouring oracle scores differ by
  more than 1e-3 relative; inside a run of closer scores any order is accepted.
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional

import numpy as np
import torch

import oracle
from kv_cache_attention_qkv_b200 import workloads

TOL = {"bf16": 1e-2, "fp32": 1e-5}
TIE_REL = 1e-3


def torch_dtype(inp):
    return torch.bfloat16 if inp.dtype == "bf16" else torch.float32


def upload(inp: workloads.StepInputs, device="cuda:0") -> Dict[str, torch.Tensor]:
    dt = torch_dtype(inp)

    def f(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dt)

    def i(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)

    return {
        "x": f(inp.x), "w": f(inp.w_qkv), "k_cache": f(inp.k_cache), "v_cache": f(inp.v_cache),
        "q_pos": i(inp.q_pos), "cu_q": i(inp.cu_seqlens_q), "cu_k": i(inp.cu_seqlens_k),
        "cand_lo": i(inp.cand_lo), "cand_hi": i(inp.cand_hi), "topk": i(inp.topk),
    }


def make_layer(inp: workloads.StepInputs, w: torch.Tensor, **over):
    from kv_cache_attention_qkv_b200 import FlashCache

    n = np.diff(inp.cu_seqlens_q)
    L = np.diff(inp.cu_seqlens_k)
    kw = dict(hidden=inp.hidden, n_heads=inp.n_heads, head_dim=inp.head_dim,
              rope_theta=inp.rope_theta, max_batch=max(inp.batch, 1),
              max_total_q=max(inp.total_q, 1), max_total_k=max(inp.total_k, 1),
              max_seqlen_q=int(max(n.max(), 1)), max_pos=int(max(L.max(), 1)),
              max_topk=int(max(inp.topk.max(), 1)))
    kw.update(over)
    return FlashCache(w, **kw)


def run_gpu(inp: workloads.StepInputs, layer=None, dev=None, want_importance=True,
            attn_split=True):
    """One fc_step + fc_topk_tracked; returns numpy results and the device state.
    ``attn_split``: True (the default rule), False (never split a small batch's
    attention) or "always" (split a small batch whatever its cache length)."""
    dev = dev or upload(inp)
    if layer is None:
        layer = make_layer(inp, dev["w"])
        if attn_split is not True:
            layer.set_attn_split(attn_split)
    T, H, d = inp.total_q, inp.n_heads, inp.head_dim
    out = torch.full((T, H, d), float("nan"), device=dev["x"].device, dtype=dev["x"].dtype)
    imp = torch.full((inp.total_k,), float("nan"), device=dev["x"].device) if want_importance else None
    layer.step(dev["x"], dev["q_pos"], dev["cu_q"], dev["cu_k"], dev["k_cache"], dev["v_cache"],
               out, imp)
    res = {"layer": layer, "dev": dev, "out_t": out, "imp_t": imp}
    if want_importance:
        K = int(inp.topk.max())
        tracked = torch.full((inp.batch, K), -7, device=out.device, dtype=torch.int32)
        layer.topk_tracked(imp, dev["cu_k"], dev["cand_lo"], dev["cand_hi"], K, tracked,
                           k_per_seq=dev["topk"])
        res["tracked"] = tracked.cpu().numpy()
        res["importance"] = imp.cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    res["err"] = layer.get_error()
    res["out"] = out.float().cpu().numpy().astype(np.float64)
    return res


def split_entries(inp: workloads.StepInputs, num_sms: int, forced=False) -> int:
    """Work entries of a small batch whose items are split over the SMs: every
    (sequence, head, 128-row tile) item becomes min(target, its 128-key tiles)
    entries, target = max(1, min(8, SMs // items))."""
    n = np.diff(inp.cu_seqlens_q)
    L = np.diff(inp.cu_seqlens_k)
    live = (n > 0) & (L > 0)
    items = inp.n_heads * ((n + 127) // 128) * live
    target = max(1, min(8, num_sms // max(int(items.sum()), 1)))
    ns = np.maximum(1, np.minimum(target, (L + 127) // 128))
    return int((items * ns).sum())


def splits_attention(inp: workloads.StepInputs, num_sms: int, forced=False,
                     importance=True) -> bool:
    """Whether fc_step takes the small-batch split path for these shapes (by
    default: a small batch without importance, or with caches of 1280 rows or
    more on average)."""
    small = inp.n_heads * ((inp.total_q + 127) // 128 + inp.batch - 1) <= num_sms
    return small and (forced or not importance or inp.total_k >= 1280 * inp.batch)


def run_oracle(inp: workloads.StepInputs, seqs: Optional[Iterable[int]] = None):
    return oracle.flashcache_step(inp.x, inp.w_qkv, inp.q_pos, inp.cu_seqlens_q, inp.cu_seqlens_k,
                                  inp.k_cache, inp.v_cache, inp.n_heads, inp.head_dim,
                                  inp.rope_theta, inp.dtype, seqs=seqs)


def assert_close(got, ref, tol, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    err = float(np.abs(got - ref).max()) if ref.size else 0.0
    assert err <= tol * scale + 1e-30, f"{what}: max|delta| {err:.3e} > {tol} * max|ref| {scale:.3e}"
    return err / scale if scale else 0.0


def assert_tracked_matches(got_row, importance_b, lo, hi, kb, what):
    """The tie-group rule on one sequence (importance_b indexed by position)."""
    cand = np.arange(lo, hi)
    sc = np.asarray(importance_b, np.float64)[cand]
    order = np.lexsort((cand, -sc))
    srt, spos = sc[order], cand[order]
    keep = min(kb, len(cand))
    got = np.asarray(got_row)
    assert (got[keep:] == -1).all(), f"{what}: padding {got[keep:]}"
    assert len(set(got[:keep].tolist())) == keep, f"{what}: duplicates"
    # group id per rank: a new group starts where the gap exceeds TIE_REL
    gid = np.zeros(len(srt), np.int64)
    for i in range(1, len(srt)):
        prev, cur = srt[i - 1], srt[i]
        close = abs(prev - cur) <= TIE_REL * max(abs(prev), abs(cur))
        gid[i] = gid[i - 1] + (0 if close else 1)
    rank_of = {int(p): r for r, p in enumerate(spos)}
    for r in range(keep):
        p = int(got[r])
        assert p in rank_of, f"{what}: {p} is not a candidate"
        assert gid[rank_of[p]] == gid[r], (
            f"{what}: rank {r} holds position {p} (oracle rank {rank_of[p]}, "
            f"score {srt[rank_of[p]]:.6g} vs {srt[r]:.6g})")


def compare_step(inp, gpu, ref, seqs: Iterable[int], written_ok=True):
    """Element-wise comparison on the given sequences; returns worst relative errors."""
    tol = TOL[inp.dtype]
    kc = gpu["dev"]["k_cache"]
    vc = gpu["dev"]["v_cache"]
    worst = {"out": 0.0, "k": 0.0, "v": 0.0, "imp": 0.0}
    for b in seqs:
        r = ref["per_seq"][b]
        qs, ks = inp.seq_slice_q(b), inp.seq_slice_k(b)
        worst["out"] = max(worst["out"], assert_close(gpu["out"][qs], r["out"], tol, f"out[seq {b}]"))
        rows = ks.start + inp.q_pos[qs]
        gk = kc[torch.from_numpy(rows).to(kc.device)].float().cpu().numpy()
        gv = vc[torch.from_numpy(rows).to(vc.device)].float().cpu().numpy()
        worst["k"] = max(worst["k"], assert_close(gk, r["k_cache"][inp.q_pos[qs]], tol, f"k rows[seq {b}]"))
        worst["v"] = max(worst["v"], assert_close(gv, r["v_cache"][inp.q_pos[qs]], tol, f"v rows[seq {b}]"))
        if "importance" in gpu:
            worst["imp"] = max(worst["imp"], assert_close(gpu["importance"][ks], r["importance"], tol,
                                                         f"importance[seq {b}]"))
            assert_tracked_matches(gpu["tracked"][b], r["importance"], int(inp.cand_lo[b]),
                                   int(inp.cand_hi[b]), int(inp.topk[b]), f"tracked[seq {b}]")
    return worst


def assert_unwritten_rows_unchanged(inp, gpu):
    """Cache rows no query row maps to must keep their prior bytes exactly."""
    S = inp.total_k
    written = np.zeros(S, bool)
    for b in range(inp.batch):
        written[inp.seq_slice_k(b).start + inp.q_pos[inp.seq_slice_q(b)]] = True
    keep = torch.from_numpy(~written).to(gpu["dev"]["k_cache"].device)
    dt = torch_dtype(inp)
    for name, prior in (("k_cache", inp.k_cache), ("v_cache", inp.v_cache)):
        cur = gpu["dev"][name][keep]
        old = torch.from_numpy(np.ascontiguousarray(prior)).to(cur.device, dtype=dt)[keep]
        assert torch.equal(cur, old), f"{name}: rows outside the query were modified"
