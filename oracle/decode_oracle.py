"""fp64 CPU oracle of one decode iteration (draft-and-verify over the model step).
TEST INFRASTRUCTURE ONLY: nothing in the product path imports this module.

Flash-dLLM decodes a masked window of the generated span in parallel; the same
model is the drafter and the verifier; the draft tokens and the [MASK] tokens
are checked through two views, and every prediction that meets the confidence
threshold is accepted in the same iteration; the tracked positions are
reselected by attention importance (infernews post "Flash-dLLM: IO-aware KV
caching and parallel decoding", Flash-Verify paragraph; paper-digest page,
Fig. 2 caption; forum post: threshold 0.9, masked window 64, tracking budget
64).

Readings taken where the pages are silent:

* the query of a sequence is its K tracked positions followed by the W
  positions of its window [ws, ws + W);
* [MASK] view: undecided window rows read the [MASK] embedding; draft view:
  they read their draft token's embedding (the [MASK] embedding when there is
  no draft yet); decided rows read their token in both views;
* a window position is accepted when the [MASK] view's confidence reaches the
  threshold (its token is the [MASK] view's), or when the draft view predicts
  the position's own draft with a confidence that reaches the threshold
  (the draft is verified); when neither happens anywhere in the window, the
  undecided position with the highest [MASK]-view confidence is accepted
  (lowest position on ties), so every iteration decodes at least one token;
* the drafts of the positions still undecided become the [MASK] view's
  predictions;
* when the whole window is decided it advances by W if the next window lies
  inside the generated span, and the new window has no drafts;
* the tracked positions are then reselected: the top-K positions of
  [0, ws) by the draft view's importance (summed over layers).
"""
from __future__ import annotations

from typing import Dict

import numpy as np


def build_query(tokens: np.ndarray, draft: np.ndarray, tracked: np.ndarray, ws: int, W: int,
                mask_id: int):
    """Positions and the token ids of both views for one sequence's query."""
    pos = np.concatenate([np.asarray(tracked, np.int64), np.arange(ws, ws + W)])
    ids_mask = tokens[pos].copy()
    ids_draft = tokens[pos].copy()
    und = ids_mask < 0
    ids_mask[und] = mask_id
    d = draft[pos]
    ids_draft[und] = np.where(d[und] >= 0, d[und], mask_id)
    return pos, ids_mask, ids_draft


def accept_and_advance(tokens: np.ndarray, draft: np.ndarray, ws: int, W: int, gen_end: int,
                       tok_m: np.ndarray, conf_m: np.ndarray, tok_d: np.ndarray,
                       conf_d: np.ndarray, threshold: float) -> Dict[str, object]:
    """Acceptance, drafts and window advance for one sequence (in place on copies).

    ``tok_*``/``conf_*``: the two views' predictions for the W window rows.
    """
    tokens = tokens.copy()
    draft = draft.copy()
    win = np.arange(ws, ws + W)
    und = tokens[win] < 0
    acc_m = und & (conf_m >= threshold)
    acc_d = und & ~acc_m & (draft[win] >= 0) & (tok_d == draft[win]) & (conf_d >= threshold)
    new_tok = np.where(acc_m, tok_m, np.where(acc_d, draft[win], -1))
    n_acc = int((acc_m | acc_d).sum())
    if n_acc == 0 and und.any():
        c = np.where(und, conf_m, -np.inf)
        j = int(np.argmax(c))  # first maximum: lowest position
        new_tok[j] = tok_m[j]
        n_acc = 1
    dec = new_tok >= 0
    tokens[win[dec]] = new_tok[dec]
    still = tokens[win] < 0
    draft[win[still]] = tok_m[still]
    draft[win[~still]] = -1
    if not still.any() and ws + 2 * W <= gen_end:  # the next window fits in the span
        ws = ws + W
        draft[ws:ws + W] = -1
    return {"tokens": tokens, "draft": draft, "ws": ws, "n_accepted": n_acc}


def decode_iteration_sequence(layers, final_norm, w_lm, embed, tokens, draft, tracked, ws: int,
                              gen_end: int, k_caches_b, v_caches_b, W: int, mask_id: int,
                              threshold: float, n_heads: int, head_dim: int, theta: float):
    """One decode iteration of one sequence: both views of the model step from
    the same caches, acceptance and window advance, reselection of the tracked
    positions.  Returns the new state and the caches after the iteration (the
    draft view writes last, so its rows are what the caches keep)."""
    from . import model_oracle as mo
    from .flashcache_oracle import topk_tracked

    K = len(tracked)
    pos, ids_m, ids_d = build_query(tokens, draft, tracked, ws, W, mask_id)
    head_rows = np.arange(K, K + W)
    e = np.asarray(embed, np.float64)
    rm = mo.model_step_sequence(e[ids_m], layers, final_norm, w_lm, pos, k_caches_b, v_caches_b,
                                head_rows, n_heads, head_dim, theta, threshold)
    rd = mo.model_step_sequence(e[ids_d], layers, final_norm, w_lm, pos, k_caches_b, v_caches_b,
                                head_rows, n_heads, head_dim, theta, threshold)
    st = accept_and_advance(tokens, draft, ws, W, gen_end, rm["token"], rm["confidence"],
                            rd["token"], rd["confidence"], threshold)
    L = len(tokens)
    tr = topk_tracked(rd["importance"], np.array([0, L]), np.array([0]), np.array([st["ws"]]),
                      np.array([K]), K)[0]
    return {**st, "tracked": tr, "k_caches": rd["k_caches"], "v_caches": rd["v_caches"],
            "importance": rd["importance"], "mask": rm, "draft_view": rd, "pos": pos}
