"""fp64 CPU oracle of the full model step around the Flash-Cache layer.
TEST INFRASTRUCTURE ONLY: nothing in the product path imports this module.

The pages evaluate Flash-dLLM on LLaDA-8B (paper-digest page, the evaluation
section; forum post quoting the README, configuration table).  One step of the
model runs every query row of a sequence (its tracked positions and its masked
window) through the decoder stack, attending in every layer through the
Flash-Cache step (projection, RoPE, cache write, bidirectional attention over
the whole cache, importance), then scores the window rows with the LM head;
Flash-Verify accepts a window position when the model's confidence in its top
token reaches the threshold (paper-digest page, the Flash-Verify description;
threshold 0.9 in the configuration).

Readings taken where the pages are silent (the decoder follows the LLaMA-style
layer that LLaDA-8B uses):

* layer: h += Wo . attn(rms_norm(h) * g_attn);  h += Wd . (silu(Wg . m) * Wu . m)
  with m = rms_norm(h) * g_mlp; no biases; final rms_norm(h) * g_final before
  the LM head;
* rms_norm(x) = x / sqrt(mean(x^2) + eps), eps = 1e-5;
* every operation reads and writes bf16 tensors, as the device does between
  kernels: its result is rounded to bf16 (``act_round``); inside an operation
  the arithmetic is exact (float64).  The KV caches store bf16 as in the
  single-layer oracle;
* importance is summed over every layer of the step (one tracked set serves
  all layers);
* confidence of a row = the largest softmax probability over the vocabulary;
  its token = the index of the largest logit, lowest index on ties; accepted
  when confidence >= threshold.

Each function is pinned by tests under ``tests/test_model_oracle.py`` against
closed forms, torch library routines and invariants.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import numpy as np

from .flashcache_oracle import bf16_round, step_sequence

RMS_EPS = 1e-5


def act_round(a: np.ndarray, act_dtype: Optional[str]) -> np.ndarray:
    """Value of ``a`` once stored as an activation of ``act_dtype`` (None = exact)."""
    a = np.asarray(a, np.float64)
    if act_dtype is None:
        return a
    if act_dtype == "bf16":
        return bf16_round(a)
    raise ValueError(act_dtype)


def rms_norm(x: np.ndarray, g: np.ndarray, eps: float = RMS_EPS) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * g, row-wise over the last axis.

    Pinned by the constant-vector closed form, by scale invariance (eps -> 0)
    and against torch.nn.functional.rms_norm in float64.
    """
    x = np.asarray(x, np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, np.float64)


def silu(u: np.ndarray) -> np.ndarray:
    """u * sigmoid(u) = u / (1 + exp(-u)).

    Pinned by silu(0) = 0, the odd-part identity silu(u) - silu(-u) = u, the
    large-|u| limits and torch.nn.functional.silu.
    """
    u = np.asarray(u, np.float64)
    return u / (1.0 + np.exp(-u))


def swiglu_mlp(m: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray,
               act_dtype: Optional[str] = None) -> np.ndarray:
    """Wd . (silu(Wg . m) * (Wu . m)) for every row of m [n, D].

    The gated product is an activation of its own (rounded by ``act_dtype``)
    before the down projection.  Pinned by a diagonal-weight closed form.
    """
    m = np.asarray(m, np.float64)
    g = m @ np.asarray(w_gate, np.float64).T
    u = m @ np.asarray(w_up, np.float64).T
    s = act_round(silu(g) * u, act_dtype)
    return s @ np.asarray(w_down, np.float64).T


def lm_head_confidence(h: np.ndarray, w_lm: np.ndarray) -> Dict[str, np.ndarray]:
    """Logits = h . W_lm^T; per row the argmax token (lowest index on ties), the
    softmax probability of that token (the confidence) and the logits.

    Pinned by planted one-hot logits (closed-form confidence), uniform logits
    (confidence 1/V) and tie order.
    """
    logits = np.asarray(h, np.float64) @ np.asarray(w_lm, np.float64).T
    top = np.argmax(logits, axis=1)  # first maximum = lowest index
    mx = logits[np.arange(logits.shape[0]), top]
    conf = 1.0 / np.exp(logits - mx[:, None]).sum(axis=1)
    return {"token": top.astype(np.int64), "confidence": conf, "logits": logits}


def decoder_layer_sequence(h_b, lw: Dict[str, np.ndarray], pos_b, k_cache_b, v_cache_b,
                           n_heads: int, head_dim: int, theta: float,
                           act_dtype: Optional[str], cache_dtype: Optional[str]):
    """One decoder layer for one sequence's query rows h_b [n, D].

    Returns the new residual stream, the layer's new caches and its importance.
    """
    a = act_round(rms_norm(h_b, lw["attn_norm"]), act_dtype)
    st = step_sequence(a, lw["w_qkv"], pos_b, k_cache_b, v_cache_b, n_heads, head_dim, theta,
                       cache_dtype)
    o = act_round(st["out"], act_dtype).reshape(a.shape[0], n_heads * head_dim)
    h = act_round(h_b + o @ np.asarray(lw["w_o"], np.float64).T, act_dtype)
    m = act_round(rms_norm(h, lw["mlp_norm"]), act_dtype)
    h = act_round(h + swiglu_mlp(m, lw["w_gate"], lw["w_up"], lw["w_down"], act_dtype), act_dtype)
    return h, st["k_cache"], st["v_cache"], st["importance"]


def model_step_sequence(x_b, layers: Sequence[Dict[str, np.ndarray]], final_norm, w_lm, pos_b,
                        k_caches_b: List[np.ndarray], v_caches_b: List[np.ndarray],
                        head_rows: np.ndarray, n_heads: int, head_dim: int, theta: float,
                        threshold: float = 0.9, act_dtype: Optional[str] = "bf16",
                        cache_dtype: Optional[str] = "bf16") -> Dict[str, object]:
    """The model step for one sequence: every layer, then the LM head on the
    rows ``head_rows`` (indices into the sequence's query rows).

    Returns the final residual stream, per-layer caches, the importance summed
    over layers, and per head row the token, confidence and acceptance.
    """
    h = act_round(x_b, act_dtype)
    imp = None
    kcs, vcs = [], []
    for l, lw in enumerate(layers):
        h, kc, vc, im = decoder_layer_sequence(h, lw, pos_b, k_caches_b[l], v_caches_b[l],
                                               n_heads, head_dim, theta, act_dtype, cache_dtype)
        kcs.append(kc)
        vcs.append(vc)
        imp = im if imp is None else imp + im
    hn = act_round(rms_norm(h[np.asarray(head_rows)], final_norm), act_dtype)
    lm = lm_head_confidence(hn, w_lm)
    return {"h": h, "k_caches": kcs, "v_caches": vcs, "importance": imp,
            "token": lm["token"], "confidence": lm["confidence"], "logits": lm["logits"],
            "accept": lm["confidence"] >= threshold}
