"""The model-step and decode-iteration pins against planted mistakes.

Each case plants a plausible mistake in the model or decode oracle (on the
CPU only) and checks that at least one pin of tests/test_model_oracle.py or
tests/test_decode_oracle.py then fails, so a pin that can never fail is
noticed.
"""
import inspect

import numpy as np
import pytest

from oracle import decode_oracle as do
from oracle import model_oracle as mo
from oracle.flashcache_oracle import step_sequence, topk_tracked
import test_decode_oracle as decode_pins
import test_model_oracle as model_pins

_real = {name: getattr(mo, name) for name in ("rms_norm", "silu", "swiglu_mlp",
                                              "lm_head_confidence", "decoder_layer_sequence")}


# ----------------------------------------------------------------- model mutants
def _rms_sum(x, g, eps=mo.RMS_EPS):
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps) * np.asarray(g, np.float64)


def _rms_no_gain(x, g, eps=mo.RMS_EPS):
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def _rms_eps_outside(x, g, eps=mo.RMS_EPS):
    x = np.asarray(x, np.float64)
    return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps) * np.asarray(g, np.float64)


def _silu_sigmoid_only(u):
    return 1.0 / (1.0 + np.exp(-np.asarray(u, np.float64)))


def _silu_gelu_tanh(u):
    u = np.asarray(u, np.float64)
    return 0.5 * u * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (u + 0.044715 * u ** 3)))


def _swiglu_gate_up_swapped(m, w_gate, w_up, w_down, act_dtype=None):
    return _real["swiglu_mlp"](m, w_up, w_gate, w_down, act_dtype)


def _swiglu_silu_of_product(m, w_gate, w_up, w_down, act_dtype=None):
    m = np.asarray(m, np.float64)
    g, u = m @ np.asarray(w_gate).T, m @ np.asarray(w_up).T
    return mo.act_round(_real["silu"](g * u), act_dtype) @ np.asarray(w_down).T


def _lm_ties_to_highest_index(h, w_lm):
    r = _real["lm_head_confidence"](h, w_lm)
    lg = r["logits"]
    top = lg.shape[1] - 1 - np.argmax(lg[:, ::-1], axis=1)
    return {**r, "token": top.astype(np.int64)}


def _lm_softmax_over_rows(h, w_lm):
    r = _real["lm_head_confidence"](h, w_lm)
    lg, top = r["logits"], r["token"]
    e = np.exp(lg - lg.max(axis=0, keepdims=True))
    p = e / e.sum(axis=0, keepdims=True)  # normalised over rows instead of the vocabulary
    return {**r, "confidence": p[np.arange(len(top)), top]}


def _layer_variant(no_attn_residual=False, mlp_norm_key="mlp_norm", mlp_from_input=False):
    def layer(h_b, lw, pos_b, k_cache_b, v_cache_b, n_heads, head_dim, theta, act_dtype,
              cache_dtype):
        a = mo.act_round(mo.rms_norm(h_b, lw["attn_norm"]), act_dtype)
        st = step_sequence(a, lw["w_qkv"], pos_b, k_cache_b, v_cache_b, n_heads, head_dim, theta,
                           cache_dtype)
        o = mo.act_round(st["out"], act_dtype).reshape(a.shape[0], n_heads * head_dim)
        proj = o @ np.asarray(lw["w_o"], np.float64).T
        h = mo.act_round(proj if no_attn_residual else h_b + proj, act_dtype)
        m = mo.act_round(mo.rms_norm(h_b if mlp_from_input else h, lw[mlp_norm_key]), act_dtype)
        h = mo.act_round(h + mo.swiglu_mlp(m, lw["w_gate"], lw["w_up"], lw["w_down"], act_dtype),
                         act_dtype)
        return h, st["k_cache"], st["v_cache"], st["importance"]
    return layer


def _model_step_variant(last_layer_importance=False, no_final_norm=False):
    def step(x_b, layers, final_norm, w_lm, pos_b, k_caches_b, v_caches_b, head_rows, n_heads,
             head_dim, theta, threshold=0.9, act_dtype="bf16", cache_dtype="bf16"):
        h = mo.act_round(x_b, act_dtype)
        imp, kcs, vcs = None, [], []
        for l, lw in enumerate(layers):
            h, kc, vc, im = mo.decoder_layer_sequence(h, lw, pos_b, k_caches_b[l], v_caches_b[l],
                                                      n_heads, head_dim, theta, act_dtype,
                                                      cache_dtype)
            kcs.append(kc)
            vcs.append(vc)
            imp = im if (imp is None or last_layer_importance) else imp + im
        hr = h[np.asarray(head_rows)]
        hn = mo.act_round(hr if no_final_norm else mo.rms_norm(hr, final_norm), act_dtype)
        lm = mo.lm_head_confidence(hn, w_lm)
        return {"h": h, "k_caches": kcs, "v_caches": vcs, "importance": imp,
                "token": lm["token"], "confidence": lm["confidence"], "logits": lm["logits"],
                "accept": lm["confidence"] >= threshold}
    return step


# ----------------------------------------------------------------- decode mutants
def _query_ignores_drafts(tokens, draft, tracked, ws, W, mask_id):
    pos = np.concatenate([np.asarray(tracked, np.int64), np.arange(ws, ws + W)])
    ids = tokens[pos].copy()
    ids[ids < 0] = mask_id
    return pos, ids, ids.copy()


def _accept_variant(strict=False, unverified_drafts=False, ties_high=False, loose_advance=False,
                    keep_stale_drafts=False, no_new_drafts=False):
    def accept(tokens, draft, ws, W, gen_end, tok_m, conf_m, tok_d, conf_d, threshold):
        tokens, draft = tokens.copy(), draft.copy()
        win = np.arange(ws, ws + W)
        und = tokens[win] < 0
        ge = (lambda c: c > threshold) if strict else (lambda c: c >= threshold)
        acc_m = und & ge(conf_m)
        verified = np.ones(W, bool) if unverified_drafts else (tok_d == draft[win])
        acc_d = und & ~acc_m & (draft[win] >= 0) & verified & ge(conf_d)
        new_tok = np.where(acc_m, tok_m, np.where(acc_d, draft[win], -1))
        n_acc = int((acc_m | acc_d).sum())
        if n_acc == 0 and und.any():
            c = np.where(und, conf_m, -np.inf)
            j = (W - 1 - int(np.argmax(c[::-1]))) if ties_high else int(np.argmax(c))
            new_tok[j] = tok_m[j]
            n_acc = 1
        dec = new_tok >= 0
        tokens[win[dec]] = new_tok[dec]
        still = tokens[win] < 0
        if not no_new_drafts:
            draft[win[still]] = tok_m[still]
        if not keep_stale_drafts:
            draft[win[~still]] = -1
        fits = ws + W <= gen_end if loose_advance else ws + 2 * W <= gen_end
        if not still.any() and fits:
            ws = ws + W
            draft[ws:ws + W] = -1
        return {"tokens": tokens, "draft": draft, "ws": ws, "n_accepted": n_acc}
    return accept


def _iteration_variant(imp_view="draft", cache_view="draft", old_ws_candidates=False):
    def iteration(layers, final_norm, w_lm, embed, tokens, draft, tracked, ws, gen_end,
                  k_caches_b, v_caches_b, W, mask_id, threshold, n_heads, head_dim, theta):
        K = len(tracked)
        pos, ids_m, ids_d = do.build_query(tokens, draft, tracked, ws, W, mask_id)
        rows = np.arange(K, K + W)
        e = np.asarray(embed, np.float64)
        views = {v: mo.model_step_sequence(e[ids], layers, final_norm, w_lm, pos, k_caches_b,
                                           v_caches_b, rows, n_heads, head_dim, theta, threshold)
                 for v, ids in (("mask", ids_m), ("draft", ids_d))}
        rm, rd = views["mask"], views["draft"]
        st = do.accept_and_advance(tokens, draft, ws, W, gen_end, rm["token"], rm["confidence"],
                                   rd["token"], rd["confidence"], threshold)
        hi = ws if old_ws_candidates else st["ws"]
        L = len(tokens)
        tr = topk_tracked(views[imp_view]["importance"], np.array([0, L]), np.array([0]),
                          np.array([hi]), np.array([K]), K)[0]
        kv = views[cache_view]
        return {**st, "tracked": tr, "k_caches": kv["k_caches"], "v_caches": kv["v_caches"],
                "importance": rd["importance"], "mask": rm, "draft_view": rd, "pos": pos}
    return iteration


def _run_all_pins():
    """Run every pin of the model and decode oracles; return how many failed."""
    failures = 0
    for mod in (model_pins, decode_pins):
        for name, fn in inspect.getmembers(mod, inspect.isfunction):
            if not name.startswith("test_") or fn.__module__ != mod.__name__:
                continue
            try:
                fn()
            except Exception:  # a planted mistake may also break a pin's preconditions
                failures += 1
    return failures


MUTANTS = [
    (mo, "rms_norm", _rms_sum),
    (mo, "rms_norm", _rms_no_gain),
    (mo, "rms_norm", _rms_eps_outside),
    (mo, "silu", _silu_sigmoid_only),
    (mo, "silu", _silu_gelu_tanh),
    (mo, "swiglu_mlp", _swiglu_gate_up_swapped),
    (mo, "swiglu_mlp", _swiglu_silu_of_product),
    (mo, "lm_head_confidence", _lm_ties_to_highest_index),
    (mo, "lm_head_confidence", _lm_softmax_over_rows),
    (mo, "decoder_layer_sequence", _layer_variant(no_attn_residual=True)),
    (mo, "decoder_layer_sequence", _layer_variant(mlp_norm_key="attn_norm")),
    (mo, "decoder_layer_sequence", _layer_variant(mlp_from_input=True)),
    (mo, "model_step_sequence", _model_step_variant(last_layer_importance=True)),
    (mo, "model_step_sequence", _model_step_variant(no_final_norm=True)),
    (do, "build_query", _query_ignores_drafts),
    (do, "accept_and_advance", _accept_variant(strict=True)),
    (do, "accept_and_advance", _accept_variant(unverified_drafts=True)),
    (do, "accept_and_advance", _accept_variant(ties_high=True)),
    (do, "accept_and_advance", _accept_variant(loose_advance=True)),
    (do, "accept_and_advance", _accept_variant(keep_stale_drafts=True)),
    (do, "accept_and_advance", _accept_variant(no_new_drafts=True)),
    (do, "decode_iteration_sequence", _iteration_variant(imp_view="mask")),
    (do, "decode_iteration_sequence", _iteration_variant(cache_view="mask")),
    (do, "decode_iteration_sequence", _iteration_variant(old_ws_candidates=True)),
]


@pytest.mark.parametrize("module,target,bad", MUTANTS,
                         ids=[f"{t}-{i}" for i, (_, t, _) in enumerate(MUTANTS)])
def test_planted_mistake_is_caught(monkeypatch, module, target, bad):
    monkeypatch.setattr(module, target, bad)
    assert _run_all_pins() >= 1, f"no pin caught the planted mistake in {target}"


def test_the_unmutated_variants_pass_every_pin(monkeypatch):
    """The mutant builders with every switch off are the oracle itself: each
    passes all pins, so a caught mutant is caught for its one planted change."""
    for module, target, good in [(mo, "decoder_layer_sequence", _layer_variant()),
                                 (mo, "model_step_sequence", _model_step_variant()),
                                 (do, "accept_and_advance", _accept_variant()),
                                 (do, "decode_iteration_sequence", _iteration_variant())]:
        with monkeypatch.context() as m:
            m.setattr(module, target, good)
            assert _run_all_pins() == 0, target


def test_pins_pass_on_the_real_oracles():
    assert _run_all_pins() == 0
