"""Pins of the decode-iteration oracle: query building, acceptance, drafts and
window advance on hand-worked cases; the composed iteration against a torch
restatement of a one-layer model's draft view (caches, importance, reselection)
and against the closed-form outcomes of uniform logits."""
import math

import numpy as np
import torch

from oracle import decode_oracle as do


def test_build_query_views():
    tokens = np.array([7, 8, 9, -1, 4, -1, -1, -1])
    draft = np.array([-1, -1, -1, 11, -1, -1, 12, -1])
    pos, im, idr = do.build_query(tokens, draft, np.array([1, 0]), ws=3, W=4, mask_id=99)
    assert list(pos) == [1, 0, 3, 4, 5, 6]
    assert list(im) == [8, 7, 99, 4, 99, 99]       # undecided rows read [MASK]
    assert list(idr) == [8, 7, 11, 4, 99, 12]      # or their draft when there is one


def _acc(tokens, draft, ws, W, gen_end, tm, cm, td, cd, thr=0.9):
    return do.accept_and_advance(np.array(tokens), np.array(draft), ws, W, gen_end,
                                 np.array(tm), np.array(cm), np.array(td), np.array(cd), thr)


def test_accept_by_confidence_and_by_verified_draft():
    r = _acc([1, 2, -1, -1, -1, -1], [-1, -1, -1, 5, 6, -1], 2, 4, 6,
             tm=[10, 11, 12, 13], cm=[0.95, 0.1, 0.2, 0.3],
             td=[20, 5, 7, 21], cd=[0.1, 0.91, 0.99, 0.5])
    # pos 2: [MASK]-view confidence 0.95 -> token 10
    # pos 3: draft 5 predicted by the draft view with 0.91 -> verified, token 5
    # pos 4: draft 6 but the draft view predicts 7 -> not verified
    # pos 5: nothing reaches the threshold
    assert list(r["tokens"]) == [1, 2, 10, 5, -1, -1] and r["n_accepted"] == 2
    assert list(r["draft"][4:]) == [12, 13]  # drafts := [MASK]-view predictions
    assert r["ws"] == 2


def test_at_least_one_token_lowest_position_on_ties():
    r = _acc([1, -1, -1, -1], [-1] * 4, 1, 3, 4, tm=[5, 6, 7], cm=[0.3, 0.5, 0.5],
             td=[0, 0, 0], cd=[0.0, 0.0, 0.0])
    assert list(r["tokens"]) == [1, -1, 6, -1] and r["n_accepted"] == 1
    assert list(r["draft"]) == [-1, 5, -1, 7]


def test_window_advances_when_complete_but_not_past_the_span():
    r = _acc([1, 2, -1, -1, -1, -1], [-1] * 6, 2, 2, 6, tm=[3, 4], cm=[0.95, 0.97],
             td=[0, 0], cd=[0.0, 0.0])
    assert list(r["tokens"][:4]) == [1, 2, 3, 4] and r["ws"] == 4
    r = _acc([1, 2, 3, 4, -1, -1], [-1] * 6, 4, 2, 6, tm=[5, 6], cm=[0.95, 0.97],
             td=[0, 0], cd=[0.0, 0.0])
    assert list(r["tokens"]) == [1, 2, 3, 4, 5, 6] and r["ws"] == 4  # the last window stays


def test_decided_positions_are_left_alone():
    r = _acc([1, 2, 3, -1], [-1, -1, 9, 9], 2, 2, 4, tm=[8, 8], cm=[0.99, 0.1],
             td=[9, 9], cd=[0.99, 0.99])
    # pos 2 is decided already (token 3) whatever the views say; pos 3's draft 9 is verified
    assert list(r["tokens"]) == [1, 2, 3, 9] and r["n_accepted"] == 1


def test_window_does_not_advance_past_the_span():
    # span [2, 7): after the window [2, 4) the next one [4, 6) fits, after [4, 6) the
    # next one [6, 8) would not
    r = _acc([1, 2, -1, -1, -1, -1, -1], [-1] * 7, 2, 2, 7, tm=[3, 4], cm=[0.95, 0.97],
             td=[0, 0], cd=[0.0, 0.0])
    assert r["ws"] == 4
    r = _acc([1, 2, 3, 4, -1, -1, -1], [-1] * 7, 4, 2, 7, tm=[5, 6], cm=[0.95, 0.97],
             td=[0, 0], cd=[0.0, 0.0])
    assert r["ws"] == 4


def test_threshold_is_inclusive():
    # two undecided positions exactly at the threshold: both accepted by the [MASK]
    # view (a strict comparison would fall back to the single at-least-one token)
    r = _acc([1, -1, -1], [-1] * 3, 1, 2, 3, tm=[4, 5], cm=[0.9, 0.9], td=[0, 0], cd=[0.0, 0.0])
    assert list(r["tokens"]) == [1, 4, 5] and r["n_accepted"] == 2
    # a draft verified at exactly the threshold is accepted too
    r = _acc([1, -1, -1], [-1, 6, -1], 1, 2, 3, tm=[4, 5], cm=[0.1, 0.2], td=[6, 0], cd=[0.9, 0.0])
    assert list(r["tokens"]) == [1, 6, -1] and r["n_accepted"] == 1


def test_decided_positions_carry_no_draft():
    r = _acc([1, -1, -1, -1], [-1, 8, 9, -1], 1, 3, 4, tm=[5, 6, 7], cm=[0.95, 0.2, 0.1],
             td=[0, 9, 0], cd=[0.0, 0.95, 0.0])
    # pos 1 by confidence, pos 2 by its verified draft; pos 3 stays undecided
    assert list(r["tokens"]) == [1, 5, 9, -1]
    assert list(r["draft"]) == [-1, -1, -1, 7]


# ------------------------------------------------ the whole iteration, composed
# A one-layer model small enough to restate the draft view's first layer with
# torch routines (rms_norm, complex-multiplication RoPE, softmax), independently
# of the oracle's own functions.
_D, _H, _d, _V, _L, _P, _K, _W, _THETA = 32, 2, 16, 40, 24, 12, 3, 4, 1e4


def _bf16(t):
    return t.to(torch.bfloat16).to(torch.float64)


def _decode_case(seed):
    from test_model_oracle import _tiny_model

    rng = np.random.default_rng(seed)
    layers, fn, wlm = _tiny_model(rng, 1, D=_D, H=_H, d=_d, V=_V)
    emb = rng.standard_normal((_V, _D))
    tokens = np.full(_L, -1)
    tokens[:_P] = rng.integers(0, _V - 1, _P)
    draft = np.full(_L, -1)
    draft[_P + 1], draft[_P + 3] = 5, 7
    tracked = np.sort(rng.choice(_P, size=_K, replace=False))
    kc, vc = rng.standard_normal((_L, _H, _d)), rng.standard_normal((_L, _H, _d))
    return dict(layers=layers, fn=fn, wlm=wlm, emb=emb, tokens=tokens, draft=draft,
                tracked=tracked, kc=kc, vc=vc)


def _first_layer_by_torch(c, view):
    """Layer-0 caches and importance of one view, restated with torch."""
    pos = np.concatenate([c["tracked"], np.arange(_P, _P + _W)])
    ids = c["tokens"][pos].copy()
    und = ids < 0
    if view == "draft":
        d = c["draft"][pos]
        ids[und] = np.where(d[und] >= 0, d[und], _V - 1)
    else:
        ids[und] = _V - 1
    lw = c["layers"][0]
    x = _bf16(torch.from_numpy(c["emb"][ids]))
    a = _bf16(torch.nn.functional.rms_norm(x, (_D,), torch.from_numpy(lw["attn_norm"]), eps=1e-5))
    y = (a @ torch.from_numpy(lw["w_qkv"]).T).numpy()
    n, hd = len(pos), _H * _d
    q, k, v = (y[:, i * hd:(i + 1) * hd].reshape(n, _H, _d) for i in range(3))
    ang = np.outer(pos, _THETA ** (-np.arange(0, _d, 2) / _d))[:, None, :]

    def rot(u):
        z = (u[..., :_d // 2] + 1j * u[..., _d // 2:]) * np.exp(1j * ang)
        return np.concatenate([z.real, z.imag], axis=-1)

    kc, vc = c["kc"].copy(), c["vc"].copy()
    kc[pos] = _bf16(torch.from_numpy(rot(k))).numpy()
    vc[pos] = _bf16(torch.from_numpy(v)).numpy()
    s = torch.einsum("nhd,lhd->hnl", torch.from_numpy(rot(q)), torch.from_numpy(kc)) / math.sqrt(_d)
    imp = torch.softmax(s, dim=-1).sum(dim=(0, 1)).numpy()
    return kc, vc, imp


def _top(imp, hi):
    j = np.arange(hi)
    return j[np.lexsort((j, -imp[:hi]))][:_K]


def _run(c, threshold, final_norm=None):
    fn = c["fn"] if final_norm is None else final_norm
    return do.decode_iteration_sequence(c["layers"], fn, c["wlm"], c["emb"], c["tokens"], c["draft"],
                                        c["tracked"], _P, _L, [c["kc"]], [c["vc"]], _W, _V - 1,
                                        threshold, _H, _d, _THETA)


def _discriminating_case():
    """A seeded case whose top-K differs between the two views' importance and
    between the old and the advanced window start, so that swapping either
    changes the tracked set."""
    for seed in range(40):
        c = _decode_case(seed)
        _, _, imp_d = _first_layer_by_torch(c, "draft")
        _, _, imp_m = _first_layer_by_torch(c, "mask")
        t_adv = _top(imp_d, _P + _W)
        if (set(_top(imp_m, _P)) != set(_top(imp_d, _P)) and set(t_adv) != set(_top(imp_d, _P))):
            return c
    raise AssertionError("no discriminating seed")


def test_iteration_keeps_the_draft_view_and_reselects_from_it():
    c = _discriminating_case()
    r = _run(c, 0.9)
    kc, vc, imp = _first_layer_by_torch(c, "draft")
    np.testing.assert_allclose(r["k_caches"][0], kc, rtol=1e-12, atol=0)
    np.testing.assert_allclose(r["v_caches"][0], vc, rtol=1e-12, atol=0)
    np.testing.assert_allclose(r["importance"], imp, rtol=1e-10)
    assert r["ws"] == _P
    assert list(r["tracked"]) == list(_top(imp, _P))


def test_iteration_threshold_zero_accepts_the_window_and_advances():
    """A zero final norm makes every logit 0: token 0 (lowest index) with
    confidence 1/V everywhere; threshold 0 accepts the whole window, which then
    advances, and the tracked set is drawn from the grown prefix."""
    c = _discriminating_case()
    r = _run(c, 0.0, final_norm=np.zeros(_D))
    np.testing.assert_allclose(r["mask"]["confidence"], 1.0 / _V, rtol=1e-12)
    assert list(r["tokens"][_P:_P + _W]) == [0] * _W and r["n_accepted"] == _W
    assert r["ws"] == _P + _W
    assert (r["draft"] == -1).all()
    _, _, imp = _first_layer_by_torch(c, "draft")
    assert list(r["tracked"]) == list(_top(imp, _P + _W))


def test_iteration_without_confident_rows_decodes_exactly_one():
    c = _discriminating_case()
    r = _run(c, 0.9, final_norm=np.zeros(_D))
    # all confidences tie at 1/V: the lowest undecided position takes token 0
    assert list(r["tokens"][_P:_P + _W]) == [0, -1, -1, -1] and r["n_accepted"] == 1
    # the other window positions' drafts become the [MASK] view's token 0
    assert list(r["draft"][_P:_P + _W]) == [-1, 0, 0, 0]
    assert r["ws"] == _P
