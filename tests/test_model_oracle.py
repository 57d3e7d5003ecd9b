"""Pins of the model-step oracle (RMSNorm, SwiGLU MLP, LM-head confidence and
their composition) against closed forms, torch routines and invariants."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import model_oracle as mo


# ----------------------------------------------------------------- rms_norm
def test_rms_norm_constant_vector_closed_form():
    # x = c * 1 (length D): mean(x^2) = c^2, so y = c / sqrt(c^2 + eps) * g
    for c in (3.0, -0.5, 1e-3):
        x = np.full((1, 8), c)
        g = np.linspace(0.5, 2.0, 8)
        y = mo.rms_norm(x, g, eps=1e-5)
        np.testing.assert_allclose(y[0], c / math.sqrt(c * c + 1e-5) * g, rtol=1e-14)


def test_rms_norm_matches_torch_and_is_scale_invariant():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 64))
    g = rng.standard_normal(64)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(g), eps=1e-5)
    np.testing.assert_allclose(mo.rms_norm(x, g), ref.numpy(), rtol=1e-12, atol=1e-12)
    # without eps the result does not depend on the row's scale
    np.testing.assert_allclose(mo.rms_norm(7.5 * x, g, eps=0.0), mo.rms_norm(x, g, eps=0.0),
                               rtol=1e-12)


# ----------------------------------------------------------------- silu / mlp
def test_silu_identities_and_torch():
    u = np.linspace(-20, 20, 81)
    s = mo.silu(u)
    assert mo.silu(np.array([0.0]))[0] == 0.0
    # silu(u) - silu(-u) = u * (sigmoid(u) + sigmoid(-u)) = u
    np.testing.assert_allclose(s - mo.silu(-u), u, rtol=1e-12, atol=1e-12)
    # large |u|: silu(u) -> u for u >> 0 and -> 0 for u << 0
    assert abs(mo.silu(np.array([40.0]))[0] - 40.0) < 1e-12
    assert abs(mo.silu(np.array([-40.0]))[0]) < 1e-15
    np.testing.assert_allclose(s, torch.nn.functional.silu(torch.from_numpy(u)).numpy(), rtol=1e-12)


def test_swiglu_hand_worked_example():
    # identity weights, m = [1, -2]: out = [silu(1) * 1, silu(-2) * (-2)]
    # silu(1) = 1 / (1 + e^-1) = 0.7310585786300049
    # silu(-2) * (-2) = 4 / (1 + e^2) = 0.47681168808847233
    eye = np.eye(2)
    out = mo.swiglu_mlp(np.array([[1.0, -2.0]]), eye, eye, eye)
    np.testing.assert_allclose(out[0], [0.7310585786300049, 0.47681168808847233], rtol=1e-14)


def test_swiglu_gate_and_up_roles_are_not_swapped():
    # gate 0 makes the output 0 whatever the up branch; up 0 likewise
    m = np.array([[0.3, 1.7]])
    eye, z = np.eye(2), np.zeros((2, 2))
    assert np.all(mo.swiglu_mlp(m, z, eye, eye) == 0.0)
    assert np.all(mo.swiglu_mlp(m, eye, z, eye) == 0.0)
    # a gate of +40 passes the up branch unchanged (silu(40) = 40 within 1e-15 relative)
    out = mo.swiglu_mlp(m, 40.0 * np.eye(2) / m[0], np.eye(2), np.eye(2))
    np.testing.assert_allclose(out[0], 40.0 * m[0], rtol=1e-12)


# ----------------------------------------------------------------- LM head
def test_lm_head_planted_logit_closed_form():
    V, D, z, k = 50, 4, 3.0, 17
    w = np.zeros((V, D))
    w[k, 0] = z
    h = np.array([[1.0, 0.0, 0.0, 0.0]])
    r = mo.lm_head_confidence(h, w)
    assert r["token"][0] == k
    np.testing.assert_allclose(r["confidence"][0], math.exp(z) / (math.exp(z) + V - 1), rtol=1e-13)


def test_lm_head_uniform_and_ties():
    V, D = 10, 3
    r = mo.lm_head_confidence(np.ones((2, D)), np.zeros((V, D)))
    assert list(r["token"]) == [0, 0]
    np.testing.assert_allclose(r["confidence"], 1.0 / V, rtol=1e-14)
    w = np.zeros((V, D))
    w[4, 0] = w[7, 0] = 2.0  # two equal maxima: the lower index wins
    r = mo.lm_head_confidence(np.array([[1.0, 0, 0]]), w)
    assert r["token"][0] == 4
    np.testing.assert_allclose(r["confidence"][0], math.exp(2) / (2 * math.exp(2) + V - 2), rtol=1e-13)


# ----------------------------------------------------------------- composition
def _tiny_model(rng, n_layers, D=32, H=2, d=16, I=48, V=40):
    def w(*shape):
        return rng.standard_normal(shape) * 0.2

    layers = [dict(attn_norm=1 + 0.1 * rng.standard_normal(D), w_qkv=w(3 * H * d, D),
                   w_o=w(D, H * d), mlp_norm=1 + 0.1 * rng.standard_normal(D), w_gate=w(I, D),
                   w_up=w(I, D), w_down=w(D, I)) for _ in range(n_layers)]
    return layers, 1 + 0.1 * rng.standard_normal(D), w(V, D)


def test_residual_identity_when_outputs_are_zero():
    """With Wo = 0 and Wd = 0 every layer leaves the residual stream as it is, the
    caches are still written and the importance is n_layers * H * n in total."""
    rng = np.random.default_rng(1)
    L, n, H, d = 24, 5, 2, 16
    layers, fn, wlm = _tiny_model(rng, 3)
    for lw in layers:
        lw["w_o"][:] = 0.0
        lw["w_down"][:] = 0.0
    x = rng.standard_normal((n, 32))
    pos = np.array([0, 3, 9, 10, 23])
    kcs = [rng.standard_normal((L, H, d)) for _ in layers]
    vcs = [rng.standard_normal((L, H, d)) for _ in layers]
    r = mo.model_step_sequence(x, layers, fn, wlm, pos, kcs, vcs, np.arange(n), H, d, 1e4,
                               act_dtype=None, cache_dtype=None)
    np.testing.assert_allclose(r["h"], x, rtol=0, atol=0)
    assert abs(r["importance"].sum() - 3 * H * n) < 1e-9
    lm = mo.lm_head_confidence(mo.rms_norm(x, fn), wlm)
    np.testing.assert_array_equal(r["token"], lm["token"])
    for l in range(3):
        assert not np.allclose(r["k_caches"][l][pos], kcs[l][pos])  # refreshed rows
        others = np.setdiff1d(np.arange(L), pos)
        np.testing.assert_array_equal(r["k_caches"][l][others], kcs[l][others])


def test_first_layer_attention_is_the_flashcache_step():
    """The attention inside the layer is exactly the single-layer step applied to
    rms_norm(x) * g_attn (same caches, same importance)."""
    rng = np.random.default_rng(2)
    L, n, H, d = 30, 6, 2, 16
    layers, fn, wlm = _tiny_model(rng, 1)
    x = rng.standard_normal((n, 32))
    pos = rng.choice(L, size=n, replace=False)
    kc, vc = rng.standard_normal((L, H, d)), rng.standard_normal((L, H, d))
    r = mo.model_step_sequence(x, layers, fn, wlm, pos, [kc], [vc], np.arange(n), H, d, 1e4,
                               act_dtype=None, cache_dtype=None)
    st = oracle.step_sequence(mo.rms_norm(x, layers[0]["attn_norm"]), layers[0]["w_qkv"], pos,
                              kc, vc, H, d, 1e4, None)
    np.testing.assert_allclose(r["importance"], st["importance"], rtol=1e-13)
    np.testing.assert_allclose(r["k_caches"][0], st["k_cache"], rtol=1e-13)
    o = st["out"].reshape(n, H * d)
    h1 = x + o @ layers[0]["w_o"].T
    m = mo.rms_norm(h1, layers[0]["mlp_norm"])
    # the MLP adds on top of the attention residual
    np.testing.assert_allclose(r["h"] - h1, mo.swiglu_mlp(m, layers[0]["w_gate"], layers[0]["w_up"],
                                                           layers[0]["w_down"]), rtol=1e-12, atol=1e-12)


def test_activation_rounding_points():
    a = np.array([1.0 + 2.0 ** -10, -3.3])
    np.testing.assert_array_equal(mo.act_round(a, None), a)
    np.testing.assert_array_equal(mo.act_round(a, "bf16"), oracle.bf16_round(a))
    with pytest.raises(ValueError):
        mo.act_round(a, "fp8")


def test_acceptance_threshold_branch():
    """Planted logits drive the confidence above and below the threshold."""
    rng = np.random.default_rng(3)
    layers, fn, wlm = _tiny_model(rng, 0)
    D, V = 32, 40
    x = np.zeros((2, D))
    x[:, 0] = 1.0
    fn = np.ones(D)
    wlm = np.zeros((V, D))
    wlm[5, 0] = 40.0  # rms_norm(x)[0] = sqrt(D) ~ 5.66: logit ~ 226 -> confidence 1
    r = mo.model_step_sequence(x, [], fn, wlm, np.array([0, 1]), [], [], np.array([0, 1]), 2, 16,
                               1e4, act_dtype=None, cache_dtype=None)
    assert list(r["token"]) == [5, 5] and r["accept"].all()
    r = mo.model_step_sequence(x, [], fn, np.zeros((V, D)), np.array([0, 1]), [], [],
                               np.array([0, 1]), 2, 16, 1e4, act_dtype=None, cache_dtype=None)
    assert not r["accept"].any()


def test_lm_head_reads_the_final_normed_stream():
    """With no layers the LM head sees rms_norm(x) * g_final: the planted
    logit is z * rms_norm(x)[0], close to z * sqrt(D) at any scale of x, and
    the confidence has the corresponding closed form."""
    D, V, z = 32, 40, 0.5
    wlm = np.zeros((V, D))
    wlm[5, 0] = z
    for s in (0.5, 3.0):
        x = np.zeros((1, D))
        x[0, 0] = s  # rms_norm(x)[0] = s / sqrt(s^2 / D + eps), about sqrt(D)
        t = z * s / math.sqrt(s * s / D + 1e-5)
        want = math.exp(t) / (math.exp(t) + V - 1)
        r = mo.model_step_sequence(x, [], np.ones(D), wlm, np.array([0]), [], [], np.array([0]),
                                   2, 16, 1e4, act_dtype=None, cache_dtype=None)
        assert r["token"][0] == 5
        np.testing.assert_allclose(r["confidence"][0], want, rtol=1e-12)
