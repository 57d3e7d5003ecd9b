"""The LM head and Flash-Verify confidence kernels alone (fc_model_lm_head) on
planted logits, against the fp64 oracle.

Random-weight models put every confidence near 1/vocab, so the model-step
tests never see the acceptance branch or large logits.  Here the LM-head rows
of chosen tokens are planted so that, per scored row, the top token's
probability lands at a chosen target: on both sides of the 0.9 threshold
(paper-digest page, Flash-Verify; threshold 0.9 in the configuration), at
probability one with a logit of 200 (far past exp's float range, so only a
max-subtracted sum of exponentials survives it), and as an exact tie of two
tokens in different 256-column tiles (lowest index wins)."""
import numpy as np
import pytest
import torch

from oracle import model_oracle as mo

pytestmark = pytest.mark.gpu

# kernel-only tolerance: both sides see the same bf16 rows and weights, so the
# confidence differs by fp32 accumulation and exp rounding only
CONF_RTOL = 1e-3
THRESHOLD = 0.9
TARGETS = (0.3, 0.6, 0.85, 0.87, 0.93, 0.95, 0.99, "big", "tie", None)


@pytest.fixture(scope="module", autouse=True)
def _need_gpu(cuda_ok):
    return cuda_ok


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy().astype(
        np.float64)


def planted_head(D, V, R, seed):
    """Final-normed rows [R, D] and an LM head [V, D] (both bf16-valued) whose
    planted tokens give row i the confidence TARGETS[i % len(TARGETS)]."""
    rng = np.random.default_rng(seed)
    rows = _bf16(rng.standard_normal((R, D)))  # unit RMS, as after the final norm
    w = rng.normal(0.0, 0.02, (V, D))
    perm = rng.permutation(V)
    plan, used, nxt = [], set(), 0

    def take(avoid_tile=None):
        nonlocal nxt
        while int(perm[nxt]) in used or (avoid_tile is not None and int(perm[nxt]) // 256 == avoid_tile):
            nxt += 1
        t = int(perm[nxt])
        used.add(t)
        return t

    for i in range(R):
        tgt = TARGETS[i % len(TARGETS)]
        if tgt == "tie":  # two tokens in different 256-column tiles
            a = take()
            b = take(avoid_tile=a // 256)
            plan.append((i, tgt, sorted((a, b))))
        elif tgt is not None:
            plan.append((i, tgt, [take()]))
    # column i of U is orthogonal to every row but row i: rows . U[:, i] = e_i,
    # so a planted LM-head row alpha * U[:, i] lifts row i's logit to alpha and
    # leaves every other row's logit of that token at 0
    U = np.linalg.pinv(rows)
    free = np.ones(V, bool)
    free[list(used)] = False
    Z = w[free] @ rows.T  # the unplanted logits, [V - planted, R]
    for i, tgt, toks in plan:
        s_other = np.exp(Z[:, i]).sum() + (len(used) - len(toks))  # planted: exp(0) each
        if tgt == "big":
            alpha = 200.0
        elif tgt == "tie":
            alpha = np.log(4.0 * s_other)  # each of the pair ~0.5 of the mass
        else:
            alpha = np.log(tgt / (1.0 - tgt) * s_other)
        for t in toks:
            w[t] = alpha * U[:, i]
    return rows, _bf16(w)


def zero_layer_model(D, V, lm_head, R, device):
    """A one-layer model whose decoder weights are zero: only the LM head of
    the model runs in these tests."""
    from kv_cache_attention_qkv_b200 import FlashCacheModel

    H, d, I = D // 128, 128, 128
    z = lambda *s: torch.zeros(s, dtype=torch.bfloat16, device=device)
    layer = {"attn_norm": z(D), "w_qkv": z(3 * H * d, D), "w_o": z(D, H * d), "mlp_norm": z(D),
             "w_gate": z(I, D), "w_up": z(I, D), "w_down": z(D, I)}
    return FlashCacheModel([layer], z(D), lm_head, hidden=D, n_heads=H, head_dim=d,
                           rope_theta=1e4, intermediate=I, max_batch=1, max_total_q=1,
                           max_total_k=1, max_seqlen_q=1, max_pos=1, max_topk=1,
                           max_head_rows=R, threshold=THRESHOLD)


def check(D, V, R, seed):
    rows, w = planted_head(D, V, R, seed)
    dev = torch.device("cuda", 0)
    lm = torch.from_numpy(w.astype(np.float32)).to(dev, dtype=torch.bfloat16)
    model = zero_layer_model(D, V, lm, R, dev)
    tok = torch.full((R,), -7, dtype=torch.int32, device=dev)
    conf = torch.full((R,), float("nan"), device=dev)
    acc = torch.full((R,), 7, dtype=torch.uint8, device=dev)
    model.lm_head(torch.from_numpy(rows.astype(np.float32)).to(dev, dtype=torch.bfloat16), tok, conf,
                  acc)
    torch.cuda.synchronize()
    assert model.get_error() == 0
    model.close()
    ref = mo.lm_head_confidence(rows, w)
    got_c, got_t, got_a = conf.cpu().numpy().astype(np.float64), tok.cpu().numpy(), acc.cpu().numpy()
    np.testing.assert_allclose(got_c, ref["confidence"], rtol=CONF_RTOL)
    # the planted targets are reached (so both acceptance outcomes are exercised)
    rc = ref["confidence"]
    assert (rc > THRESHOLD + 0.02).sum() >= 3 and ((rc < THRESHOLD - 0.02) & (rc > 0.5)).sum() >= 3
    assert (rc == 1.0).any()  # the logit-200 rows
    # tokens: the oracle's (lowest index among equal logits) wherever the best
    # two logits are not within fp32 rounding of each other
    lg = ref["logits"]
    for i in range(R):
        srt = np.sort(lg[i])[::-1]
        if srt[0] - srt[1] > 1e-4 * np.abs(lg[i]).max() or srt[0] == srt[1]:
            assert got_t[i] == ref["token"][i], (i, got_t[i], ref["token"][i])
    # acceptance: the oracle's decision away from the threshold
    clear = np.abs(rc - THRESHOLD) > CONF_RTOL * THRESHOLD
    np.testing.assert_array_equal(got_a[clear], (rc[clear] >= THRESHOLD).astype(np.uint8))
    assert set(np.unique(got_a).tolist()) <= {0, 1}


def test_lm_head_planted_small():
    """hidden 256, vocabulary 1000 (a ragged last 256-column tile), 40 rows."""
    check(256, 1000, 40, seed=11)


@pytest.mark.slow
def test_lm_head_planted_llada8b_shape():
    """hidden 4096, vocabulary 126464 (the LLaDA-8B LM head), 64 rows."""
    check(4096, 126464, 64, seed=12)
