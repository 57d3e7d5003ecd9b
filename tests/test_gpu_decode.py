"""GPU parity of the draft-and-verify decode iteration against the oracle,
iteration by iteration from the device's own state."""
import numpy as np
import pytest
import torch

import oracle
from oracle import decode_oracle as do
from kv_cache_attention_qkv_b200 import workloads
import fc_testlib as tl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu(cuda_ok):
    return cuda_ok


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


# relative tolerance of a confidence (see the model-step parity test)
CONF_TOL = 5e-2


def _tok_ok(tok, logits, vocab):
    """A device token agrees with the oracle unless its logit ties the top one."""
    spread = np.abs(logits).max()
    return 0 <= tok < vocab and logits[tok] >= logits.max() - 5e-3 * spread


@pytest.mark.parametrize("threshold,iters", [(0.9, 4), (0.0, 3)])
def test_decode_iterations_follow_the_oracle(threshold, iters):
    """threshold 0.9: random weights never reach it, so each iteration accepts
    the one most confident position; threshold 0: the whole window is accepted
    at once and the window advances every iteration."""
    from kv_cache_attention_qkv_b200 import FlashCacheModel

    mi = workloads.generate_model("model_small")
    dev = mi.embed.device
    B, K, W = mi.batch, 16, 16
    L = np.diff(mi.cu_seqlens_k)
    prompt = mi.window_start.astype(np.int64)  # the generated span starts at the window
    model = FlashCacheModel(mi.layers, mi.final_norm, mi.lm_head, hidden=mi.hidden,
                            n_heads=mi.n_heads, head_dim=mi.head_dim, rope_theta=mi.rope_theta,
                            intermediate=mi.intermediate, max_batch=B, max_total_q=B * (K + W),
                            max_total_k=mi.total_k, max_seqlen_q=K + W, max_pos=int(L.max()),
                            max_topk=K, max_head_rows=B * W, threshold=threshold)
    rng = np.random.default_rng(7)
    mask_id = mi.vocab - 1
    tokens = np.full(mi.total_k, -1, np.int32)
    tracked = np.zeros((B, K), np.int32)
    for b in range(B):
        k0 = mi.cu_seqlens_k[b]
        tokens[k0:k0 + prompt[b]] = rng.integers(0, mi.vocab - 1, size=prompt[b])
        tracked[b] = np.sort(rng.choice(prompt[b], size=K, replace=False))
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    st = {"tokens": i32(tokens), "draft": i32(np.full(mi.total_k, -1)), "tracked": i32(tracked),
          "ws": i32(prompt), "n_acc": i32(np.zeros(B))}
    gen_end, cu_k = i32(L), i32(mi.cu_seqlens_k)
    imp_t = torch.full((mi.total_k,), float("nan"), device=dev)
    layers64 = [{k: _f64(v) for k, v in lw.items()} for lw in mi.layers]
    fn64, lm64, emb64 = _f64(mi.final_norm), _f64(mi.lm_head), _f64(mi.embed)
    for it in range(iters):
        before = {k: v.cpu().numpy() for k, v in st.items()}
        caches = ([_f64(t) for t in mi.k_caches], [_f64(t) for t in mi.v_caches])
        model.decode_iteration(cu_k, mi.k_caches, mi.v_caches, mi.embed, mask_id, st["tracked"],
                               st["ws"], gen_end, st["tokens"], st["draft"], st["n_acc"], W,
                               importance=imp_t)
        torch.cuda.synchronize()
        assert model.get_error() == 0, it
        after = {k: v.cpu().numpy() for k, v in st.items()}
        imp_dev = imp_t.cpu().numpy().astype(np.float64)
        # the reselection, bit for bit: the oracle's top-k over [0, ws) (ws as
        # advanced) of the very importance the device ranked
        want_tr = oracle.topk_tracked(imp_dev, mi.cu_seqlens_k, np.zeros(B, np.int32), after["ws"],
                                      np.full(B, K, np.int32), K)
        np.testing.assert_array_equal(after["tracked"], want_tr, err_msg=f"iteration {it}")
        for b in range(B):
            ks = slice(int(mi.cu_seqlens_k[b]), int(mi.cu_seqlens_k[b + 1]))
            ws0 = int(before["ws"][b])
            ref = do.decode_iteration_sequence(
                layers64, fn64, lm64, emb64, before["tokens"][ks], before["draft"][ks],
                before["tracked"][b], ws0, int(L[b]), [c[ks] for c in caches[0]],
                [c[ks] for c in caches[1]], W, mask_id, threshold, mi.n_heads, mi.head_dim,
                mi.rope_theta)
            got_tok, got_dr = after["tokens"][ks], after["draft"][ks]
            win = np.arange(ws0, ws0 + W)
            lg_m, conf_m = ref["mask"]["logits"], ref["mask"]["confidence"]
            und = before["tokens"][ks][win] < 0
            new = np.nonzero(und & (got_tok[win] >= 0))[0]
            want = np.nonzero(und & (ref["tokens"][win] >= 0))[0]
            assert len(new) == after["n_acc"][b] == ref["n_accepted"], (it, b)
            if not und.any():
                assert len(new) == 0, (it, b)  # the sequence's last window is done
            elif (conf_m[und] >= threshold).any():
                # acceptance by threshold: the oracle's decision wherever the
                # confidence is not within the tolerance of the threshold
                clear = np.abs(conf_m - threshold) > CONF_TOL * threshold
                sel = und & clear
                assert np.array_equal(np.isin(np.nonzero(sel)[0], new), (conf_m >= threshold)[sel]), (it, b)
            else:
                # at least one: the oracle's choice (highest [MASK]-view confidence,
                # lowest position on ties) wherever the best two undecided
                # confidences are further apart than the tolerance; otherwise one
                # of the positions within the tolerance of the best
                assert len(new) == 1, (it, b)
                cu_ = np.sort(conf_m[und])[::-1]
                if len(cu_) == 1 or cu_[0] - cu_[1] > CONF_TOL * cu_[0]:
                    assert new.tolist() == want.tolist(), (it, b, new, want)
                else:
                    assert conf_m[new[0]] >= cu_[0] * (1 - CONF_TOL), (it, b)
            for j in new:
                assert _tok_ok(got_tok[win[j]], lg_m[j], mi.vocab), (it, b, j)
            # drafts of the still-undecided positions: the [MASK] view's predictions
            for j in np.nonzero(got_tok[win] < 0)[0]:
                assert _tok_ok(got_dr[win[j]], lg_m[j], mi.vocab), (it, b, j)
            assert after["ws"][b] == ref["ws"], (it, b)
            if threshold == 0.0 and ws0 + 2 * W <= L[b]:
                assert after["ws"][b] == ws0 + W, (it, b)  # the window advanced
            # the importance the reselection ranked (the draft view's, summed over
            # layers) against the oracle's, at the bf16 bar
            # (the tracked set itself was checked bit for bit above)
            tl.assert_close(imp_dev[ks], ref["importance"], 1e-2,
                            f"iteration {it} seq {b} importance")
            # the caches keep the draft view's rows
            for l in range(mi.n_layers):
                tl.assert_close(_f64(mi.k_caches[l][ks]), ref["k_caches"][l], 1e-2,
                                f"iteration {it} seq {b} k cache layer {l}")
    model.close()
