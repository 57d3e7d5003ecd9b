"""Pins of the decode-iteration oracle (query building, acceptance, drafts,
window advance) on hand-worked cases."""
import numpy as np

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
