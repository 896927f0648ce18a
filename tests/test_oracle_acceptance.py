"""Pins for the oracle's greedy MTP acceptance (CPU only): hand-worked
cases, the first-maximum tie rule, brute force against an independent
formulation, and invariances."""

import numpy as np

from oracle import acceptance


def test_argmax_first_takes_the_first_maximum():
    assert acceptance.argmax_first([1.0, 3.0, 3.0, 2.0]) == 1
    assert acceptance.argmax_first([5.0, 5.0, 5.0]) == 0
    assert acceptance.argmax_first([-4.0, -1.5, -1.5, -9.0]) == 1
    assert acceptance.argmax_first([0.0]) == 0
    assert acceptance.argmax_first([-0.0, 0.0, 1e-30]) == 2


def test_targets_match_the_scan_on_rows_with_ties():
    rng = np.random.default_rng(3)
    x = rng.integers(-3, 4, size=(4, 5, 9)).astype(np.float32)   # many ties
    tg = acceptance.targets(x)
    for b in range(4):
        for i in range(5):
            assert tg[b, i] == acceptance.argmax_first(x[b, i])


def test_hand_worked_batch():
    # V = 6, K = 4.  Row targets are planted by a single large logit.
    B, K, V = 3, 4, 6
    logits = np.zeros((B, K + 1, V), np.float32)
    want_t = np.array([[2, 5, 1, 1, 0],
                       [4, 4, 3, 0, 2],
                       [0, 1, 2, 3, 4]])
    for b in range(B):
        for i in range(K + 1):
            logits[b, i, want_t[b, i]] = 7.0
    drafts = np.array([[3, 5, 1, 1],     # first draft rejected: n = 0, emit 2
                       [4, 4, 1, 0],     # two accepted: n = 2, emit 3
                       [0, 1, 2, 3]])    # all accepted: n = 4, emit the bonus 4
    n, nxt, tg = acceptance.greedy_accept(logits, drafts)
    assert np.array_equal(tg, want_t)
    assert n.tolist() == [0, 2, 4]
    assert nxt.tolist() == [2, 3, 4]


def test_brute_force_against_first_mismatch():
    rng = np.random.default_rng(11)
    for _ in range(200):
        B, K, V = int(rng.integers(1, 5)), int(rng.integers(1, 6)), int(rng.integers(1, 7))
        logits = rng.integers(-2, 3, size=(B, K + 1, V)).astype(np.float64)
        tg = np.array([[acceptance.argmax_first(logits[b, i]) for i in range(K + 1)]
                       for b in range(B)])
        # drafts agree with the targets on a random prefix, then maybe differ
        drafts = tg[:, :K].copy()
        for b in range(B):
            cut = int(rng.integers(0, K + 1))
            if cut < K:
                drafts[b, cut] = (drafts[b, cut] + 1 + int(rng.integers(0, max(V - 1, 1)))) % max(V, 2)
        n, nxt, _ = acceptance.greedy_accept(logits, drafts)
        for b in range(B):
            mism = np.nonzero(drafts[b] != tg[b, :K])[0]
            want = int(mism[0]) if mism.size else K
            assert n[b] == want
            assert nxt[b] == tg[b, want]


def test_row_shift_and_draft_independence_of_targets():
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((2, 5, 50)).astype(np.float32)
    shifted = logits + np.float32(3.0)
    assert np.array_equal(acceptance.targets(logits), acceptance.targets(shifted))
    d1 = rng.integers(0, 50, (2, 4))
    d2 = rng.integers(0, 50, (2, 4))
    assert np.array_equal(acceptance.greedy_accept(logits, d1)[2],
                          acceptance.greedy_accept(logits, d2)[2])
