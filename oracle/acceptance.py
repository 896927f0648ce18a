"""Greedy acceptance of MTP draft tokens against the verify step's logits, as
the plain definition.  Test infrastructure only.

The verify step scores the q_len = K + 1 new positions of each sequence (the
last accepted token followed by K drafts; GB10 page, ainews.surl.tw: MTP with
K = 4).  Row i of the verify logits predicts the token that follows new
position i.  Greedy acceptance keeps the drafts while each equals the
target model's choice at its position and stops at the first mismatch; the
target's choice at that position is emitted in place of the rejected draft
(or after the last draft when all K are accepted).  The speculative-decoding
page (blog.hotdry.top, "Implementing kernel fusion in ATLAS speculative
decoding") describes the draft -> verify -> accept loop this closes.

Reading taken where the pages are silent: the target's choice is the
argmax of the row's logits, ties going to the lowest token id (the first
maximum); logits are finite.
"""

import numpy as np


def argmax_first(row) -> int:
    """Index of the first maximum of a 1-D array of finite values, by a plain
    scan (strictly greater replaces)."""
    best, idx = None, 0
    for j, v in enumerate(np.asarray(row, dtype=np.float64).tolist()):
        if best is None or v > best:
            best, idx = v, j
    return idx


def targets(logits) -> np.ndarray:
    """int32 ``[B, K + 1]``: the target model's choice at every new position
    (first maximum of each row; vectorised equivalent of :func:`argmax_first`
    -- numpy's argmax returns the first maximum)."""
    x = np.asarray(logits, dtype=np.float64)
    return np.argmax(x, axis=-1).astype(np.int32)


def greedy_accept(logits, drafts):
    """``logits`` ``[B, K + 1, V]`` (any float dtype, finite), ``drafts`` int
    ``[B, K]``.  Returns ``(n_accepted int32 [B], next_token int32 [B],
    targets int32 [B, K + 1])``: the number of leading drafts equal to the
    target at their position, and the target at the first position not
    covered by an accepted draft."""
    tg = targets(logits)
    d = np.asarray(drafts, dtype=np.int64)
    B, K = d.shape
    assert tg.shape == (B, K + 1)
    n_acc = np.zeros(B, np.int32)
    nxt = np.zeros(B, np.int32)
    for b in range(B):
        n = 0
        while n < K and d[b, n] == tg[b, n]:
            n += 1
        n_acc[b] = n
        nxt[b] = tg[b, n]
    return n_acc, nxt, tg
