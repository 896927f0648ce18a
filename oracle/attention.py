"""Decode / MTP-verify grouped-query attention over the paged FP8 cache, as
the plain definition in float64.  Test infrastructure only.

For sequence b with context length ``L = seq_lens[b]`` (the q_len new tokens
included, their K/V already appended), query row i (0 <= i < q_len) of
q-head hq attends KV head ``h = hq // G`` with ``G = Hq / Hkv`` (contiguous
groups -- the grouped-query sharing of the Atlas deep-dive, ainews.cool,
"Attention" paragraph):

    s_t   = sm_scale * sum_d q[b, i, hq, d] * K_b[t, h, d]   for t <= L - q_len + i
    p     = softmax(s)            (float64, max subtracted)
    out   = sum_t p_t * V_b[t, h, :]

with ``K_b``/``V_b`` the dequantised, contiguously re-assembled cache
(:mod:`oracle.paged`).  The causal limit ``t <= L - q_len + i`` is the MTP
verify mask: the new rows are the last q_len positions, and draft row i does
not see drafts after it (GB10 page, ainews.surl.tw: MTP with K = 4 drafts).
``sm_scale`` defaults to ``1 / sqrt(D)``.  Query values are the exact bf16
values, passed in as float64.  The result is float64 and is not rounded.
"""

import math

import numpy as np

from . import paged


def _softmax_rows(s):
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attend(q_rows, K, V, limits, sm_scale):
    """Masked attention for one KV head.

    ``q_rows`` float64 ``[R, D]``, ``K``/``V`` float64 ``[L, D]``, ``limits[r]``
    = last visible key position of row r.  Returns float64 ``[R, D]``.
    """
    s = sm_scale * (q_rows @ K.T)                            # [R, L]
    t = np.arange(K.shape[0])[None, :]
    s = np.where(t <= np.asarray(limits)[:, None], s, -np.inf)
    return _softmax_rows(s) @ V


def paged_gqa_decode(q, k_pages, v_pages, k_scale, v_scale, block_table,
                     seq_lens, q_len, page_size, sm_scale=None, sequences=None,
                     k_layout="tok", v_layout="tok"):
    """float64 ``[B, q_len, Hq, D]`` reference output.

    ``q``: float64 ``[B, q_len, Hq, D]``; ``k_pages``/``v_pages``: uint8
    ``[P, Hkv, ps, D]``; scales float32 ``[Hkv]``; ``block_table`` int
    ``[B, max_blocks]``; ``seq_lens`` int ``[B]``.  ``sequences`` restricts the
    work to a subset of b (other rows are left NaN), for sampled checks.
    ``k_layout`` / ``v_layout`` name the in-page order of each page array
    (:mod:`oracle.paged`): ``"tok"`` ``[P, Hkv, ps, D]``, ``"grp16"``
    ``[P, Hkv, ps/16, D, 16]`` or ``"dim"`` ``[P, Hkv, D, ps]``.
    """
    q = np.asarray(q, dtype=np.float64)
    B, ql, Hq, D = q.shape
    assert ql == q_len
    Hkv = np.asarray(k_pages).shape[1]
    assert Hq % Hkv == 0, "Hq must be a multiple of Hkv"
    G = Hq // Hkv
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / math.sqrt(D)
    out = np.full((B, q_len, Hq, D), np.nan)
    for b in (range(B) if sequences is None else sequences):
        L = int(seq_lens[b])
        if L < q_len:
            raise ValueError(f"sequence {b}: seq_len {L} < q_len {q_len}")
        K = paged.gather_dequant(k_pages, k_scale, block_table, b, L, page_size, k_layout)
        V = paged.gather_dequant(v_pages, v_scale, block_table, b, L, page_size, v_layout)
        limits = [L - q_len + i for i in range(q_len)]
        for h in range(Hkv):
            for g in range(G):
                hq = h * G + g
                out[b, :, hq, :] = attend(q[b, :, hq, :], K[:, h, :], V[:, h, :],
                                          limits, sm_scale)
    return out


def paged_gqa_decode_varlen(q, cu_q_lens, k_pages, v_pages, k_scale, v_scale, block_table,
                            seq_lens, page_size, sm_scale=None, sequences=None,
                            k_layout="tok", v_layout="tok"):
    """Ragged verify / chunked prefill: sequence b has its own number of new
    rows ``q_len_b = cu_q_lens[b + 1] - cu_q_lens[b]`` (packed: rows
    ``cu_q_lens[b] .. cu_q_lens[b + 1] - 1`` of ``q``), and new row i of it
    sees key positions ``t <= L_b - q_len_b + i`` (the GB10 page's MTP under
    concurrency: sequences verify different numbers of drafts; a prefill
    chunk is the same with many rows).  ``q`` float64 ``[total, Hq, D]``;
    returns float64 ``[total, Hq, D]`` (rows of skipped sequences NaN)."""
    q = np.asarray(q, dtype=np.float64)
    cu = np.asarray(cu_q_lens, dtype=np.int64)
    total, Hq, D = q.shape
    assert cu[0] == 0 and cu[-1] == total and np.all(np.diff(cu) >= 0)
    Hkv = np.asarray(k_pages).shape[1]
    assert Hq % Hkv == 0, "Hq must be a multiple of Hkv"
    G = Hq // Hkv
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / math.sqrt(D)
    out = np.full((total, Hq, D), np.nan)
    B = len(cu) - 1
    for b in (range(B) if sequences is None else sequences):
        L = int(seq_lens[b])
        ql = int(cu[b + 1] - cu[b])
        if ql == 0:
            continue
        if L < ql:
            raise ValueError(f"sequence {b}: seq_len {L} < q_len {ql}")
        K = paged.gather_dequant(k_pages, k_scale, block_table, b, L, page_size, k_layout)
        V = paged.gather_dequant(v_pages, v_scale, block_table, b, L, page_size, v_layout)
        limits = [L - ql + i for i in range(ql)]
        rows = slice(cu[b], cu[b + 1])
        for h in range(Hkv):
            for g in range(G):
                hq = h * G + g
                out[rows, hq, :] = attend(q[rows, hq, :], K[:, h, :], V[:, h, :], limits,
                                          sm_scale)
    return out


def paged_gqa_decode_tokscale(q, k_pages, v_pages, k_tok_scale, v_tok_scale, block_table,
                              seq_lens, q_len, page_size, sm_scale=None, sequences=None,
                              k_layout="tok", v_layout="tok"):
    """The same attention over a cache quantised with one dynamic scale per
    (token, KV head) (``paged.append_tokscale``): K and V are dequantised with
    the per-token scales ``[P, Hkv, ps]``, everything else as
    :func:`paged_gqa_decode`."""
    q = np.asarray(q, dtype=np.float64)
    B, ql, Hq, D = q.shape
    assert ql == q_len
    Hkv = np.asarray(k_pages).shape[1]
    G = Hq // Hkv
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / math.sqrt(D)
    out = np.full((B, q_len, Hq, D), np.nan)
    for b in (range(B) if sequences is None else sequences):
        L = int(seq_lens[b])
        if L < q_len:
            raise ValueError(f"sequence {b}: seq_len {L} < q_len {q_len}")
        K = paged.gather_dequant_tokscale(k_pages, k_tok_scale, block_table, b, L, page_size,
                                          k_layout)
        V = paged.gather_dequant_tokscale(v_pages, v_tok_scale, block_table, b, L, page_size,
                                          v_layout)
        limits = [L - q_len + i for i in range(q_len)]
        for h in range(Hkv):
            for g in range(G):
                hq = h * G + g
                out[b, :, hq, :] = attend(q[b, :, hq, :], K[:, h, :], V[:, h, :], limits,
                                          sm_scale)
    return out
