"""Helpers shared by the GPU parity tests: the oracle side of each check
(computed only from the seeded generator's inputs, never from GPU output)
and the tolerance rule."""

import numpy as np

from oracle import attention, e4m3, paged

# Tolerance of the decode / verify output against the float64 oracle (bf16
# out, f32 softmax): relative L2 <= 5e-3 over the compared rows, and per
# element |got - ref| <= max(1e-2, 2^-8 |ref|).  The 1e-2 absolute bound is
# the stated one for unit-scale outputs; bf16 keeps 8 significant bits, so
# the correctly rounded output of a value of magnitude >= 4 (half an ulp is
# then 2^-6 or more) can already be more than 1e-2 away.  2^-8 |ref| bounds
# that rounding (at most 2^-9 |ref|) with room for the f32 arithmetic; it
# only exceeds 1e-2 where |ref| > 2.56, so unit-scale outputs keep the plain
# 1e-2 bound.
MAX_ABS = 1e-2
REL_ELEM = 2.0 ** -8
REL_L2 = 5e-3


def oracle_pages(w, which):
    """Token-major uint8 pages ``[P, Hkv, ps, D]`` the oracle expects after
    every token of every sequence of workload ``w`` is appended, and the mask
    of written (page, head, slot) triples.  (The GPU keeps V in 16-slot
    groups and, with D = 128, K rows chunk-permuted; tests bring them to
    token-major with :func:`v_token_major` and :func:`k_token_major`.)"""
    P, Hkv, ps, D = w.num_pages, w.num_kv_heads, w.page_size, w.head_dim
    pages = np.zeros((P, Hkv, ps, D), np.uint8)
    written = np.zeros((P, Hkv, ps), bool)
    scale = w.k_scale if which == "k" else w.v_scale
    src = w.k if which == "k" else w.v
    for b in range(w.batch):
        L = int(w.seq_lens[b])
        codes = e4m3.encode(src[w.cu_seqlens[b]:w.cu_seqlens[b + 1]], scale[None, :, None])
        t = np.arange(L)
        pg = w.block_table[b, t // ps]
        pages[pg, :, t % ps, :] = codes
        written[pg, :, t % ps] = True
    return pages, written


def k_token_major(k):
    """GPU K pages ``[P, Hkv, ps, D]`` (chunk-permuted rows when D = 128) ->
    plain token-major ``[P, Hkv, ps, D]``."""
    k = np.asarray(k)
    P, H, ps, D = k.shape
    if paged.k_layout(D) == "tok":
        return k
    out = np.empty_like(k)
    for s in range(ps):
        for j in range(D // 16):
            c = paged.ksw_chunk(s, j)
            out[:, :, s, 16 * j:16 * j + 16] = k[:, :, s, 16 * c:16 * c + 16]
    return out


def v_token_major(v):
    """``[P, Hkv, ps/16, D, 16]`` (16-slot groups, interleaved) -> ``[P, Hkv, ps, D]``."""
    v = np.asarray(v)[..., paged.GROUP_POS]
    P, H, G, D, _ = v.shape
    return v.transpose(0, 1, 2, 4, 3).reshape(P, H, G * 16, D)


def oracle_decode(w, sequences=None, sm_scale=None):
    kp, _ = oracle_pages_subset(w, "k", sequences)
    vp, _ = oracle_pages_subset(w, "v", sequences)
    return attention.paged_gqa_decode(w.q_f64(), kp, vp, w.k_scale, w.v_scale, w.block_table,
                                      w.seq_lens, w.q_len, w.page_size, sm_scale=sm_scale,
                                      sequences=sequences)


def oracle_pages_subset(w, which, sequences):
    """Like :func:`oracle_pages` but only for the listed sequences."""
    if sequences is None:
        return oracle_pages(w, which)
    P, Hkv, ps, D = w.num_pages, w.num_kv_heads, w.page_size, w.head_dim
    pages = np.zeros((P, Hkv, ps, D), np.uint8)
    scale = w.k_scale if which == "k" else w.v_scale
    src = w.k if which == "k" else w.v
    for b in sequences:
        L = int(w.seq_lens[b])
        codes = e4m3.encode(src[w.cu_seqlens[b]:w.cu_seqlens[b + 1]], scale[None, :, None])
        t = np.arange(L)
        pages[w.block_table[b, t // ps], :, t % ps, :] = codes
    return pages, None


def errors(got, ref):
    """(max-abs, rel-L2) of ``got`` against ``ref`` over the finite rows of ref."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    sel = np.isfinite(ref)
    d = got[sel] - ref[sel]
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    den = float(np.linalg.norm(ref[sel]))
    rel = float(np.linalg.norm(d) / den) if den > 0 else float(np.linalg.norm(d))
    return max_abs, rel


# (case, max-abs, rel-L2) of every parity check of the run, printed at the end
# of the session by tests/conftest.py
PARITY_LOG = []


def record_parity(case, max_abs, rel):
    PARITY_LOG.append((case, float(max_abs), float(rel)))


def elementwise_excess(got, ref):
    """Largest ratio |got - ref| / max(MAX_ABS, REL_ELEM |ref|) over the finite
    rows of ref (<= 1 passes)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    sel = np.isfinite(ref)
    if not sel.any():
        return 0.0
    d = np.abs(got[sel] - ref[sel])
    allowed = np.maximum(MAX_ABS, REL_ELEM * np.abs(ref[sel]))
    return float(np.max(d / allowed))


def assert_close(got, ref, what=""):
    max_abs, rel = errors(got, ref)
    assert np.all(np.isfinite(np.asarray(got, np.float64)[np.isfinite(ref)])), f"{what}: non-finite output"
    excess = elementwise_excess(got, ref)
    assert excess <= 1.0 and rel <= REL_L2, (
        f"{what}: max-abs {max_abs:.3g} ({excess:.3g} of the per-element bound), rel-L2 {rel:.3g}")
    return max_abs, rel


__all__ = ["oracle_pages", "oracle_decode", "k_token_major", "v_token_major", "errors",
           "assert_close", "elementwise_excess", "record_parity", "PARITY_LOG", "MAX_ABS",
           "REL_ELEM", "REL_L2", "paged"]
