"""Pins for the oracle's decode / verify attention (CPU only).

Checked against: torch's own scaled_dot_product_attention on float64 with
K/V dequantised through torch's float8_e4m3fn (an independent library path),
a pure-Python loop on a tiny case, closed forms (single token, two tokens,
identical keys, GQA head mapping, scale linearity) and invariants (page
permutation, MTP causal independence).
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention, paged


def _rand_case(rng, B, Hq, Hkv, D, ps, lens, q_len, P=None):
    need = [(L + ps - 1) // ps for L in lens]
    P = P or sum(need) + 3
    perm = rng.permutation(P)
    table = np.full((B, max(need)), -1, np.int32)
    at = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[at:at + n]
        at += n
    finite = np.concatenate([np.arange(0x7F), np.arange(0x80, 0xFF)]).astype(np.uint8)
    kp = rng.choice(finite, (P, Hkv, ps, D))
    vp = rng.choice(finite, (P, Hkv, ps, D))
    ks = rng.uniform(0.001, 0.02, Hkv).astype(np.float32)
    vs = rng.uniform(0.001, 0.02, Hkv).astype(np.float32)
    q = torch.randn(B, q_len, Hq, D, generator=torch.Generator().manual_seed(int(rng.integers(1 << 30))))
    q = q.to(torch.bfloat16).to(torch.float64).numpy()
    return dict(q=q, k_pages=kp, v_pages=vp, k_scale=ks, v_scale=vs, block_table=table,
                seq_lens=np.array(lens, np.int32), q_len=q_len, page_size=ps)


def _torch_reference(c, sm_scale):
    """SDPA on float64 with explicit gathers and torch's float8 decode."""
    q = torch.from_numpy(c["q"])
    B, ql, Hq, D = q.shape
    Hkv = c["k_pages"].shape[1]
    ps = c["page_size"]
    out = torch.empty(B, ql, Hq, D, dtype=torch.float64)
    for b in range(B):
        L = int(c["seq_lens"][b])
        K = torch.empty(L, Hkv, D, dtype=torch.float64)
        V = torch.empty(L, Hkv, D, dtype=torch.float64)
        for t in range(L):
            page = int(c["block_table"][b, t // ps])
            for name, dst, sc in (("k_pages", K, "k_scale"), ("v_pages", V, "v_scale")):
                raw = torch.from_numpy(c[name][page, :, t % ps, :].copy())
                val = raw.view(torch.float8_e4m3fn).to(torch.float64)
                dst[t] = val * torch.from_numpy(c[sc].astype(np.float64))[:, None]
        G = Hq // Hkv
        Kq = K.permute(1, 0, 2).repeat_interleave(G, dim=0)       # [Hq, L, D]
        Vq = V.permute(1, 0, 2).repeat_interleave(G, dim=0)
        qq = q[b].permute(1, 0, 2)                                 # [Hq, ql, D]
        i = torch.arange(ql)[:, None]
        t = torch.arange(L)[None, :]
        mask = t <= (L - ql + i)                                   # True = attend
        o = torch.nn.functional.scaled_dot_product_attention(
            qq, Kq, Vq, attn_mask=mask, scale=sm_scale)
        out[b] = o.permute(1, 0, 2)
    return out.numpy()


@pytest.mark.parametrize("Hq,Hkv,D,ps,lens,q_len", [
    (4, 2, 8, 4, [1, 7], 1),
    (4, 1, 8, 4, [9, 16, 17], 1),
    (6, 3, 64, 16, [40, 33], 3),
    (8, 2, 64, 16, [5, 31], 5),
    (2, 2, 16, 8, [12, 8], 4),
    (8, 8, 8, 4, [2], 2),
])
def test_matches_torch_sdpa(Hq, Hkv, D, ps, lens, q_len):
    rng = np.random.default_rng(hash((Hq, Hkv, D, ps, q_len)) & 0xFFFF)
    c = _rand_case(rng, len(lens), Hq, Hkv, D, ps, lens, q_len)
    for sm in (None, 0.37):
        got = attention.paged_gqa_decode(sm_scale=sm, **c)
        ref = _torch_reference(c, 1.0 / math.sqrt(D) if sm is None else sm)
        assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_pure_python_loop_tiny():
    rng = np.random.default_rng(3)
    c = _rand_case(rng, 1, 2, 1, 4, 2, [5], 2)
    got = attention.paged_gqa_decode(**c)
    from oracle import e4m3
    L, D = 5, 4
    for hq in range(2):
        for i in range(2):
            lim = L - 2 + i
            s = []
            for t in range(lim + 1):
                page, slot = c["block_table"][0][t // 2], t % 2
                acc = 0.0
                for d in range(D):
                    kv = float(e4m3.decode(c["k_pages"][page, 0, slot, d])) * float(c["k_scale"][0])
                    acc += c["q"][0, i, hq, d] * kv
                s.append(acc / math.sqrt(D))
            mx = max(s)
            w = [math.exp(x - mx) for x in s]
            tot = sum(w)
            for d in range(D):
                o = 0.0
                for t in range(lim + 1):
                    page, slot = c["block_table"][0][t // 2], t % 2
                    vv = float(e4m3.decode(c["v_pages"][page, 0, slot, d])) * float(c["v_scale"][0])
                    o += w[t] / tot * vv
                assert abs(o - got[0, i, hq, d]) < 1e-12


def test_single_token_context_returns_the_v_row():
    rng = np.random.default_rng(11)
    c = _rand_case(rng, 3, 8, 2, 16, 4, [1, 1, 1], 1)
    got = attention.paged_gqa_decode(**c)
    for b in range(3):
        V = paged.gather_dequant(c["v_pages"], c["v_scale"], c["block_table"], b, 1, 4)
        for hq in range(8):
            assert np.array_equal(got[b, 0, hq], V[0, hq // 4])


def test_two_tokens_closed_form():
    # q = e0, k0 = 0, k1 = e0 (code 0x38 = 1.0), sm_scale = 1 -> s = (0, 1)
    P, ps, D = 2, 4, 4
    kp = np.zeros((P, 1, ps, D), np.uint8)
    kp[1, 0, 1, 0] = 0x38
    vp = np.zeros((P, 1, ps, D), np.uint8)
    vp[1, 0, 0, :] = 0x40                        # v0 = 2
    vp[1, 0, 1, :] = 0xB8                        # v1 = -1
    q = np.zeros((1, 1, 1, D))
    q[0, 0, 0, 0] = 1.0
    out = attention.paged_gqa_decode(q, kp, vp, np.ones(1, np.float32), np.ones(1, np.float32),
                                     np.array([[1]]), np.array([2]), 1, ps, sm_scale=1.0)
    p1 = math.e / (1 + math.e)
    want = (1 - p1) * 2.0 + p1 * (-1.0)
    assert np.allclose(out[0, 0, 0], want, rtol=0, atol=1e-15)


def test_identical_keys_give_the_mean_of_v():
    rng = np.random.default_rng(12)
    c = _rand_case(rng, 2, 4, 2, 8, 4, [13, 6], 1)
    c["k_pages"][:] = c["k_pages"][0, 0, 0][None, None, None, :]
    got = attention.paged_gqa_decode(**c)
    for b, L in enumerate(c["seq_lens"]):
        V = paged.gather_dequant(c["v_pages"], c["v_scale"], c["block_table"], b, int(L), 4)
        for hq in range(4):
            assert np.allclose(got[b, 0, hq], V[:, hq // 2].mean(axis=0), rtol=0, atol=1e-12)


def test_gqa_head_mapping_is_contiguous_groups():
    # KV head h holds the constant value h + 1: q-head hq must read hq // G + 1
    Hkv, G, ps, D = 4, 3, 4, 8
    kp = np.zeros((2, Hkv, ps, D), np.uint8)
    vp = np.zeros((2, Hkv, ps, D), np.uint8)
    codes = {1: 0x38, 2: 0x40, 3: 0x44, 4: 0x48}    # 1, 2, 3, 4
    for h in range(Hkv):
        vp[:, h] = codes[h + 1]
    q = np.ones((1, 1, Hkv * G, D))
    out = attention.paged_gqa_decode(q, kp, vp, np.ones(Hkv, np.float32),
                                     np.ones(Hkv, np.float32), np.array([[1, 0]]),
                                     np.array([6]), 1, ps)
    for hq in range(Hkv * G):
        assert np.all(out[0, 0, hq] == hq // G + 1)


def test_scales_enter_linearly():
    rng = np.random.default_rng(13)
    c = _rand_case(rng, 2, 4, 2, 16, 4, [9, 14], 2)
    base = attention.paged_gqa_decode(**c)
    c2 = dict(c, v_scale=c["v_scale"] * np.float32(2.0))
    assert np.array_equal(attention.paged_gqa_decode(**c2), 2.0 * base)
    c3 = dict(c, k_scale=c["k_scale"] * np.float32(4.0))
    sm = 1.0 / math.sqrt(16)
    assert np.allclose(attention.paged_gqa_decode(**c3),
                       attention.paged_gqa_decode(sm_scale=4.0 * sm, **c), rtol=0, atol=1e-12)


def test_page_permutation_invariance():
    rng = np.random.default_rng(14)
    c = _rand_case(rng, 3, 6, 2, 16, 4, [10, 4, 15], 1, P=20)
    base = attention.paged_gqa_decode(**c)
    perm = rng.permutation(20)                      # new id of old page p is perm[p]
    kp = np.empty_like(c["k_pages"])
    vp = np.empty_like(c["v_pages"])
    kp[perm] = c["k_pages"]
    vp[perm] = c["v_pages"]
    table = np.where(c["block_table"] >= 0, perm[np.maximum(c["block_table"], 0)], -1)
    got = attention.paged_gqa_decode(**dict(c, k_pages=kp, v_pages=vp, block_table=table))
    assert np.array_equal(got, base)


def test_mtp_causal_rows_ignore_later_drafts():
    rng = np.random.default_rng(15)
    q_len, L, ps = 5, 23, 4
    c = _rand_case(rng, 1, 4, 2, 16, ps, [L], q_len)
    base = attention.paged_gqa_decode(**c)
    for i in range(q_len):
        c2 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in c.items()}
        for t in range(L - q_len + i + 1, L):          # drafts after row i
            page, slot = c["block_table"][0][t // ps], t % ps
            c2["k_pages"][page, :, slot, :] ^= 0x15
            c2["v_pages"][page, :, slot, :] ^= 0x22
        c2["k_pages"][c2["k_pages"] & 0x7F == 0x7F] = 0x11      # keep codes finite
        c2["v_pages"][c2["v_pages"] & 0x7F == 0x7F] = 0x11
        got = attention.paged_gqa_decode(**c2)
        assert np.array_equal(got[0, : i + 1], base[0, : i + 1])
        if i < q_len - 1:
            assert not np.array_equal(got[0, i + 1:], base[0, i + 1:])


def test_seq_len_below_q_len_is_rejected():
    rng = np.random.default_rng(16)
    c = _rand_case(rng, 1, 2, 1, 8, 4, [3], 3)
    c["seq_lens"] = np.array([2], np.int32)
    with pytest.raises(ValueError):
        attention.paged_gqa_decode(**c)


def test_v_layout_dim_matches_token_major():
    rng = np.random.default_rng(17)
    c = _rand_case(rng, 2, 8, 2, 16, 4, [9, 14], 3)
    base = attention.paged_gqa_decode(**c)
    c2 = dict(c, v_pages=np.ascontiguousarray(c["v_pages"].transpose(0, 1, 3, 2)))
    assert np.array_equal(attention.paged_gqa_decode(v_layout="dim", **c2), base)
    c3 = dict(c, k_pages=np.ascontiguousarray(c["k_pages"].transpose(0, 1, 3, 2)))
    assert np.array_equal(attention.paged_gqa_decode(k_layout="dim", **c3), base)
    # ps = 4 has no full 16-slot group: use a 16-slot page for grp16
    c4 = _rand_case(rng, 2, 8, 2, 16, 16, [9, 30], 2)
    base4 = attention.paged_gqa_decode(**c4)
    v = c4["v_pages"]                                              # [P, Hkv, 16, D]
    g = np.empty((v.shape[0], v.shape[1], 1, v.shape[3], 16), np.uint8)
    for t in range(16):
        g[:, :, 0, :, paged.GROUP_POS[t]] = v[:, :, t, :]
    assert np.array_equal(attention.paged_gqa_decode(v_layout="grp16", **dict(c4, v_pages=g)), base4)


def _varlen_case(rng, Hq, Hkv, D, ps, lens, qlens):
    c = _rand_case(rng, len(lens), Hq, Hkv, D, ps, lens, 1)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = torch.randn(int(cu[-1]), Hq, D, generator=torch.Generator().manual_seed(int(rng.integers(1 << 30))))
    q = q.to(torch.bfloat16).to(torch.float64).numpy()
    del c["q"], c["q_len"]
    return dict(c, q=q, cu_q_lens=cu)


@pytest.mark.parametrize("Hq,Hkv,D,ps,lens,qlens", [
    (4, 2, 8, 4, [7, 9, 3], [1, 5, 3]),
    (8, 2, 64, 16, [40, 33, 64], [2, 1, 17]),      # a 17-row prefill chunk
    (6, 3, 16, 8, [12, 8, 20, 5], [4, 0, 2, 5]),   # a sequence with no new rows
])
def test_varlen_matches_torch_sdpa_per_sequence(Hq, Hkv, D, ps, lens, qlens):
    """Each sequence's rows against torch SDPA (float64, GQA by
    repeat_interleave, boolean causal mask with that sequence's q_len)."""
    rng = np.random.default_rng(sum(lens))
    c = _varlen_case(rng, Hq, Hkv, D, ps, lens, qlens)
    got = attention.paged_gqa_decode_varlen(**c)
    cu = c["cu_q_lens"]
    for b, L in enumerate(lens):
        ql = qlens[b]
        if ql == 0:
            continue
        one = dict(q=c["q"][cu[b]:cu[b + 1]][None], k_pages=c["k_pages"], v_pages=c["v_pages"],
                   k_scale=c["k_scale"], v_scale=c["v_scale"], block_table=c["block_table"][b:b + 1],
                   seq_lens=np.array([L], np.int32), q_len=ql, page_size=ps)
        ref = _torch_reference(one, 1.0 / math.sqrt(D))[0]
        assert np.max(np.abs(got[cu[b]:cu[b + 1]] - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_varlen_with_equal_lengths_is_the_uniform_path():
    rng = np.random.default_rng(8)
    c = _rand_case(rng, 3, 8, 2, 16, 4, [9, 12, 30], 3)
    uni = attention.paged_gqa_decode(**c)
    cu = np.arange(4, dtype=np.int32) * 3
    var = attention.paged_gqa_decode_varlen(c["q"].reshape(9, 8, 16), cu, c["k_pages"],
                                            c["v_pages"], c["k_scale"], c["v_scale"],
                                            c["block_table"], c["seq_lens"], 4)
    assert np.array_equal(var.reshape(3, 3, 8, 16), uni)


def test_varlen_rows_ignore_later_drafts_and_empty_sequences_stay_nan():
    rng = np.random.default_rng(9)
    c = _varlen_case(rng, 4, 1, 8, 4, [10, 6], [4, 0])
    base = attention.paged_gqa_decode_varlen(**c)
    assert np.all(np.isnan(base[4:]))               # no rows of sequence 1 (empty)
    L, ql = 10, 4
    for i in range(ql - 1):
        kp = c["k_pages"].copy()
        for t in range(L - ql + i + 1, L):
            page, slot = c["block_table"][0][t // 4], t % 4
            kp[page, 0, slot, :] = 0x3C
        got = attention.paged_gqa_decode_varlen(**dict(c, k_pages=kp))
        assert np.array_equal(got[:i + 1], base[:i + 1])
        assert not np.array_equal(got[i + 1:4], base[i + 1:4])
