"""Pins for the finer-grained FP8 scales (one dynamic scale per token and KV
head, computed at append): hand-worked codes, the row maximum landing on
+-448, exact power-of-two linearity, equivalence with the per-head path when
every row has the same maximum, and the attention against torch SDPA on the
dequantised cache (CPU only)."""

import math

import numpy as np
import torch

from oracle import attention, e4m3, paged


def test_hand_worked_row():
    # amax 2 -> scale = 2 / 448 (IEEE division in float32); the row divided by
    # it: 1 -> 224 (1.75 * 2^7, code 0x76), -2 -> -448 (0xFE), 0.5 -> 112 (0x6E)
    x = np.array([[1.0, -2.0, 0.5, 0.0]], np.float32)
    codes, s = e4m3.encode_rows(x)
    assert s[0] == np.float32(2.0) / np.float32(448.0)
    assert codes[0].tolist() == [0x76, 0xFE, 0x6E, 0x00]
    z, sz = e4m3.encode_rows(np.zeros((1, 4), np.float32))
    assert sz[0] == 1.0 and np.all(z == 0)


def test_row_maximum_codes_to_448():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((500, 8, 128)) * rng.uniform(1e-3, 1e3, (500, 8, 1))).astype(np.float32)
    codes, s = e4m3.encode_rows(x)
    mag = codes & 0x7F
    assert np.all(mag.max(axis=-1) == 0x7E)          # every row reaches +-448
    assert np.all(s == (np.abs(x).max(axis=-1) / np.float32(448)).astype(np.float32))


def test_power_of_two_linearity():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 4, 128)).astype(np.float32)
    c1, s1 = e4m3.encode_rows(x)
    for k in (-7, -1, 3, 11):
        ck, sk = e4m3.encode_rows(x * np.float32(2.0 ** k))
        assert np.array_equal(ck, c1)
        assert np.array_equal(sk, s1 * np.float32(2.0 ** k))


def test_equal_row_maxima_give_the_per_head_codes():
    rng = np.random.default_rng(3)
    x = rng.uniform(-1, 1, (40, 2, 64)).astype(np.float32)
    x[:, :, 5] = np.float32(3.0)                       # every row's maximum is 3
    codes, s = e4m3.encode_rows(x)
    head = np.full(2, np.float32(3.0) / np.float32(448.0), np.float32)
    assert np.all(s == head[0])
    assert np.array_equal(codes, e4m3.encode(x, head[None, :, None]))
    # and so does the paged append
    P, ps = 4, 16
    bt = np.array([[2, 0, 3]], np.int32)
    pa, sa = paged.append_tokscale(np.zeros((P, 2, ps, 64), np.uint8),
                                   np.zeros((P, 2, ps), np.float32), x[None], bt,
                                   np.array([3]), ps)
    pb = paged.append(np.zeros((P, 2, ps, 64), np.uint8), x[None], head, bt, np.array([3]), ps)
    assert np.array_equal(pa, pb)


def test_decode_matches_torch_sdpa_on_the_dequantised_cache():
    rng = np.random.default_rng(4)
    B, Hq, Hkv, D, ps, q_len = 2, 8, 2, 64, 16, 3
    lens = [37, 60]
    P = 8
    bt = np.array([[5, 1, 7, -1], [0, 2, 6, 3]], np.int32)
    kp = np.zeros((P, Hkv, ps, D), np.uint8)
    vp = np.zeros_like(kp)
    ks = np.zeros((P, Hkv, ps), np.float32)
    vs = np.zeros_like(ks)
    for b, L in enumerate(lens):
        k = (rng.standard_normal((1, L, Hkv, D)) * rng.uniform(0.1, 10, (1, L, Hkv, 1))).astype(np.float32)
        v = rng.standard_normal((1, L, Hkv, D)).astype(np.float32)
        kp, ks = paged.append_tokscale(kp, ks, k, bt[b:b + 1], np.array([0]), ps)
        vp, vs = paged.append_tokscale(vp, vs, v, bt[b:b + 1], np.array([0]), ps)
    q = torch.randn(B, q_len, Hq, D, generator=torch.Generator().manual_seed(4))
    q = q.to(torch.bfloat16).double().numpy()
    got = attention.paged_gqa_decode_tokscale(q, kp, vp, ks, vs, bt, np.array(lens), q_len, ps)
    for b, L in enumerate(lens):
        K = torch.empty(L, Hkv, D, dtype=torch.float64)
        V = torch.empty(L, Hkv, D, dtype=torch.float64)
        for t in range(L):
            page = int(bt[b, t // ps])
            K[t] = torch.from_numpy(kp[page, :, t % ps].copy()).view(torch.float8_e4m3fn).double() \
                * torch.from_numpy(ks[page, :, t % ps].astype(np.float64))[:, None]
            V[t] = torch.from_numpy(vp[page, :, t % ps].copy()).view(torch.float8_e4m3fn).double() \
                * torch.from_numpy(vs[page, :, t % ps].astype(np.float64))[:, None]
        G = Hq // Hkv
        Kq = K.permute(1, 0, 2).repeat_interleave(G, 0)
        Vq = V.permute(1, 0, 2).repeat_interleave(G, 0)
        i = torch.arange(q_len)[:, None]
        mask = torch.arange(L)[None, :] <= (L - q_len + i)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b]).permute(1, 0, 2), Kq, Vq, attn_mask=mask,
            scale=1.0 / math.sqrt(D)).permute(1, 0, 2).numpy()
        assert np.max(np.abs(got[b] - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))
