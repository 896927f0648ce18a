"""Pins for the oracle's paged-cache indexing (append scatter, gather)."""

import numpy as np

from oracle import e4m3, paged


def _pattern_pages(P, Hkv, ps, D):
    # every byte names its own coordinates, so a wrong index is visible
    p, h, s, d = np.meshgrid(np.arange(P), np.arange(Hkv), np.arange(ps), np.arange(D),
                             indexing="ij")
    return ((p * 7 + h * 31 + s * 5 + d * 3) % 251).astype(np.uint8)


def test_gather_codes_follows_block_table_slot_by_slot():
    P, Hkv, ps, D = 9, 3, 4, 5
    pages = _pattern_pages(P, Hkv, ps, D)
    table = np.array([[7, 2, 5, -1], [0, 8, -1, -1]], dtype=np.int32)
    for b, L in [(0, 11), (1, 5), (0, 1), (1, 8)]:
        got = paged.gather_codes(pages, table, b, L, ps)
        assert got.shape == (L, Hkv, D)
        for t in range(L):
            page = table[b][t // ps]
            for h in range(Hkv):
                assert np.array_equal(got[t, h], pages[page, h, t % ps])


def test_gather_dequant_applies_the_head_scale():
    P, Hkv, ps, D = 4, 2, 4, 3
    pages = np.full((P, Hkv, ps, D), 0x38, np.uint8)        # 1.0 everywhere
    table = np.array([[3, 1]], dtype=np.int32)
    scale = np.array([0.5, 3.0], np.float32)
    x = paged.gather_dequant(pages, scale, table, 0, 6, ps)
    assert np.array_equal(x[:, 0], np.full((6, D), 0.5))
    assert np.array_equal(x[:, 1], np.full((6, D), 3.0))


def test_append_writes_exactly_the_new_slots():
    rng = np.random.default_rng(5)
    P, Hkv, ps, D = 12, 2, 4, 8
    pages = rng.integers(0, 256, (P, Hkv, ps, D), dtype=np.uint8)
    table = np.array([[4, 9, 1, -1], [0, 11, 6, 3]], dtype=np.int32)
    start = np.array([3, 6], np.int32)
    n_new = 5
    new = rng.standard_normal((2, n_new, Hkv, D)).astype(np.float32)
    scale = np.array([0.02, 0.3], np.float32)
    out = paged.append(pages, new, scale, table, start, ps)
    touched = np.zeros(pages.shape, bool)
    for b in range(2):
        for t in range(n_new):
            pos = start[b] + t
            page, slot = table[b][pos // ps], pos % ps
            for h in range(Hkv):
                want = e4m3.encode(new[b, t, h], scale[h])
                assert np.array_equal(out[page, h, slot], want)
                touched[page, h, slot] = True
    assert np.array_equal(out[~touched], pages[~touched])
    assert np.array_equal(pages, np.asarray(pages))                  # input untouched


def test_append_in_two_calls_equals_one_call():
    rng = np.random.default_rng(6)
    P, Hkv, ps, D = 8, 1, 4, 4
    pages = np.zeros((P, Hkv, ps, D), np.uint8)
    table = np.array([[5, 2, 7]], dtype=np.int32)
    new = rng.standard_normal((1, 10, Hkv, D)).astype(np.float32)
    scale = np.array([0.01], np.float32)
    one = paged.append(pages, new, scale, table, np.array([0]), ps)
    two = paged.append(pages, new[:, :3], scale, table, np.array([0]), ps)
    two = paged.append(two, new[:, 3:], scale, table, np.array([3]), ps)
    assert np.array_equal(one, two)
    back = paged.gather_dequant(one, scale, table, 0, 10, ps)
    # the round trip is within half an E4M3 step (relative 1/16) of the input
    err = np.abs(back[:, 0] - new[0, :, 0])
    assert np.all(err <= np.abs(new[0, :, 0]) / 16 + 2.0 ** -10 * scale[0])


def test_dim_major_layout_is_the_per_page_transpose():
    rng = np.random.default_rng(21)
    P, Hkv, ps, D = 7, 2, 4, 6
    tok = rng.integers(0, 256, (P, Hkv, ps, D), dtype=np.uint8)
    dim = np.ascontiguousarray(tok.transpose(0, 1, 3, 2))        # [P, Hkv, D, ps]
    table = np.array([[3, 0, 6], [5, 1, -1]], dtype=np.int32)
    for b, L in [(0, 11), (1, 6), (0, 1)]:
        a = paged.gather_codes(tok, table, b, L, ps, "tok")
        g = paged.gather_codes(dim, table, b, L, ps, "dim")
        assert np.array_equal(a, g)
        for t in range(L):                                         # explicit indexing
            for h in range(Hkv):
                for d in range(D):
                    assert g[t, h, d] == dim[table[b][t // ps], h, d, t % ps]


def test_append_dim_major_writes_one_column_per_token():
    rng = np.random.default_rng(22)
    P, Hkv, ps, D = 5, 2, 4, 8
    pages = rng.integers(0, 256, (P, Hkv, D, ps), dtype=np.uint8)
    table = np.array([[2, 4, 0]], dtype=np.int32)
    new = rng.standard_normal((1, 6, Hkv, D)).astype(np.float32)
    scale = np.array([0.02, 0.05], np.float32)
    out = paged.append(pages, new, scale, table, np.array([3]), ps, layout="dim")
    touched = np.zeros(pages.shape, bool)
    for t in range(6):
        pos = 3 + t
        page, slot = table[0][pos // ps], pos % ps
        for h in range(Hkv):
            assert np.array_equal(out[page, h, :, slot], e4m3.encode(new[0, t, h], scale[h]))
            touched[page, h, :, slot] = True
    assert np.array_equal(out[~touched], pages[~touched])
    # same tokens through the token-major layout give the transposed pages
    tok = paged.append(np.ascontiguousarray(pages.transpose(0, 1, 3, 2)), new, scale, table,
                       np.array([3]), ps, layout="tok")
    assert np.array_equal(tok.transpose(0, 1, 3, 2), out)


def test_grp16_layout_groups_sixteen_slots_head_dim_major():
    rng = np.random.default_rng(23)
    P, Hkv, ps, D = 5, 2, 48, 8
    tok = rng.integers(0, 256, (P, Hkv, ps, D), dtype=np.uint8)
    # slot t of a group sits at this byte: bytes 4c..4c+3 hold slots 2c, 2c+1, 2c+8, 2c+9
    where = {0: 0, 1: 1, 8: 2, 9: 3, 2: 4, 3: 5, 10: 6, 11: 7, 4: 8, 5: 9, 12: 10, 13: 11,
             6: 12, 7: 13, 14: 14, 15: 15}
    assert [where[t] for t in range(16)] == list(paged.GROUP_POS)
    grp = np.empty((P, Hkv, ps // 16, D, 16), np.uint8)
    for s in range(ps):                                            # explicit construction
        grp[:, :, s // 16, :, where[s % 16]] = tok[:, :, s, :]
    table = np.array([[4, 1, 3], [0, 2, -1]], dtype=np.int32)
    for b, L in [(0, 130), (1, 49), (0, 16), (1, 1)]:
        assert np.array_equal(paged.gather_codes(tok, table, b, L, ps, "tok"),
                              paged.gather_codes(grp, table, b, L, ps, "grp16"))
    new = rng.standard_normal((1, 20, Hkv, D)).astype(np.float32)
    sc = np.array([0.03, 0.01], np.float32)
    a = paged.append(grp, new, sc, table, np.array([40]), ps, layout="grp16")
    t = paged.append(tok, new, sc, table, np.array([40]), ps, layout="tok")
    for s in range(ps):
        assert np.array_equal(a[:, :, s // 16, :, where[s % 16]], t[:, :, s, :])


def test_ksw_layout_permutes_sixteen_byte_chunks_by_slot():
    """Explicit construction: byte 16 * (j ^ (s % 8)) + k of slot s holds
    logical byte 16 * j + k (the 128-byte swizzle of a 128-byte row)."""
    rng = np.random.default_rng(29)
    P, Hkv, ps, D = 4, 2, 32, 128
    tok = rng.integers(0, 256, (P, Hkv, ps, D), dtype=np.uint8)
    sw = np.empty_like(tok)
    for s_ in range(ps):
        for j in range(8):
            dst = (j ^ (s_ % 8)) * 16
            sw[:, :, s_, dst:dst + 16] = tok[:, :, s_, 16 * j:16 * j + 16]
    # slot 0 is unpermuted; slot 3 moves chunk 0 to position 3 and chunk 3 to 0
    assert np.array_equal(sw[:, :, 0], tok[:, :, 0])
    assert np.array_equal(sw[:, :, 3, 48:64], tok[:, :, 3, 0:16])
    assert np.array_equal(sw[:, :, 3, 0:16], tok[:, :, 3, 48:64])
    table = np.array([[2, 0, 3], [1, -1, -1]], dtype=np.int32)
    for b, L in [(0, 70), (1, 32), (0, 1), (1, 17)]:
        assert np.array_equal(paged.gather_codes(tok, table, b, L, ps, "tok"),
                              paged.gather_codes(sw, table, b, L, ps, "ksw"))
    new = rng.standard_normal((1, 9, Hkv, D)).astype(np.float32)
    sc = np.array([0.02, 0.05], np.float32)
    a = paged.append(sw, new, sc, table, np.array([28]), ps, layout="ksw")
    t = paged.append(tok, new, sc, table, np.array([28]), ps, layout="tok")
    assert np.array_equal(paged.gather_codes(a, table, 0, 37, ps, "ksw"),
                          paged.gather_codes(t, table, 0, 37, ps, "tok"))
    assert paged.k_layout(128) == "ksw" and paged.k_layout(64) == "tok"
