"""GPU: the fused rotary embedding + FP8 append is bit-exact with the oracle
(rotated bf16 queries, K and V pages), and decode over the cache it fills
matches the oracle's attention with the rotated queries."""

import numpy as np
import pytest
import torch

from oracle import attention, rope
from paged_fp8_kv_05_b200 import build, workloads

from parity import assert_close, k_token_major, record_parity, v_token_major

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ak():
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv
    return atlas_kv


CASES = [
    # (B, n_new, Hq, Hkv, D, ps, start positions)
    (32, 1, 32, 8, 128, 16, "ragged"),     # LLaMA-3-8B-shaped decode step
    (3, 37, 8, 2, 64, 16, "ragged"),       # cache fill, page crossings, D = 64
    (4, 5, 40, 8, 128, 64, "ragged"),      # MTP verify step (K = 4 drafts + 1), page 64
    (2, 300, 8, 1, 128, 16, "zero"),       # long fill from position 0
]


@pytest.mark.parametrize("case", CASES)
def test_rope_append_bit_exact_and_decode(ak, case):
    B, n_new, Hq, Hkv, D, ps, starts = case
    rng = np.random.default_rng(B * 7 + n_new)
    start = (rng.integers(0, 3000, B) if starts == "ragged" else np.zeros(B, np.int64)).astype(np.int32)
    L = start + n_new
    max_pos = int(L.max()) + 1
    qkv, cos_sin = workloads.make_rope_inputs(batch=B, n_new=n_new, num_q_heads=Hq,
                                              num_kv_heads=Hkv, head_dim=D, max_pos=max_pos,
                                              seed=B + n_new)
    need = [int((l + ps - 1) // ps) for l in L]
    P = sum(need) + 3
    perm = rng.permutation(P)
    table = np.full((B, max(need)), -1, np.int32)
    at = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[at:at + n]
        at += n
    ks = rng.uniform(0.005, 0.02, Hkv).astype(np.float32)
    vs = rng.uniform(0.005, 0.02, Hkv).astype(np.float32)
    pool = ak.KVPool(P, ps, Hkv, D, ks, vs, max_batch=B, max_q_len=n_new, num_q_heads=Hq,
                     max_seq_len=int(L.max()), fill=0x7F)
    d_qkv = qkv.cuda().contiguous()
    d_cs = torch.from_numpy(cos_sin).cuda().contiguous()
    d_bt = torch.from_numpy(table).cuda()
    d_st = torch.from_numpy(start).cuda()
    q_out = ak.atlas_rope_fp8_kv_append(pool, d_qkv, Hq, d_cs, d_bt, d_st)
    torch.cuda.synchronize()
    assert pool.device_error() == 0

    init = np.full((P, Hkv, ps, D), 0x7F, np.uint8)
    q_ref, kp_ref, vp_ref = rope.rope_append(init, init, qkv.float().numpy(), Hq, Hkv, cos_sin,
                                             ks, vs, table, start, ps)
    assert np.array_equal(q_out.float().cpu().numpy().view(np.uint32), q_ref.view(np.uint32))
    assert np.array_equal(k_token_major(pool.k_pages.cpu().numpy()), kp_ref)
    assert np.array_equal(v_token_major(pool.v_pages.cpu().numpy()), vp_ref)

    # decode / verify over the rotated cache: the new rows attend to the cache
    # up to their own position (only the appended tokens are in it when
    # start == 0; otherwise the earlier slots hold NaN codes, never read
    # because their positions are below start -- so attend the new tokens only)
    if starts == "zero":
        sl = torch.from_numpy(L.astype(np.int32)).cuda()
        q_dec = q_out.contiguous()
        out = ak.atlas_paged_gqa_decode(pool, q_dec, d_bt, sl, int(L.max()))
        ref = attention.paged_gqa_decode(q_ref.astype(np.float64), kp_ref, vp_ref, ks, vs, table,
                                         L, n_new, ps)
        max_abs, rel = assert_close(out.float().cpu().numpy(), ref, f"decode after rope {case}")
        record_parity(f"decode over the rotated cache {case[:6]}", max_abs, rel)


def test_rope_append_flags_positions_outside_the_table(ak):
    B, n_new, Hq, Hkv, D, ps = 2, 3, 4, 2, 128, 16
    qkv, cos_sin = workloads.make_rope_inputs(batch=B, n_new=n_new, num_q_heads=Hq,
                                              num_kv_heads=Hkv, head_dim=D, max_pos=10, seed=1)
    pool = ak.KVPool(8, ps, Hkv, D, [0.01, 0.01], [0.01, 0.01], max_batch=B, max_q_len=1,
                     num_q_heads=Hq, max_seq_len=64, fill=0x7F)
    bt = torch.arange(8, dtype=torch.int32, device="cuda").view(2, 4)
    st = torch.tensor([0, 9], dtype=torch.int32, device="cuda")   # 9, 10, 11: 10 and 11 outside
    ak.atlas_rope_fp8_kv_append(pool, qkv.cuda(), Hq, torch.from_numpy(cos_sin).cuda(), bt, st)
    assert pool.device_error() & ak.DEVERR_APPEND
    k = pool.k_pages.cpu().numpy()
    assert np.all(k[4, :, 10:12] == 0x7F)          # rows 10, 11 of sequence 1 not written
    assert not np.all(k[4, :, 9] == 0x7F)


def test_rope_append_aligned_window_crossing_the_table_end(ak):
    """A full 16-token window starting at a group boundary whose last tokens
    lie past the rotary table: those tokens' K and V rows stay unwritten (the
    whole-row V store is not taken)."""
    Hq, Hkv, D, ps = 4, 2, 128, 16
    qkv, cos_sin = workloads.make_rope_inputs(batch=1, n_new=16, num_q_heads=Hq,
                                              num_kv_heads=Hkv, head_dim=D, max_pos=10, seed=3)
    pool = ak.KVPool(2, ps, Hkv, D, [0.01, 0.01], [0.01, 0.01], max_batch=1, max_q_len=1,
                     num_q_heads=Hq, max_seq_len=32, fill=0x7F)
    bt = torch.tensor([[1, 0]], dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ak.atlas_rope_fp8_kv_append(pool, qkv.cuda(), Hq, torch.from_numpy(cos_sin).cuda(), bt, st)
    assert pool.device_error() & ak.DEVERR_APPEND
    v = v_token_major(pool.v_pages.cpu().numpy())
    k = pool.k_pages.cpu().numpy()
    assert np.all(v[1, :, 10:16] == 0x7F) and np.all(k[1, :, 10:16] == 0x7F)
    assert not np.all(v[1, :, 0:10] == 0x7F)
