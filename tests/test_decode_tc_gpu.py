"""GPU parity of the 5th-generation tensor-core decode kernel (tcgen05.mma,
accumulators in tensor memory) against the float64 oracle.

The kernel is forced with ATLAS_OPT_KERNEL = 2 on shapes it would not get
automatically too (few query rows, every page size, two 64-row blocks), with
the automatic split length and with short splits that cut every segment into
many parts merged by log-sum-exp.  The named verify and MQA workloads, which
select it automatically, are covered in test_decode_gpu.py and
test_sharp_gpu.py.
"""

import numpy as np
import pytest
import torch

from paged_fp8_kv_05_b200 import build, workloads

from parity import assert_close, oracle_decode, record_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ak():
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv
    return atlas_kv


def _case(B, Hq, Hkv, D, ps, lens, q_len, seed=0, P=None, table="perm"):
    need = sum((L + ps - 1) // ps for L in lens)
    return workloads.make_workload(batch=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                                   page_size=ps, q_len=q_len, num_pages=P or need + 5,
                                   lengths=("fixed", list(lens)), table=table, seed=seed)


def _dw(w, **kw):
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload
    return DeviceWorkload(w, min_split_tokens=64, **kw)


CASES = [
    # (B, Hq, Hkv, D, ps, lens, q_len)
    (3, 8, 2, 128, 16, [1, 15, 16], 1),           # 4 rows, one-token and one-piece contexts
    (4, 8, 2, 128, 16, [17, 31, 32, 33], 1),
    (2, 32, 8, 128, 16, [5, 16], 5),              # 20 rows, causal drafts
    (3, 40, 8, 128, 16, [5, 6, 21], 5),           # 25 rows (the verify shape)
    (2, 16, 1, 128, 64, [63, 65], 1),             # MQA, 16 rows, page 64 tails
    (2, 64, 1, 128, 64, [64, 200, ], 1),          # MQA, 64 rows
    (2, 128, 1, 128, 16, [300, 129], 1),          # two 64-row blocks
    (1, 8, 1, 128, 16, [1000], 2),
    (5, 8, 2, 128, 48, [47, 48, 49, 96, 1], 1),   # page 48
    (2, 8, 2, 128, 1024, [1500, 3000], 1),        # largest page size
    (2, 40, 8, 128, 16, [300, 77], 5),
    (3, 64, 1, 128, 64, [127, 128, 129], 1),      # tile boundaries
    (2, 40, 8, 128, 16, [2000, 4500], 5),         # long verify: many tiles, rescales
]


@pytest.mark.parametrize("split", [0, 128, 256])
@pytest.mark.parametrize("case", CASES)
def test_tc_kernel_matches_oracle(ak, case, split):
    w = _case(*case, seed=17)
    dw = _dw(w)
    dw.pool.set_option(ak.OPT_KERNEL, ak.KERNEL_TC)
    dw.pool.set_split_tokens(split)
    plan = dw.plan()
    assert plan["kernel"] == 3
    if split:
        assert plan["split_tokens"] == split
    out = torch.full_like(dw.q, float("nan"))
    got = dw.decode(out=out).float().cpu().numpy()
    assert dw.pool.device_error() == 0
    max_abs, rel = assert_close(got, oracle_decode(w), f"tcgen05 {case} split {split}")
    record_parity(f"tcgen05 {case} split {split or 'auto'}", max_abs, rel)


def test_tc_kernel_is_selected_for_the_verify_and_mqa_workloads(ak):
    for cfg in (2, 4):
        w = workloads.make_workload(**{**{k: v for k, v in workloads.CONFIGS[cfg].items()
                                         if k != "name"}, "batch": 2,
                                       "lengths": ("fixed", [300, 700])})
        dw = _dw(w)
        assert dw.plan()["kernel"] == 3, cfg
    w = _case(2, 32, 8, 128, 16, [300, 700], 1)      # 4 rows per KV head: warp-MMA kernel
    assert _dw(w).plan()["kernel"] in (1, 2)


def test_tc_mtp_rows_ignore_later_drafts(ak):
    from oracle.paged import GROUP_POS
    q_len = 5
    w = _case(2, 40, 8, 128, 16, [130, 77], q_len, seed=8)
    dw = _dw(w)
    dw.pool.set_option(ak.OPT_KERNEL, ak.KERNEL_TC)
    base = dw.decode(out=torch.empty_like(dw.q)).clone()
    for i in range(q_len - 1):
        kp = dw.pool.k_pages.clone()
        vp = dw.pool.v_pages.clone()
        for b in range(w.batch):
            L = int(w.seq_lens[b])
            for t in range(L - q_len + i + 1, L):
                page, slot = int(w.block_table[b, t // 16]), t % 16
                kp[page, :, slot, :] = 0x3C
                vp[page, :, slot // 16, :, int(GROUP_POS[slot % 16])] = 0xC4
        got = ak.atlas_paged_gqa_decode(dw.pool, dw.q, dw.block_table, dw.seq_lens,
                                        w.max_seq_len, out=torch.empty_like(dw.q),
                                        k_pages=kp, v_pages=vp)
        a = got[:, : i + 1].contiguous().view(torch.int16)
        b_ = base[:, : i + 1].contiguous().view(torch.int16)
        assert torch.equal(a, b_), f"row {i} changed"
        assert not torch.equal(got[:, i + 1:], base[:, i + 1:])


def test_tc_deterministic_and_page_permutation_bit_identical(ak):
    w = _case(3, 64, 1, 128, 16, [333, 1000, 700], 1, seed=6, P=200)
    dw = _dw(w)
    dw.pool.set_option(ak.OPT_KERNEL, ak.KERNEL_TC)
    base = dw.decode(out=torch.empty_like(dw.q)).clone()
    again = dw.decode(out=torch.empty_like(dw.q))
    assert torch.equal(again.view(torch.int16), base.view(torch.int16))
    rng = np.random.default_rng(1)
    perm = torch.from_numpy(rng.permutation(w.num_pages)).cuda()
    kp = torch.empty_like(dw.pool.k_pages)
    vp = torch.empty_like(dw.pool.v_pages)
    kp[perm] = dw.pool.k_pages
    vp[perm] = dw.pool.v_pages
    bt = dw.block_table.clone()
    valid = bt >= 0
    bt[valid] = perm[bt[valid].long()].int()
    got = ak.atlas_paged_gqa_decode(dw.pool, dw.q, bt, dw.seq_lens, w.max_seq_len,
                                    out=torch.empty_like(dw.q), k_pages=kp, v_pages=vp)
    assert torch.equal(got.view(torch.int16), base.view(torch.int16))


def test_tc_fused_step_equals_append_then_decode(ak):
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload
    w = _case(3, 40, 8, 128, 16, [66, 400, 17], 5, seed=31)
    sep = DeviceWorkload(w, fill_cache=False, min_split_tokens=64)
    fus = DeviceWorkload(w, fill_cache=False, min_split_tokens=64)
    for dw in (sep, fus):
        dw.fill_prefix()
        dw.pool.set_option(ak.OPT_KERNEL, ak.KERNEL_TC)
        dw.pool.set_split_tokens(128)
    sep.append_new()
    out_sep = sep.decode(out=torch.empty_like(sep.q))
    out_fus = fus.step(out=torch.empty_like(fus.q))
    torch.cuda.synchronize()
    assert sep.pool.device_error() == 0 and fus.pool.device_error() == 0
    assert torch.equal(sep.pool.k_pages, fus.pool.k_pages)
    assert torch.equal(sep.pool.v_pages, fus.pool.v_pages)
    assert torch.equal(out_sep.view(torch.int16), out_fus.view(torch.int16))
    assert_close(out_fus.float().cpu().numpy(), oracle_decode(w), "tcgen05 fused step")


def test_tc_bad_inputs_flag_device_errors(ak):
    w = _case(3, 40, 8, 128, 16, [40, 300, 40], 2, seed=11)
    dw = _dw(w)
    dw.pool.set_option(ak.OPT_KERNEL, ak.KERNEL_TC)
    dw.decode()
    assert dw.pool.device_error() == 0
    bt = dw.block_table.clone()
    bt[1, 3] = w.num_pages + 7                      # page id out of range in sequence 1
    sl = dw.seq_lens.clone()
    sl[2] = 1                                       # seq_len < q_len
    out = torch.full_like(dw.q, 5.0)
    ak.atlas_paged_gqa_decode(dw.pool, dw.q, bt, sl, w.max_seq_len, out=out)
    err = dw.pool.device_error()
    assert err & ak.DEVERR_PAGE_ID and err & ak.DEVERR_SEQ_LEN
    assert torch.all(out[2] == 0)
    assert torch.isfinite(out.float()).all()        # the skipped page never reaches O
    ref = oracle_decode(w)
    assert_close(out[0:1].float().cpu().numpy(), ref[0:1], "untouched sequence")
    dw.decode()
    assert dw.pool.device_error() == 0


def test_tc_lost_copy_times_out_and_the_library_stays_usable(ak):
    """CTA 0's producer never issues its second tile (test-only option), the
    wait for it runs out after 1 ms: ATLAS_DEVERR_TIMEOUT, every other
    (sequence, KV head) still matches the oracle, tensor memory is released
    (the next call runs and matches everywhere)."""
    w = _case(4, 40, 8, 128, 16, [700, 1500, 64, 300], 5, seed=12)
    dw = _dw(w)
    dw.pool.set_option(ak.OPT_KERNEL, ak.KERNEL_TC)
    dw.pool.set_option(ak.OPT_WAIT_LIMIT_US, 1000)
    dw.pool.set_option(ak.OPT_TEST_SKIP_UNIT, 1)
    out = torch.full_like(dw.q, float("nan"))
    dw.decode(out=out)
    err = dw.pool.device_error()
    assert err & ak.DEVERR_TIMEOUT, err
    ref = oracle_decode(w)
    got = out.float().cpu().numpy()
    G = w.num_q_heads // w.num_kv_heads
    keep = np.ones(got.shape[:3], bool)
    keep[0, :, 0:G] = False                          # sequence 0, KV head 0: unspecified
    assert_close(got[keep], ref[keep], "segments other than the timed-out one")
    dw.pool.set_option(ak.OPT_TEST_SKIP_UNIT, -1)
    dw.pool.set_option(ak.OPT_WAIT_LIMIT_US, 0)
    again = dw.decode(out=torch.empty_like(dw.q))
    assert dw.pool.device_error() == 0
    assert_close(again.float().cpu().numpy(), ref, "the call after the timeout")


def test_tc_work_order_serves_every_item_once(ak):
    """The CTAs rank their (sequence, segment, split) items in-kernel, longest
    first.  230 sequences (more than one 192-sequence chunk of the rank
    search) with lengths on every side of the 128-token tile and 256-token
    split boundaries, and three sequences the kernel must skip (length 0 <
    q_len) spread over both chunks: every served row matches the oracle (no
    item lost: the output starts as NaN; none served twice: the split partials
    would not merge to the oracle), the skipped ones are zero and flagged."""
    base = [1, 2, 127, 128, 129, 200, 255, 256, 257, 300, 383, 384, 385, 511, 512,
            513, 640, 700, 767, 768, 769, 1000, 1023, 1024, 1025]
    rng = np.random.default_rng(5)
    lens = [int(x) for x in rng.permutation(np.resize(base, 230))]
    w = _case(230, 8, 2, 128, 16, lens, 1, seed=23)
    dw = _dw(w)
    dw.pool.set_option(ak.OPT_KERNEL, ak.KERNEL_TC)
    dw.pool.set_split_tokens(256)
    plan = dw.plan()
    assert plan["kernel"] == 3 and plan["split_tokens"] == 256
    skip = [0, 150, 229]
    sl = dw.seq_lens.clone()
    sl[skip] = 0
    out = torch.full_like(dw.q, float("nan"))
    ak.atlas_paged_gqa_decode(dw.pool, dw.q, dw.block_table, sl, w.max_seq_len, out=out)
    err = dw.pool.device_error()
    assert err & ak.DEVERR_SEQ_LEN and not err & ~ak.DEVERR_SEQ_LEN, err
    got = out.float().cpu().numpy()
    assert np.all(got[skip] == 0)
    keep = np.ones(len(lens), bool)
    keep[skip] = False
    ref = oracle_decode(w)
    max_abs, rel = assert_close(got[keep], ref[keep], "tcgen05 work order, 230 sequences")
    record_parity("tcgen05 work order, 230 sequences, split 256", max_abs, rel)
