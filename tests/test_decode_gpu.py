"""GPU parity of paged decode / MTP-verify attention against the float64
oracle, on the five named workloads (full output; the long-context case on
sampled sequences), edge cases and invariants."""

import numpy as np
import pytest
import torch

from oracle import attention
from oracle.paged import GROUP_POS
from paged_fp8_kv_05_b200 import build, workloads

from parity import assert_close, errors, oracle_decode, oracle_pages, record_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ak():
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv
    return atlas_kv


def _dw(w, **kw):
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload
    return DeviceWorkload(w, **kw)


_ORACLE = {}


def _oracle_named(cfg, w):
    if cfg not in _ORACLE:
        _ORACLE[cfg] = oracle_decode(w)
    return _ORACLE[cfg]


# kernel 0 = automatic (the tensor-core kernel for the verify and MQA
# workloads 2 and 4, the warp-MMA kernel for 0 and 1); the warp-MMA kernel is
# also checked on 2 and 4, in both of its partitions where they differ
# (partition 0 = automatic: grid, or balanced when one K/V stream serves a CTA)
@pytest.mark.parametrize("cfg,kernel,partition", [
    (0, 0, 0), (1, 0, 0), (2, 0, 0), (4, 0, 0),
    (1, 1, 2), (2, 1, 0), (4, 1, 0), (4, 1, 1)])
def test_named_workload_full_output(ak, cfg, kernel, partition):
    w = workloads.config_workload(cfg)
    dw = _dw(w)
    dw.pool.set_option(ak.OPT_KERNEL, kernel)
    dw.pool.set_option(ak.OPT_PARTITION, partition)
    got = dw.decode().float().cpu().numpy()
    assert dw.pool.device_error() == 0
    ref = _oracle_named(cfg, w)
    plan = dw.plan()
    what = f"config {cfg}, kernel {plan['kernel']} (option {kernel}), partition {partition}"
    max_abs, rel = assert_close(got, ref, what)
    record_parity(what, max_abs, rel)
    print(f"config {cfg}: max-abs {max_abs:.3e} rel-L2 {rel:.3e} plan {dw.plan()}")


def test_long_context_every_sequence(ak):
    """The long-context workload (B=4, 65k-131k tokens, 1 % of key rows x8
    before quantisation): every output element of all four sequences against
    the oracle, with the automatic plan (several splits per sequence)."""
    w = workloads.config_workload(3)
    dw = _dw(w)
    got = dw.decode().float().cpu().numpy()
    assert dw.pool.device_error() == 0
    plan = dw.plan()
    assert plan["num_splits"] > 1
    del dw
    torch.cuda.empty_cache()
    ref = oracle_decode(w)
    assert np.all(np.isfinite(ref))
    max_abs, rel = assert_close(got, ref, "config 3 (all sequences)")
    record_parity("config 3, all 4 sequences", max_abs, rel)
    print(f"config 3: max-abs {max_abs:.3e} rel-L2 {rel:.3e} plan {plan}")


def _case(B, Hq, Hkv, D, ps, lens, q_len, seed=0, P=None, table="perm"):
    need = sum((L + ps - 1) // ps for L in lens)
    return workloads.make_workload(batch=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                                   page_size=ps, q_len=q_len, num_pages=P or need + 5,
                                   lengths=("fixed", list(lens)), table=table, seed=seed)


EDGE = [
    # (B, Hq, Hkv, D, ps, lens, q_len)
    (3, 8, 2, 64, 16, [1, 15, 16], 1),
    (4, 8, 2, 128, 16, [17, 31, 32, 33], 1),
    (2, 32, 8, 128, 16, [5, 16], 5),
    (3, 40, 8, 128, 16, [5, 6, 21], 5),
    (2, 4, 4, 128, 16, [1, 40], 1),              # MHA (G = 1)
    (2, 16, 1, 128, 64, [63, 65], 1),            # MQA, page 64, ragged tails
    (2, 64, 1, 128, 64, [64, 200], 1),           # MQA with 64 rows
    (2, 12, 4, 64, 32, [95, 97], 3),             # page 32, D 64, G 3, q_len 3
    (1, 8, 1, 128, 16, [1000], 2),
    (5, 8, 2, 128, 48, [47, 48, 49, 96, 1], 1),  # page 48
    (2, 8, 2, 128, 1024, [1500, 3000], 1),       # largest page size
    (2, 40, 8, 64, 16, [300, 77], 5),            # D 64, two warps per K/V stream
    (2, 64, 1, 64, 16, [500, 33], 1),            # D 64, four warps per stream (balanced)
]


@pytest.mark.parametrize("kernel", [0, 1])
@pytest.mark.parametrize("case", EDGE)
def test_edge_cases(ak, case, kernel):
    w = _case(*case)
    dw = _dw(w)
    dw.pool.set_option(ak.OPT_KERNEL, kernel)
    got = dw.decode().float().cpu().numpy()
    assert dw.pool.device_error() == 0
    assert_close(got, oracle_decode(w), f"edge {case}")


@pytest.mark.parametrize("partition", [1, 2])
@pytest.mark.parametrize("split", [0, 64])
@pytest.mark.parametrize("case", [
    (4, 8, 2, 128, 16, [17, 31, 32, 33], 1),
    (6, 32, 8, 128, 16, [1, 40, 900, 2000, 33, 64], 1),
    (3, 40, 8, 128, 16, [5, 6, 210], 5),
    (3, 64, 1, 128, 64, [64, 200, 1500], 1),
])
def test_both_partitions(ak, case, split, partition):
    """Grid splits and balanced ranges, with automatic and 64-token parts (a
    segment cut into many parts, merged by the CTA that finishes it last)."""
    w = _case(*case, seed=11)
    dw = _dw(w, min_split_tokens=64)
    dw.pool.set_option(ak.OPT_KERNEL, ak.KERNEL_WARP_MMA)
    dw.pool.set_option(ak.OPT_PARTITION, partition)
    dw.pool.set_split_tokens(split)
    plan = dw.plan()
    assert plan["kernel"] == partition
    got = dw.decode().float().cpu().numpy()
    assert dw.pool.device_error() == 0
    assert_close(got, oracle_decode(w), f"{case} split {split} partition {partition}")


@pytest.mark.parametrize("split", [64, 128, 192, 512, 8192])
def test_split_count_invariance(ak, split):
    w = _case(3, 32, 8, 128, 16, [700, 1500, 64], 2, seed=3)
    dw = _dw(w, min_split_tokens=64)
    dw.pool.set_split_tokens(split)
    plan = dw.plan()
    assert plan["split_tokens"] == split
    got = dw.decode().float().cpu().numpy()
    assert dw.pool.device_error() == 0
    assert_close(got, oracle_decode(w), f"split {split}")


def test_split_results_agree_with_each_other(ak):
    w = _case(2, 16, 4, 128, 16, [2000, 1333], 1, seed=4)
    dw = _dw(w, min_split_tokens=64)
    outs = []
    for split in (64, 448, 8192):
        dw.pool.set_split_tokens(split)
        outs.append(dw.decode(out=torch.empty_like(dw.q)).float().cpu().numpy())
    for o in outs[1:]:
        max_abs, rel = errors(o, outs[0])
        assert max_abs <= 1e-2 and rel <= 5e-3


def test_deterministic_bits(ak):
    w = _case(4, 32, 8, 128, 16, [3000, 100, 2049, 17], 1, seed=5)
    dw = _dw(w)
    a = dw.decode(out=torch.empty_like(dw.q)).clone()
    b = dw.decode(out=torch.empty_like(dw.q)).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_page_permutation_bit_identical(ak):
    w = _case(3, 16, 4, 128, 16, [333, 100, 700], 3, seed=6, P=200)
    dw = _dw(w)
    base = dw.decode(out=torch.empty_like(dw.q)).clone()
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


def test_mtp_rows_ignore_later_drafts(ak):
    q_len = 5
    w = _case(2, 40, 8, 128, 16, [130, 77], q_len, seed=8)
    dw = _dw(w)
    dw.pool.set_option(ak.OPT_KERNEL, ak.KERNEL_WARP_MMA)
    base = dw.decode(out=torch.empty_like(dw.q)).clone()
    for i in range(q_len - 1):
        kp = dw.pool.k_pages.clone()
        vp = dw.pool.v_pages.clone()
        for b in range(w.batch):
            L = int(w.seq_lens[b])
            for t in range(L - q_len + i + 1, L):
                page, slot = int(w.block_table[b, t // 16]), t % 16
                kp[page, :, slot, :] = 0x3C                 # K pages: token-major
                vp[page, :, slot // 16, :, int(GROUP_POS[slot % 16])] = 0xC4  # V: 16-slot groups
        got = ak.atlas_paged_gqa_decode(dw.pool, dw.q, dw.block_table, dw.seq_lens,
                                        w.max_seq_len, out=torch.empty_like(dw.q),
                                        k_pages=kp, v_pages=vp)
        a = got[:, : i + 1].contiguous().view(torch.int16)
        b_ = base[:, : i + 1].contiguous().view(torch.int16)
        assert torch.equal(a, b_), f"row {i} changed"
        assert not torch.equal(got[:, i + 1:], base[:, i + 1:])


def test_explicit_sm_scale_and_unit_scales(ak):
    w = _case(2, 8, 2, 64, 16, [50, 90], 1, seed=9)
    dw = _dw(w)
    got = ak.atlas_paged_gqa_decode(dw.pool, dw.q, dw.block_table, dw.seq_lens, w.max_seq_len,
                                    out=torch.empty_like(dw.q), sm_scale=0.3)
    assert_close(got.float().cpu().numpy(), oracle_decode(w, sm_scale=0.3), "sm_scale 0.3")
    ones = torch.ones(w.num_kv_heads, device="cuda")
    got1 = ak.atlas_paged_gqa_decode(dw.pool, dw.q, dw.block_table, dw.seq_lens, w.max_seq_len,
                                     out=torch.empty_like(dw.q), k_scale=ones, v_scale=ones)
    kp, _ = oracle_pages(w, "k")
    vp, _ = oracle_pages(w, "v")
    ref1 = attention.paged_gqa_decode(w.q_f64(), kp, vp, np.ones(2, np.float32),
                                      np.ones(2, np.float32), w.block_table, w.seq_lens, 1, 16)
    # raw E4M3 values reach +-448: compare relative to the output's scale
    g = got1.float().cpu().numpy()
    assert np.linalg.norm(g - ref1) / np.linalg.norm(ref1) <= 5e-3


def test_full_table_max_seq_len(ak):
    # every sequence uses all of its block-table row: max_seq_len = max_blocks * page_size
    w = _case(2, 8, 2, 128, 16, [256, 256], 1, seed=10)
    assert w.max_seq_len == w.max_blocks * w.page_size
    dw = _dw(w)
    assert_close(dw.decode().float().cpu().numpy(), oracle_decode(w), "full table")


def test_bad_inputs_flag_device_errors_without_faulting(ak):
    w = _case(3, 8, 2, 128, 16, [40, 40, 40], 2, seed=11)
    dw = _dw(w)
    dw.decode()
    assert dw.pool.device_error() == 0
    bt = dw.block_table.clone()
    bt[1, 1] = w.num_pages + 7                       # page id out of range
    sl = dw.seq_lens.clone()
    sl[2] = 1                                        # seq_len < q_len
    out = torch.full_like(dw.q, 5.0)
    ak.atlas_paged_gqa_decode(dw.pool, dw.q, bt, sl, w.max_seq_len, out=out)
    err = dw.pool.device_error()
    assert err & ak.DEVERR_PAGE_ID and err & ak.DEVERR_SEQ_LEN
    assert torch.all(out[2] == 0)
    ref = oracle_decode(w)
    assert_close(out[0:1].float().cpu().numpy(), ref[0:1], "untouched sequence")
    # the library stays usable
    dw.decode()
    assert dw.pool.device_error() == 0


def test_lost_copy_times_out_and_the_library_stays_usable(ak):
    """Bounded-wait error path, without any fault: CTA 0's first K/V stream
    never issues the bulk copies of its second unit (a test-only pool option),
    so nothing is ever in flight for that stage and the wait for it runs out
    after 1 ms.  The call must flag ATLAS_DEVERR_TIMEOUT and return; every
    (sequence, KV head) other than CTA 0's -- sequence 0, KV head 0 in the grid
    partition -- must still match the oracle, and the next normal call on the
    same pool must be clean and match everywhere."""
    w = _case(4, 32, 8, 128, 16, [700, 1500, 64, 300], 1, seed=12)
    dw = _dw(w)
    dw.pool.set_option(ak.OPT_KERNEL, ak.KERNEL_WARP_MMA)
    dw.pool.set_option(ak.OPT_PARTITION, 1)
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
    keep[0, :, 0:G] = False                         # sequence 0, KV head 0: unspecified
    assert_close(got[keep], ref[keep], "segments other than the timed-out one")
    dw.pool.set_option(ak.OPT_TEST_SKIP_UNIT, -1)
    dw.pool.set_option(ak.OPT_WAIT_LIMIT_US, 0)
    again = dw.decode(out=torch.empty_like(dw.q))
    assert dw.pool.device_error() == 0
    assert_close(again.float().cpu().numpy(), ref, "the call after the timeout")


def test_empty_batch_is_a_noop(ak):
    w = _case(1, 8, 2, 64, 16, [10], 1)
    dw = _dw(w)
    q0 = dw.q[:0]
    out0 = torch.empty_like(q0)
    ak.atlas_paged_gqa_decode(dw.pool, q0, dw.block_table[:0], dw.seq_lens[:0], 10, out=out0)
    assert dw.pool.device_error() == 0


FUSED_CASES = [
    # (workload builder, split override): new tokens inside one piece, across a
    # page and a split boundary, and the two named decode / verify shapes
    (lambda: _case(3, 32, 8, 128, 16, [66, 200, 17], 5, seed=31), 64),
    (lambda: _case(2, 16, 1, 128, 64, [130, 64], 3, seed=32), 64),
    (lambda: workloads.config_workload(1), 0),
    (lambda: workloads.config_workload(2), 0),
]


@pytest.mark.parametrize("case", range(len(FUSED_CASES)))
def test_fused_step_equals_append_then_decode(ak, case):
    make, split = FUSED_CASES[case]
    w = make()
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload
    sep = DeviceWorkload(w, fill_cache=False, min_split_tokens=64)
    fus = DeviceWorkload(w, fill_cache=False, min_split_tokens=64)
    for dw in (sep, fus):
        dw.fill_prefix()
        if split:
            dw.pool.set_split_tokens(split)
    sep.append_new()
    out_sep = sep.decode(out=torch.empty_like(sep.q))
    out_fus = fus.step(out=torch.empty_like(fus.q))
    torch.cuda.synchronize()
    assert sep.pool.device_error() == 0 and fus.pool.device_error() == 0
    assert torch.equal(sep.pool.k_pages, fus.pool.k_pages)
    assert torch.equal(sep.pool.v_pages, fus.pool.v_pages)
    assert torch.equal(out_sep.view(torch.int16), out_fus.view(torch.int16))
    # and the fused step on its own matches the oracle
    assert_close(out_fus.float().cpu().numpy(), oracle_decode(w), f"fused case {case}")
