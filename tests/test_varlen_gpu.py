"""GPU parity of ragged verify (a different number of new rows per
sequence) and chunked prefill over the paged FP8 cache against the oracle's
packed-row definition, on both decode kernels."""

import numpy as np
import pytest
import torch

from oracle import attention
from paged_fp8_kv_05_b200 import build, workloads

from parity import assert_close, oracle_pages, record_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ak():
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv
    return atlas_kv


def _run(ak, w, q_lens, kernel, split=0, seed=5):
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload
    q, cu = workloads.make_packed_queries(q_lens=q_lens, num_q_heads=w.num_q_heads,
                                          head_dim=w.head_dim, seed=seed)
    maxq = int(max(q_lens))
    dw = DeviceWorkload(w, min_split_tokens=64, max_q_len=maxq)
    dw.pool.set_option(ak.OPT_KERNEL, kernel)
    dw.pool.set_split_tokens(split)
    dq = q.cuda().contiguous()
    dcu = torch.from_numpy(cu).cuda()
    out = torch.full_like(dq, float("nan"))
    ak.atlas_paged_gqa_decode_varlen(dw.pool, dq, dcu, dw.block_table, dw.seq_lens, maxq,
                                     w.max_seq_len, out=out)
    got = out.float().cpu().numpy()
    assert dw.pool.device_error() == 0
    kp, _ = oracle_pages(w, "k")
    vp, _ = oracle_pages(w, "v")
    ref = attention.paged_gqa_decode_varlen(q.float().numpy().astype(np.float64), cu, kp, vp,
                                            w.k_scale, w.v_scale, w.block_table, w.seq_lens,
                                            w.page_size)
    return got, ref


@pytest.mark.parametrize("kernel", [0, 1])
def test_ragged_mtp_verify_on_the_27b_shape(ak, kernel):
    """MTP-verify shape (Hq 40, Hkv 8, D 128, page 16, contexts U[128, 1152])
    with q_len drawn from 1..5 per sequence, batch 128."""
    w = workloads.make_workload(batch=128, num_q_heads=40, num_kv_heads=8, head_dim=128,
                                page_size=16, q_len=1, num_pages=16384,
                                lengths=("uniform", 128, 1152), seed=13)
    q_lens = np.random.default_rng(13).integers(1, 6, size=128)
    got, ref = _run(ak, w, q_lens, kernel)
    max_abs, rel = assert_close(got, ref, f"ragged verify kernel {kernel}")
    record_parity(f"ragged verify (q_len 1..5), kernel option {kernel}", max_abs, rel)


@pytest.mark.parametrize("kernel,split", [(0, 0), (1, 0), (0, 128), (1, 128)])
def test_chunked_prefill_512_rows_over_4k(ak, kernel, split):
    """A 512-token prefill chunk at the end of a 4096-token context (LLaMA-3-8B
    heads): 2048 query rows per KV head, causal inside the chunk; plus a
    second sequence verifying 3 rows and a third with no rows."""
    w = workloads.make_workload(batch=3, num_q_heads=32, num_kv_heads=8, head_dim=128,
                                page_size=16, q_len=1, num_pages=3 * 256 + 8,
                                lengths=("fixed", [4096, 1500, 700]), seed=14)
    got, ref = _run(ak, w, [512, 3, 0], kernel, split)
    max_abs, rel = assert_close(got, ref, f"prefill chunk kernel {kernel} split {split}")
    record_parity(f"prefill 512 over 4096, kernel option {kernel}, split {split or 'auto'}",
                  max_abs, rel)


def test_uniform_q_lens_equal_the_uniform_entry_point(ak):
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload
    w = workloads.make_workload(batch=6, num_q_heads=40, num_kv_heads=8, head_dim=128,
                                page_size=16, q_len=5, num_pages=600,
                                lengths=("uniform", 100, 1000), seed=15)
    dw = DeviceWorkload(w)
    uni = dw.decode(out=torch.empty_like(dw.q))
    cu = torch.arange(0, 31, 5, dtype=torch.int32, device="cuda")
    var = ak.atlas_paged_gqa_decode_varlen(dw.pool, dw.q.reshape(30, 40, 128).contiguous(), cu,
                                           dw.block_table, dw.seq_lens, 5, w.max_seq_len)
    assert torch.equal(var.view(torch.int16).reshape(uni.shape), uni.view(torch.int16))
