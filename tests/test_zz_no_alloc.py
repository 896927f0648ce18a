"""GPU: the no-allocation decode entry point.

Callers that cannot allocate device memory (a host framework that owns every
allocation and hands the library only its inputs and outputs) use
atlas_paged_gqa_decode_noalloc, whose scratch is a static device array inside
the library.  Its output must match the pool-based atlas_paged_gqa_decode
within the decode tolerance, on two calls in a row (the second call reuses
the scratch the first one left behind).  This file sorts last so that a run
stopping at the first failure has already run every other test.
"""

import pytest
import torch

from paged_fp8_kv_05_b200 import build, workloads

from parity import errors

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 1e-2, 5e-3


def _workload(name):
    if name == "decode":      # LLaMA-3-8B-shaped decode: split-KV partials live in the scratch
        return workloads.config_workload(1)
    if name == "verify":      # MTP verify, q_len 5, two warps per K/V stream
        return workloads.make_workload(
            batch=6, num_q_heads=40, num_kv_heads=8, head_dim=128, page_size=16, q_len=5,
            num_pages=700, lengths=("uniform", 100, 1500), seed=21)
    # ragged MQA, page 64: the partials would not fit, so one split per sequence
    return workloads.make_workload(
        batch=96, num_q_heads=64, num_kv_heads=1, head_dim=128, page_size=64, q_len=1,
        num_pages=20000, lengths=("loguniform", 256, 8192), table="frag", seed=22)


@pytest.mark.parametrize("name", ["decode", "verify", "mqa"])
def test_noalloc_matches_pool_entry_point_on_two_calls(name):
    w = _workload(name)
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv as ak
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload

    dw = DeviceWorkload(w)
    ref = dw.decode(out=torch.empty_like(dw.q)).float()
    assert dw.pool.device_error() == 0
    for call in range(2):
        out = torch.full_like(dw.q, float("nan"))
        ak.atlas_paged_gqa_decode_noalloc(dw.q, dw.pool.k_pages, dw.pool.v_pages,
                                          dw.pool.k_scale, dw.pool.v_scale, dw.block_table,
                                          dw.seq_lens, w.max_seq_len, out=out)
        torch.cuda.synchronize()
        got = out.float()
        assert torch.isfinite(got).all(), f"{name}, call {call}: non-finite output"
        max_abs, rel = errors(got.cpu().numpy(), ref.cpu().numpy())
        assert max_abs <= MAX_ABS and rel <= REL_L2, f"{name}, call {call}: {max_abs}, {rel}"
