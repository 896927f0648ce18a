"""GPU: the no-allocation decode entry point.

Callers that cannot allocate device memory (a host framework that owns every
allocation and hands the library only its inputs and outputs) use
atlas_paged_gqa_decode_noalloc, whose scratch is a static device array inside
the library.  Its output must match the pool-based atlas_paged_gqa_decode
within the decode tolerance, and the float64 oracle, on two calls in a row
(the second call reuses the scratch the first one left behind).  A call whose
segments are too long for the scratch is rejected before anything runs.
This file sorts last so that a run stopping at the first failure has already
run every other test.
"""

import numpy as np
import pytest
import torch

from paged_fp8_kv_05_b200 import build, workloads

from parity import assert_close, errors, oracle_decode, record_parity

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 1e-2, 5e-3
SCRATCH_BYTES = 8 << 20          # the library's static scratch array
MAX_WHOLE_SEGMENT = 65536        # longest segment of the one-CTA-per-segment fallback


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


def _partial_bytes(plan, w):
    """Split-KV partial bytes the automatic plan of the pool entry point needs
    (float32 O rows plus one log2-sum-exp per row and slot)."""
    segs = w.batch * w.num_kv_heads * plan["row_blocks"]
    slots = segs * plan["num_splits"] if plan["kernel"] == 1 else segs + plan["grid_ctas"]
    if plan["kernel"] == 1 and plan["num_splits"] == 1:
        slots = 0
    return slots * plan["rows_per_cta"] * (w.head_dim + 1) * 4


@pytest.mark.parametrize("name", ["decode", "verify", "mqa"])
def test_noalloc_matches_pool_entry_point_on_two_calls(name):
    w = _workload(name)
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv as ak
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload

    dw = DeviceWorkload(w)
    # the no-allocation entry point runs the FP8 warp-MMA kernel with the
    # automatic partition; compare with the pool entry point on that kernel
    dw.pool.set_option(ak.OPT_KERNEL, ak.KERNEL_WARP_MMA)
    ref = dw.decode(out=torch.empty_like(dw.q)).float()
    assert dw.pool.device_error() == 0
    needs = _partial_bytes(dw.plan(), w)
    if name == "mqa":
        # this case is the fallback: the automatic plan's partials exceed the scratch
        assert needs > SCRATCH_BYTES, needs
    else:
        assert 0 < needs < SCRATCH_BYTES, needs
    oracle = oracle_decode(w)
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
        max_abs, rel = assert_close(got.cpu().numpy(), oracle, f"noalloc {name}, call {call}")
        record_parity(f"noalloc {name}, call {call} (vs oracle)", max_abs, rel)


def test_noalloc_rejects_a_segment_longer_than_the_fallback_allows():
    """Ragged-MQA shape whose automatic partials exceed the scratch and whose
    max_seq_len (80000) exceeds the fallback's one-CTA-per-segment bound: the
    call returns ATLAS_ERR_WORKSPACE and launches nothing."""
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv as ak
    dev = torch.device("cuda")
    B, Hq, Hkv, D, ps, P = 64, 64, 1, 128, 64, 8
    max_seq_len = 80000
    assert max_seq_len > MAX_WHOLE_SEGMENT
    max_blocks = (max_seq_len + ps - 1) // ps
    q = torch.zeros(B, 1, Hq, D, dtype=torch.bfloat16, device=dev)
    out = torch.full_like(q, float("nan"))
    kp = torch.zeros(P, Hkv, ps, D, dtype=torch.uint8, device=dev)
    vp = torch.zeros(P, Hkv, ps // 16, D, 16, dtype=torch.uint8, device=dev)
    sc = torch.ones(Hkv, dtype=torch.float32, device=dev)
    table = torch.zeros(B, max_blocks, dtype=torch.int32, device=dev)
    lens = torch.full((B,), max_seq_len, dtype=torch.int32, device=dev)
    with pytest.raises(ak.AtlasError) as exc:
        ak.atlas_paged_gqa_decode_noalloc(q, kp, vp, sc, sc, table, lens, max_seq_len, out=out)
    assert exc.value.status == ak.ATLAS_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.isnan(out.float()).all()
