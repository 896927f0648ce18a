"""CPU: properties of the launch plan (A1) over random shapes.

Host-only: pools are created on fake addresses and only the plan query and
the workspace sizing are called (no kernel, no device memory).  Without a
GPU the library plans for a 148-SM part.
"""

import ctypes
import math

import pytest
import torch
from hypothesis import given, settings, strategies as st

from paged_fp8_kv_05_b200 import build

build.build()
from paged_fp8_kv_05_b200 import atlas_kv as ak  # noqa: E402

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="plans for a 148-SM part")

_BUF = ctypes.create_string_buffer(1 << 12)
_ADDR = ctypes.c_void_p((ctypes.addressof(_BUF) + 255) // 256 * 256)
ALIGN = 256


def _align(x):
    return (x + ALIGN - 1) // ALIGN * ALIGN


def _plan(pool, B, Hq, q_len, msl):
    buf = (ctypes.c_int32 * 7)()
    assert ak._lib.atlas_paged_gqa_decode_plan(pool, B, Hq, q_len, msl, buf, 7) == ak.ATLAS_OK
    return dict(zip(ak.PLAN_FIELDS, buf))


shapes = st.tuples(
    st.integers(1, 300),                      # batch
    st.sampled_from([1, 2, 4, 8]),            # KV heads
    st.sampled_from([1, 2, 3, 4, 5, 8, 16]),  # group size G
    st.integers(1, 5),                        # q_len
    st.integers(1, 140000),                   # max_seq_len (before the q_len floor)
    st.sampled_from([64, 128]),               # head_dim
    st.sampled_from([0, 1, 2]),               # partition option
    st.sampled_from([0, 64, 128, 448, 2048, 8192]),  # split override
    st.sampled_from([0, 1, 2]),               # kernel option (auto, warp-MMA, tcgen05)
)


@settings(max_examples=300, deadline=None)
@given(shapes)
def test_plan_covers_every_token_and_fits_its_workspace(shape):
    B, Hkv, G, q_len, msl, D, part, split, kern = shape
    Hq = Hkv * G
    msl = max(msl, q_len)
    h = ctypes.c_void_p()
    assert ak._lib.atlas_kv_pool_create(ctypes.byref(h), 1024, 16, Hkv, D, _ADDR, _ADDR, _ADDR,
                                        _ADDR, B, q_len, Hq, _ADDR,
                                        ctypes.c_size_t(1 << 40)) == ak.ATLAS_OK
    try:
        assert ak._lib.atlas_kv_pool_set_option(h, ak.OPT_PARTITION, part) == ak.ATLAS_OK
        assert ak._lib.atlas_kv_pool_set_split_tokens(h, split) == ak.ATLAS_OK
        st_k = ak._lib.atlas_kv_pool_set_option(h, ak.OPT_KERNEL, kern)
        if kern == 2 and D != 128:
            assert st_k == ak.ATLAS_ERR_UNSUPPORTED
            return
        assert st_k == ak.ATLAS_OK
        p = _plan(h, B, Hq, q_len, msl)
    finally:
        ak._lib.atlas_kv_pool_destroy(h)

    R = q_len * G
    rc, rb = p["rows_per_cta"], p["row_blocks"]
    tc = kern == 2 or (kern == 0 and D == 128 and R >= 16)
    assert (p["kernel"] == 3) == tc
    if tc:                                     # tensor-core kernel: 64-row blocks, grid
        T = p["split_tokens"]
        segs = B * Hkv * math.ceil(R / 64)
        assert rc == 64 and rb == math.ceil(R / 64)
        assert T % 128 == 0 and p["num_splits"] * T >= msl and (p["num_splits"] - 1) * T < msl
        if split:
            assert T == (split + 127) // 128 * 128
        else:
            assert 256 <= T <= 8192
        assert p["grid_ctas"] == segs * p["num_splits"]
        slots = segs * p["num_splits"] if p["num_splits"] > 1 else 0
        need = ALIGN + _align(segs * 4) + _align(slots * rc * 4) + _align(slots * rc * D * 4)
        have = ak.atlas_kv_workspace_bytes(B, q_len, Hq, Hkv, D, msl, 64)
        assert have >= need, (p, have, need)
        return
    # the row block is the smallest of 4, 8, 16, 32, 64 holding R rows (or 64)
    assert rc in (4, 8, 16, 32, 64) and rb == math.ceil(R / rc)
    assert rc == 64 or rc >= R
    assert rc == 4 or rc // 2 < R
    segs = B * Hkv * rb
    units = math.ceil(msl / 32)                # 32-token units of a max-length segment
    T = p["split_tokens"]
    if split:
        assert T == split
    if p["kernel"] == 1:                       # grid partition
        assert part in (0, 1)
        assert part == 1 or rc != 64
        assert T % 64 == 0 and p["num_splits"] * T >= msl
        assert (p["num_splits"] - 1) * T < msl
        assert p["grid_ctas"] == segs * p["num_splits"]
        if not split:
            assert 256 <= T <= 8192
        slots = segs * p["num_splits"] if p["num_splits"] > 1 else 0
    else:                                      # balanced partition
        assert p["kernel"] == 2 and part in (0, 2)
        assert part == 2 or rc == 64
        per_cta = math.ceil(segs * units / p["grid_ctas"])
        assert p["grid_ctas"] <= segs * units
        assert split or per_cta <= 1024        # the per-CTA unit table bound
        if not split:
            assert T == 32 * per_cta
        slots = segs + p["grid_ctas"]
    need = ALIGN + _align(segs * 4) + _align(slots * rc * 4) + _align(slots * rc * D * 4)
    # a workspace sized for every override down to 64 tokens holds this plan
    have = ak.atlas_kv_workspace_bytes(B, q_len, Hq, Hkv, D, msl, 64)
    assert have >= need, (p, have, need)
