"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before anything is enqueued (CPU only: every call
below that carries fake pointers also carries at least one invalid argument,
so no kernel is ever launched on them)."""

import ctypes
import os
import re

import pytest

from paged_fp8_kv_05_b200 import build

build.build()  # in-tree, no-op when up to date

from paged_fp8_kv_05_b200 import atlas_kv as ak  # noqa: E402

HEADER = os.path.join(build.ROOT, "include", "atlas_kv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(atlas_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("atlas_kv_pool_create", "atlas_fp8_kv_append", "atlas_paged_gqa_decode"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(ak.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert missing == []
    assert set(declared_functions()) == set(ak.EXPORTED)


def test_library_exports_nothing_else():
    out = os.popen(f"nm -D --defined-only {ak.LIB_PATH}").read()
    atlas_syms = sorted(set(re.findall(r"\b(atlas_[A-Za-z0-9_]+)\b", out)))
    assert atlas_syms == declared_functions()


def test_status_strings_and_version():
    assert ak.status_string(0) == "ok"
    assert "workspace" in ak.status_string(-3)
    assert ak.version().count(".") == 2


def test_workspace_bytes():
    # batch 32, 8 KV heads, group 4 -> 256 segments of 4 rows; 4096 tokens = 128
    # units each; 256-token ranges -> 32768 / 8 = 4096 CTAs; one partial slot per
    # segment plus one per CTA, each 4 rows x (128 + 1) floats
    n = ak.atlas_kv_workspace_bytes(32, 1, 32, 8, 128, 4096, 256)
    segs, ctas = 32 * 8, 32 * 8 * 128 // 8
    assert n >= 256 + segs * 4 + (segs + ctas) * 4 * (128 + 1) * 4
    assert ak.atlas_kv_workspace_bytes(32, 1, 32, 8, 96, 4096) == 0     # head_dim
    assert ak.atlas_kv_workspace_bytes(32, 0, 32, 8, 128, 4096) == 0    # q_len
    assert ak.atlas_kv_workspace_bytes(32, 1, 32, 6, 128, 4096) == 0    # 32 % 6 != 0
    assert (ak.atlas_kv_workspace_bytes(32, 1, 32, 8, 128, 4096, 64)
            > ak.atlas_kv_workspace_bytes(32, 1, 32, 8, 128, 4096, 256)
            > ak.atlas_kv_workspace_bytes(32, 1, 32, 8, 128, 4096, 0))


class _Fake:
    """A host buffer used only as an address; never dereferenced here."""

    def __init__(self, n=1 << 16):
        self.buf = ctypes.create_string_buffer(n + 512)
        addr = ctypes.addressof(self.buf)
        self.ptr = ctypes.c_void_p((addr + 255) // 256 * 256)


F = _Fake()


def _create(**kw):
    args = dict(num_pages=64, page_size=16, num_kv_heads=2, head_dim=64, k=F.ptr, v=F.ptr,
                ks=F.ptr, vs=F.ptr, max_batch=4, max_q_len=5, num_q_heads=8, ws=F.ptr,
                ws_bytes=1 << 16)
    args.update(kw)
    h = ctypes.c_void_p()
    st = ak._lib.atlas_kv_pool_create(ctypes.byref(h), args["num_pages"], args["page_size"],
                                      args["num_kv_heads"], args["head_dim"], args["k"],
                                      args["v"], args["ks"], args["vs"], args["max_batch"],
                                      args["max_q_len"], args["num_q_heads"], args["ws"],
                                      args["ws_bytes"])
    return st, h


@pytest.mark.parametrize("kw,status", [
    (dict(page_size=8), ak.ATLAS_ERR_UNSUPPORTED),
    (dict(page_size=24), ak.ATLAS_ERR_UNSUPPORTED),
    (dict(head_dim=96), ak.ATLAS_ERR_UNSUPPORTED),
    (dict(num_pages=0), ak.ATLAS_ERR_INVALID_ARG),
    (dict(num_q_heads=7), ak.ATLAS_ERR_INVALID_ARG),
    (dict(k=None), ak.ATLAS_ERR_INVALID_ARG),
    (dict(ws=None), ak.ATLAS_ERR_INVALID_ARG),
    (dict(ws_bytes=16), ak.ATLAS_ERR_WORKSPACE),
    (dict(k=ctypes.c_void_p(F.ptr.value + 8)), ak.ATLAS_ERR_INVALID_ARG),
])
def test_pool_create_rejects(kw, status):
    st, h = _create(**kw)
    assert st == status and not h.value


def test_pool_create_ok_and_plan_is_host_only():
    st, h = _create()
    assert st == ak.ATLAS_OK and h.value
    try:
        buf = (ctypes.c_int32 * 7)()
        assert ak._lib.atlas_paged_gqa_decode_plan(h, 2, 8, 1, 100, buf, 7) == ak.ATLAS_OK
        plan = dict(zip(ak.PLAN_FIELDS, buf))
        # grid partition: 2 x 2 segments of 4 rows, one split of 256 tokens each
        # (the smallest automatic split) for max_seq_len 100
        assert plan["kernel"] == 1 and plan["split_tokens"] == 256 and plan["num_splits"] == 1
        assert plan["grid_ctas"] == 4
        assert plan["rows_per_cta"] == 4 and plan["row_blocks"] == 1 and plan["launches"] == 1
        assert ak._lib.atlas_paged_gqa_decode_plan(h, 2, 8, 5, 100, buf, 7) == ak.ATLAS_OK
        assert buf[3] == 32 and buf[4] == 1           # 5 x 4 rows: two warps of 16 share K/V
        assert ak._lib.atlas_kv_pool_set_split_tokens(h, 128) == ak.ATLAS_OK
        assert ak._lib.atlas_paged_gqa_decode_plan(h, 2, 8, 1, 1000, buf, 7) == ak.ATLAS_OK
        # grid: 1000 tokens in splits of 128 -> 8 splits x 4 segments
        assert buf[0] == 128 and buf[1] == 8 and buf[2] == 1 and buf[6] == 32
        # balanced: 4 segments x 32 units in ranges of 4 units: 32 CTAs; a
        # segment meets at most 9 of them
        assert ak._lib.atlas_kv_pool_set_option(h, ak.OPT_PARTITION, 2) == ak.ATLAS_OK
        assert ak._lib.atlas_paged_gqa_decode_plan(h, 2, 8, 1, 1000, buf, 7) == ak.ATLAS_OK
        assert buf[0] == 128 and buf[1] == 9 and buf[2] == 2 and buf[6] == 32
        for bad in (-1, 3):
            assert ak._lib.atlas_kv_pool_set_option(h, ak.OPT_PARTITION, bad) == ak.ATLAS_ERR_INVALID_ARG
        assert ak._lib.atlas_kv_pool_set_option(h, ak.OPT_PARTITION, 0) == ak.ATLAS_OK
        for bad in (-64, 32, 100, 16384):
            assert ak._lib.atlas_kv_pool_set_split_tokens(h, bad) == ak.ATLAS_ERR_INVALID_ARG
        for opt, val, st in ((ak.OPT_STAGES, 3, 0), (ak.OPT_STAGES, 2, 0), (ak.OPT_STAGES, 0, 0),
                             (ak.OPT_STAGES, 4, -1), (ak.OPT_SPLIT_TOKENS, 256, 0), (99, 1, -1),
                             (ak.OPT_WAIT_LIMIT_US, 1000, 0), (ak.OPT_WAIT_LIMIT_US, 0, 0),
                             (ak.OPT_WAIT_LIMIT_US, -1, -1), (ak.OPT_WAIT_LIMIT_US, 10**8, -1),
                             (ak.OPT_TEST_SKIP_UNIT, 3, 0), (ak.OPT_TEST_SKIP_UNIT, -1, 0),
                             (ak.OPT_TEST_SKIP_UNIT, -2, -1)):
            assert ak._lib.atlas_kv_pool_set_option(h, opt, val) == st
        assert ak._lib.atlas_paged_gqa_decode_plan(h, 5, 8, 1, 100, buf, 7) == ak.ATLAS_ERR_INVALID_ARG
        assert ak._lib.atlas_paged_gqa_decode_plan(h, 2, 8, 6, 100, buf, 7) == ak.ATLAS_ERR_INVALID_ARG
    finally:
        assert ak._lib.atlas_kv_pool_destroy(h) == ak.ATLAS_OK


def _decode(h, **kw):
    a = dict(q=F.ptr, kp=F.ptr, vp=F.ptr, ks=F.ptr, vs=F.ptr, bt=F.ptr, max_blocks=8,
             sl=F.ptr, batch=2, hq=8, q_len=1, max_seq=100, sm=0.0, out=F.ptr)
    a.update(kw)
    return ak._lib.atlas_paged_gqa_decode(h, a["q"], a["kp"], a["vp"], a["ks"], a["vs"], a["bt"],
                                          a["max_blocks"], a["sl"], a["batch"], a["hq"],
                                          a["q_len"], a["max_seq"], a["sm"], a["out"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), ak.ATLAS_ERR_INVALID_ARG),
    (dict(out=None), ak.ATLAS_ERR_INVALID_ARG),
    (dict(bt=None), ak.ATLAS_ERR_INVALID_ARG),
    (dict(sl=None), ak.ATLAS_ERR_INVALID_ARG),
    (dict(q_len=0), ak.ATLAS_ERR_INVALID_ARG),
    (dict(q_len=6), ak.ATLAS_ERR_INVALID_ARG),              # > max_q_len
    (dict(hq=7), ak.ATLAS_ERR_INVALID_ARG),                 # not a multiple of Hkv
    (dict(batch=-1), ak.ATLAS_ERR_INVALID_ARG),
    (dict(batch=5), ak.ATLAS_ERR_INVALID_ARG),              # > max_batch
    (dict(max_seq=129), ak.ATLAS_ERR_INVALID_ARG),          # > max_blocks * page_size
    (dict(max_blocks=0), ak.ATLAS_ERR_INVALID_ARG),
    (dict(q_len=3, max_seq=2), ak.ATLAS_ERR_INVALID_ARG),   # max_seq_len < q_len
    (dict(sm=float("nan")), ak.ATLAS_ERR_INVALID_ARG),
    (dict(q=ctypes.c_void_p(F.ptr.value + 2)), ak.ATLAS_ERR_INVALID_ARG),
])
def test_decode_rejects_before_launch(kw, status):
    st, h = _create()
    try:
        assert _decode(h, **kw) == status
    finally:
        ak._lib.atlas_kv_pool_destroy(h)


def test_decode_and_append_empty_batch_are_noops():
    st, h = _create()
    try:
        assert _decode(h, batch=0, q=None, out=None) == ak.ATLAS_OK
        assert ak._lib.atlas_fp8_kv_append(h, None, None, 0, None, 4, None, 0, 3, None) == ak.ATLAS_OK
        assert ak._lib.atlas_fp8_kv_append(h, None, None, 0, None, 4, None, 2, 0, None) == ak.ATLAS_OK
    finally:
        ak._lib.atlas_kv_pool_destroy(h)


@pytest.mark.parametrize("args,status", [
    (dict(k=None), ak.ATLAS_ERR_INVALID_ARG),
    (dict(dtype=7), ak.ATLAS_ERR_INVALID_ARG),
    (dict(max_blocks=0), ak.ATLAS_ERR_INVALID_ARG),
    (dict(n_new=-1), ak.ATLAS_ERR_INVALID_ARG),
    (dict(k=ctypes.c_void_p(F.ptr.value + 4)), ak.ATLAS_ERR_INVALID_ARG),
])
def test_append_rejects_before_launch(args, status):
    st, h = _create()
    a = dict(k=F.ptr, v=F.ptr, dtype=0, bt=F.ptr, max_blocks=4, sp=F.ptr, batch=2, n_new=3)
    a.update(args)
    try:
        assert ak._lib.atlas_fp8_kv_append(h, a["k"], a["v"], a["dtype"], a["bt"], a["max_blocks"],
                                           a["sp"], a["batch"], a["n_new"], None) == status
    finally:
        ak._lib.atlas_kv_pool_destroy(h)


def test_null_pool_is_rejected_everywhere():
    buf = (ctypes.c_int32 * 7)()
    code = ctypes.c_int32()
    assert ak._lib.atlas_paged_gqa_decode_plan(None, 1, 8, 1, 10, buf, 7) == ak.ATLAS_ERR_INVALID_ARG
    assert ak._lib.atlas_get_device_error(None, None, ctypes.byref(code)) == ak.ATLAS_ERR_INVALID_ARG
    assert ak._lib.atlas_kv_pool_set_split_tokens(None, 0) == ak.ATLAS_ERR_INVALID_ARG
    assert ak._lib.atlas_kv_pool_destroy(None) == ak.ATLAS_OK
    assert _decode(None) == ak.ATLAS_ERR_INVALID_ARG


def _plan_on_148_sms(B, Hq, Hkv, D, ps, q_len, max_seq_len, P=1024):
    h = ctypes.c_void_p()
    p = F.ptr
    st = ak._lib.atlas_kv_pool_create(ctypes.byref(h), P, ps, Hkv, D, p, p, p, p, B, q_len, Hq,
                                      p, ctypes.c_size_t(1 << 40))
    assert st == ak.ATLAS_OK
    try:
        buf = (ctypes.c_int32 * 7)()
        assert ak._lib.atlas_paged_gqa_decode_plan(h, B, Hq, q_len, max_seq_len, buf, 7) == 0
        return dict(zip(ak.PLAN_FIELDS, buf))
    finally:
        ak._lib.atlas_kv_pool_destroy(h)


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="plans for a 148-SM part")
@pytest.mark.parametrize("shape,want", [
    # LLaMA-3-8B decode: 256 segments of 4 rows; two waves would need 1024-token
    # splits, under the 2048-token floor that one wave allows -> 2048, 512 CTAs
    ((32, 32, 8, 128, 16, 1, 4096), dict(kernel=1, split_tokens=2048, grid_ctas=512, rows_per_cta=4)),
    # long context: 32 segments; two waves -> 4736 tokens, rounded down to 4096
    ((4, 32, 8, 128, 16, 1, 131072), dict(kernel=1, split_tokens=4096, num_splits=32, grid_ctas=1024)),
    # MTP verify, 25 rows per KV head: the tensor-core kernel; 1024 segments of
    # one 64-row block already fill the GPU -> one split of the whole length
    ((128, 40, 8, 128, 16, 5, 1152), dict(kernel=3, split_tokens=1152, grid_ctas=1024, rows_per_cta=64)),
    # MQA with 64 rows: the tensor-core kernel; two waves of 296 CTA slots over
    # 256 segments -> 2816 tokens, rounded down to 2048: 4 splits
    ((256, 64, 1, 128, 64, 1, 8192), dict(kernel=3, split_tokens=2048, num_splits=4, grid_ctas=1024,
                                          rows_per_cta=64)),
])
def test_automatic_plan_of_the_named_shapes(shape, want):
    plan = _plan_on_148_sms(*shape)
    for k, v in want.items():
        assert plan[k] == v, (k, plan)
