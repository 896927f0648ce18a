"""Thin ctypes binding of ``libatlas_kv.so`` (see ``include/atlas_kv.h``).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  torch is used for device memory and the current stream.  The
library must have been built (``python -m paged_fp8_kv_05_b200.build``);
importing this module raises if it is missing -- there is no fallback.
"""

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libatlas_kv.so")

ATLAS_OK = 0
ATLAS_ERR_INVALID_ARG = -1
ATLAS_ERR_UNSUPPORTED = -2
ATLAS_ERR_WORKSPACE = -3
ATLAS_ERR_CUDA = -4
ATLAS_ERR_DEVICE_CHECK = -5
ATLAS_DTYPE_F32 = 0
ATLAS_DTYPE_BF16 = 1
DEVERR_PAGE_ID = 0x1
DEVERR_SEQ_LEN = 0x2
DEVERR_APPEND = 0x4
DEVERR_TIMEOUT = 0x8
OPT_SPLIT_TOKENS = 1
OPT_STAGES = 2
OPT_WAVES = 3
OPT_PARTITION = 4
OPT_ROWS_PER_CTA = 5
OPT_WAIT_LIMIT_US = 6
OPT_TEST_SKIP_UNIT = 7
OPT_KERNEL = 8
KERNEL_AUTO, KERNEL_WARP_MMA, KERNEL_TC = 0, 1, 2
PLAN_FIELDS = ("split_tokens", "num_splits", "kernel", "rows_per_cta", "row_blocks",
               "launches", "grid_ctas")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m paged_fp8_kv_05_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

_c_i32 = ctypes.c_int32
_c_ptr = ctypes.c_void_p
_c_size = ctypes.c_size_t

# (name, restype, argtypes) -- the exported C ABI
_SIGNATURES = [
    ("atlas_version", ctypes.c_char_p, []),
    ("atlas_status_string", ctypes.c_char_p, [ctypes.c_int]),
    ("atlas_kv_workspace_bytes", _c_size, [_c_i32] * 7),
    ("atlas_kv_pool_create", ctypes.c_int,
     [ctypes.POINTER(_c_ptr), _c_i32, _c_i32, _c_i32, _c_i32, _c_ptr, _c_ptr, _c_ptr, _c_ptr,
      _c_i32, _c_i32, _c_i32, _c_ptr, _c_size]),
    ("atlas_kv_pool_destroy", ctypes.c_int, [_c_ptr]),
    ("atlas_kv_pool_set_split_tokens", ctypes.c_int, [_c_ptr, _c_i32]),
    ("atlas_kv_pool_set_option", ctypes.c_int, [_c_ptr, _c_i32, _c_i32]),
    ("atlas_fp8_kv_append", ctypes.c_int,
     [_c_ptr, _c_ptr, _c_ptr, _c_i32, _c_ptr, _c_i32, _c_ptr, _c_i32, _c_i32, _c_ptr]),
    ("atlas_paged_gqa_decode", ctypes.c_int,
     [_c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_i32, _c_ptr, _c_i32, _c_i32,
      _c_i32, _c_i32, ctypes.c_float, _c_ptr, _c_ptr]),
    ("atlas_paged_gqa_append_decode", ctypes.c_int,
     [_c_ptr, _c_ptr, _c_ptr, _c_i32, _c_ptr, _c_ptr, _c_i32, _c_ptr, _c_i32, _c_i32, _c_i32,
      _c_i32, ctypes.c_float, _c_ptr, _c_ptr]),
    ("atlas_paged_gqa_decode_noalloc", ctypes.c_int,
     [_c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_i32, _c_ptr, _c_i32, _c_i32, _c_i32,
      _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, ctypes.c_float, _c_ptr, _c_ptr]),
    ("atlas_paged_gqa_decode_plan", ctypes.c_int,
     [_c_ptr, _c_i32, _c_i32, _c_i32, _c_i32, ctypes.POINTER(_c_i32), _c_i32]),
    ("atlas_fp8_kv_append_tokscale", ctypes.c_int,
     [_c_ptr, _c_ptr, _c_ptr, _c_i32, _c_ptr, _c_i32, _c_ptr, _c_i32, _c_i32, _c_ptr, _c_ptr,
      _c_ptr, _c_ptr]),
    ("atlas_paged_gqa_decode_tokscale", ctypes.c_int,
     [_c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_i32, _c_ptr, _c_i32, _c_i32, _c_i32,
      _c_i32, ctypes.c_float, _c_ptr, _c_ptr]),
    ("atlas_paged_gqa_decode_varlen", ctypes.c_int,
     [_c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_i32, _c_ptr, _c_i32,
      _c_i32, _c_i32, _c_i32, ctypes.c_float, _c_ptr, _c_ptr]),
    ("atlas_rope_fp8_kv_append", ctypes.c_int,
     [_c_ptr, _c_ptr, _c_i32, _c_ptr, _c_i32, _c_ptr, _c_i32, _c_ptr, _c_i32, _c_i32, _c_ptr,
      _c_ptr]),
    ("atlas_mtp_greedy_accept", ctypes.c_int,
     [_c_ptr, _c_ptr, _c_i32, _c_i32, _c_i32, _c_i32, _c_ptr, _c_ptr, _c_ptr, _c_ptr, _c_ptr]),
    ("atlas_get_device_error", ctypes.c_int, [_c_ptr, _c_ptr, ctypes.POINTER(_c_i32)]),
]
for _name, _res, _args in _SIGNATURES:
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(n for n, _, _ in _SIGNATURES)


class AtlasError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def status_string(status: int) -> str:
    return _lib.atlas_status_string(status).decode()


def version() -> str:
    return _lib.atlas_version().decode()


def _check(status, what):
    if status != ATLAS_OK:
        raise AtlasError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def atlas_kv_workspace_bytes(max_batch, max_q_len, num_q_heads, num_kv_heads, head_dim,
                             max_seq_len, min_split_tokens=256) -> int:
    return int(_lib.atlas_kv_workspace_bytes(max_batch, max_q_len, num_q_heads, num_kv_heads,
                                             head_dim, max_seq_len, min_split_tokens))


class KVPool:
    """A page pool (K and V page arrays, per-head scales, decode workspace).

    ``atlas_kv_pool_create`` on caller-owned torch buffers; the buffers live
    as long as this object.  ``k_pages`` is uint8
    ``[num_pages, num_kv_heads, page_size, head_dim]`` (token-major; with
    head_dim 128 the 16-byte chunk j of slot s sits at chunk j ^ (s % 8)) and
    ``v_pages`` uint8 ``[num_pages, num_kv_heads, page_size // 16, head_dim, 16]``
    (16-slot groups, head-dim-major inside a group).
    """

    def __init__(self, num_pages, page_size, num_kv_heads, head_dim, k_scale, v_scale, *,
                 max_batch, max_q_len, num_q_heads, max_seq_len, device="cuda",
                 min_split_tokens=256, k_pages=None, v_pages=None, fill=None):
        dev = torch.device(device)
        kshape = (num_pages, num_kv_heads, page_size, head_dim)   # token-major
        vshape = (num_pages, num_kv_heads, page_size // 16, head_dim, 16)   # 16-slot groups
        self.k_pages = k_pages if k_pages is not None else torch.empty(kshape, dtype=torch.uint8, device=dev)
        self.v_pages = v_pages if v_pages is not None else torch.empty(vshape, dtype=torch.uint8, device=dev)
        if fill is not None:
            self.k_pages.fill_(fill)
            self.v_pages.fill_(fill)
        self.k_scale = torch.as_tensor(k_scale, dtype=torch.float32).to(dev).contiguous()
        self.v_scale = torch.as_tensor(v_scale, dtype=torch.float32).to(dev).contiguous()
        nbytes = atlas_kv_workspace_bytes(max_batch, max_q_len, num_q_heads, num_kv_heads,
                                          head_dim, max_seq_len, min_split_tokens)
        if nbytes == 0:
            raise AtlasError(ATLAS_ERR_INVALID_ARG, "atlas_kv_workspace_bytes")
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        self.num_pages, self.page_size = num_pages, page_size
        self.num_kv_heads, self.head_dim = num_kv_heads, head_dim
        self.num_q_heads = num_q_heads
        h = ctypes.c_void_p()
        _check(_lib.atlas_kv_pool_create(ctypes.byref(h), num_pages, page_size, num_kv_heads,
                                         head_dim, _ptr(self.k_pages), _ptr(self.v_pages),
                                         _ptr(self.k_scale), _ptr(self.v_scale), max_batch,
                                         max_q_len, num_q_heads, _ptr(self.workspace),
                                         nbytes), "atlas_kv_pool_create")
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            _lib.atlas_kv_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_split_tokens(self, tokens: int):
        _check(_lib.atlas_kv_pool_set_split_tokens(self.handle, tokens),
               "atlas_kv_pool_set_split_tokens")

    def set_option(self, option: int, value: int):
        _check(_lib.atlas_kv_pool_set_option(self.handle, option, value),
               "atlas_kv_pool_set_option")

    def device_error(self, stream=None) -> int:
        code = _c_i32(0)
        st = _lib.atlas_get_device_error(self.handle, _stream(stream), ctypes.byref(code))
        if st not in (ATLAS_OK, ATLAS_ERR_DEVICE_CHECK):
            _check(st, "atlas_get_device_error")
        return int(code.value)


def atlas_fp8_kv_append(pool: KVPool, k_new, v_new, block_table, start_pos, stream=None):
    """Quantise ``k_new``/``v_new`` (``[B, n_new, Hkv, D]`` float32 or bf16) and
    write them at positions ``start_pos[b] + t``."""
    assert k_new.shape == v_new.shape and k_new.dtype == v_new.dtype
    assert k_new.is_contiguous() and v_new.is_contiguous() and block_table.is_contiguous()
    dtype = {torch.float32: ATLAS_DTYPE_F32, torch.bfloat16: ATLAS_DTYPE_BF16}[k_new.dtype]
    B, n_new = int(k_new.shape[0]), int(k_new.shape[1])
    _check(_lib.atlas_fp8_kv_append(pool.handle, _ptr(k_new), _ptr(v_new), dtype,
                                    _ptr(block_table), int(block_table.shape[1]),
                                    _ptr(start_pos), B, n_new, _stream(stream)),
           "atlas_fp8_kv_append")


def atlas_paged_gqa_decode(pool: KVPool, q, block_table, seq_lens, max_seq_len, out=None,
                           sm_scale=0.0, k_pages=None, v_pages=None, k_scale=None,
                           v_scale=None, stream=None):
    """Decode / MTP-verify attention.  ``q``: bf16 ``[B, q_len, Hq, D]``;
    returns ``out`` (bf16, same shape)."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous() and block_table.is_contiguous()
    B, q_len, Hq, D = (int(x) for x in q.shape)
    if out is None:
        out = torch.empty_like(q)
    kp = pool.k_pages if k_pages is None else k_pages
    vp = pool.v_pages if v_pages is None else v_pages
    ks = pool.k_scale if k_scale is None else k_scale
    vs = pool.v_scale if v_scale is None else v_scale
    _check(_lib.atlas_paged_gqa_decode(pool.handle, _ptr(q), _ptr(kp), _ptr(vp), _ptr(ks),
                                       _ptr(vs), _ptr(block_table), int(block_table.shape[1]),
                                       _ptr(seq_lens), B, Hq, q_len, int(max_seq_len),
                                       float(sm_scale), _ptr(out), _stream(stream)),
           "atlas_paged_gqa_decode")
    return out


def atlas_paged_gqa_append_decode(pool: KVPool, k_new, v_new, q, block_table, seq_lens,
                                  max_seq_len, out=None, sm_scale=0.0, stream=None):
    """One fused step: append the q_len new tokens (``k_new``/``v_new``
    ``[B, q_len, Hkv, D]`` f32 or bf16) at positions ``seq_lens - q_len`` and
    decode.  Returns ``out`` (bf16 ``[B, q_len, Hq, D]``)."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous() and block_table.is_contiguous()
    assert k_new.shape == v_new.shape and k_new.dtype == v_new.dtype
    assert k_new.is_contiguous() and v_new.is_contiguous()
    dtype = {torch.float32: ATLAS_DTYPE_F32, torch.bfloat16: ATLAS_DTYPE_BF16}[k_new.dtype]
    B, q_len, Hq, D = (int(x) for x in q.shape)
    if out is None:
        out = torch.empty_like(q)
    _check(_lib.atlas_paged_gqa_append_decode(pool.handle, _ptr(k_new), _ptr(v_new), dtype,
                                              _ptr(q), _ptr(block_table),
                                              int(block_table.shape[1]), _ptr(seq_lens), B, Hq,
                                              q_len, int(max_seq_len), float(sm_scale),
                                              _ptr(out), _stream(stream)),
           "atlas_paged_gqa_append_decode")
    return out


def atlas_paged_gqa_decode_noalloc(q, k_pages, v_pages, k_scale, v_scale, block_table,
                                   seq_lens, max_seq_len, out=None, sm_scale=0.0, stream=None):
    """The no-allocation decode entry point (scratch in the library's static
    device array).  Page arrays as in :class:`KVPool`; ``q``/``out`` bf16
    ``[B, q_len, Hq, D]``."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous() and block_table.is_contiguous()
    B, q_len, Hq, D = (int(x) for x in q.shape)
    P, Hkv, ps, Dk = (int(x) for x in k_pages.shape)
    assert Dk == D
    if out is None:
        out = torch.empty_like(q)
    _check(_lib.atlas_paged_gqa_decode_noalloc(_ptr(q), _ptr(k_pages), _ptr(v_pages),
                                               _ptr(k_scale), _ptr(v_scale), _ptr(block_table),
                                               int(block_table.shape[1]), _ptr(seq_lens), B, Hq,
                                               Hkv, D, ps, P, q_len, int(max_seq_len),
                                               float(sm_scale), _ptr(out), _stream(stream)),
           "atlas_paged_gqa_decode_noalloc")
    return out


class TokenScales:
    """Per-(token, KV head) scale arrays of a pool in the finer-grained mode:
    ``k``, ``v`` float32 ``[num_pages, num_kv_heads, page_size]`` and the
    per-head V bound ``v_bound`` float32 ``[num_kv_heads]`` (zero-filled)."""

    def __init__(self, pool: KVPool):
        dev = pool.k_pages.device
        shape = (pool.num_pages, pool.num_kv_heads, pool.page_size)
        self.k = torch.zeros(shape, dtype=torch.float32, device=dev)
        self.v = torch.zeros(shape, dtype=torch.float32, device=dev)
        self.v_bound = torch.zeros(pool.num_kv_heads, dtype=torch.float32, device=dev)


def atlas_fp8_kv_append_tokscale(pool: KVPool, scales: TokenScales, k_new, v_new, block_table,
                                 start_pos, stream=None):
    """Append with one dynamic scale per (token, KV head) into ``scales``."""
    assert k_new.shape == v_new.shape and k_new.dtype == v_new.dtype
    assert k_new.is_contiguous() and v_new.is_contiguous() and block_table.is_contiguous()
    dtype = {torch.float32: ATLAS_DTYPE_F32, torch.bfloat16: ATLAS_DTYPE_BF16}[k_new.dtype]
    B, n_new = int(k_new.shape[0]), int(k_new.shape[1])
    _check(_lib.atlas_fp8_kv_append_tokscale(pool.handle, _ptr(k_new), _ptr(v_new), dtype,
                                             _ptr(block_table), int(block_table.shape[1]),
                                             _ptr(start_pos), B, n_new, _ptr(scales.k),
                                             _ptr(scales.v), _ptr(scales.v_bound),
                                             _stream(stream)),
           "atlas_fp8_kv_append_tokscale")


def atlas_paged_gqa_decode_tokscale(pool: KVPool, scales: TokenScales, q, block_table, seq_lens,
                                    max_seq_len, out=None, sm_scale=0.0, stream=None):
    """Decode / verify over a cache with per-(token, KV head) scales."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous() and block_table.is_contiguous()
    B, q_len, Hq, D = (int(x) for x in q.shape)
    if out is None:
        out = torch.empty_like(q)
    _check(_lib.atlas_paged_gqa_decode_tokscale(pool.handle, _ptr(q), _ptr(scales.k),
                                                _ptr(scales.v), _ptr(scales.v_bound),
                                                _ptr(block_table), int(block_table.shape[1]),
                                                _ptr(seq_lens), B, Hq, q_len, int(max_seq_len),
                                                float(sm_scale), _ptr(out), _stream(stream)),
           "atlas_paged_gqa_decode_tokscale")
    return out


def atlas_paged_gqa_decode_varlen(pool: KVPool, q, cu_q_lens, block_table, seq_lens,
                                  max_q_len, max_seq_len, out=None, sm_scale=0.0, k_pages=None,
                                  v_pages=None, k_scale=None, v_scale=None, stream=None):
    """Ragged verify / chunked prefill.  ``q``: bf16 ``[total_rows, Hq, D]``
    packed by ``cu_q_lens`` (int32 ``[B + 1]``); returns ``out`` (same shape)."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous() and q.dim() == 3
    assert cu_q_lens.dtype == torch.int32 and block_table.is_contiguous()
    B = int(cu_q_lens.shape[0]) - 1
    Hq = int(q.shape[1])
    if out is None:
        out = torch.empty_like(q)
    kp = pool.k_pages if k_pages is None else k_pages
    vp = pool.v_pages if v_pages is None else v_pages
    ks = pool.k_scale if k_scale is None else k_scale
    vs = pool.v_scale if v_scale is None else v_scale
    _check(_lib.atlas_paged_gqa_decode_varlen(pool.handle, _ptr(q), _ptr(cu_q_lens), _ptr(kp),
                                              _ptr(vp), _ptr(ks), _ptr(vs), _ptr(block_table),
                                              int(block_table.shape[1]), _ptr(seq_lens), B, Hq,
                                              int(max_q_len), int(max_seq_len), float(sm_scale),
                                              _ptr(out), _stream(stream)),
           "atlas_paged_gqa_decode_varlen")
    return out


def atlas_rope_fp8_kv_append(pool: KVPool, qkv, num_q_heads, cos_sin, block_table, start_pos,
                             q_out=None, stream=None):
    """Rotate Q and K of the new tokens, quantise and append K and V.
    ``qkv``: bf16 ``[B, n_new, Hq + 2 Hkv, D]``; ``cos_sin``: float32
    ``[max_pos, D]``.  Returns the rotated queries ``q_out`` (bf16
    ``[B, n_new, Hq, D]``)."""
    assert qkv.dtype == torch.bfloat16 and qkv.is_contiguous() and cos_sin.is_contiguous()
    assert cos_sin.dtype == torch.float32 and block_table.is_contiguous()
    B, n_new, heads, D = (int(x) for x in qkv.shape)
    if q_out is None:
        q_out = torch.empty(B, n_new, num_q_heads, D, dtype=torch.bfloat16, device=qkv.device)
    _check(_lib.atlas_rope_fp8_kv_append(pool.handle, _ptr(qkv), num_q_heads, _ptr(cos_sin),
                                         int(cos_sin.shape[0]), _ptr(block_table),
                                         int(block_table.shape[1]), _ptr(start_pos), B, n_new,
                                         _ptr(q_out), _stream(stream)),
           "atlas_rope_fp8_kv_append")
    return q_out


def atlas_mtp_greedy_accept(pool: KVPool, logits, drafts, targets=None, n_accepted=None,
                            next_token=None, stream=None):
    """Greedy MTP acceptance.  ``logits``: ``[B, K + 1, V]`` float32 or bf16;
    ``drafts``: int32 ``[B, K]``.  Returns ``(n_accepted [B], next_token [B],
    targets [B, K + 1])`` (int32 device tensors)."""
    assert logits.dim() == 3 and logits.is_contiguous() and drafts.is_contiguous()
    B, K1, V = (int(x) for x in logits.shape)
    assert tuple(drafts.shape) == (B, K1 - 1) and drafts.dtype == torch.int32
    dtype = {torch.float32: ATLAS_DTYPE_F32, torch.bfloat16: ATLAS_DTYPE_BF16}[logits.dtype]
    dev = logits.device
    if targets is None:
        targets = torch.empty(B, K1, dtype=torch.int32, device=dev)
    if n_accepted is None:
        n_accepted = torch.empty(B, dtype=torch.int32, device=dev)
    if next_token is None:
        next_token = torch.empty(B, dtype=torch.int32, device=dev)
    _check(_lib.atlas_mtp_greedy_accept(pool.handle, _ptr(logits), dtype, B, K1 - 1, V,
                                        _ptr(drafts), _ptr(targets), _ptr(n_accepted),
                                        _ptr(next_token), _stream(stream)),
           "atlas_mtp_greedy_accept")
    return n_accepted, next_token, targets


def atlas_paged_gqa_decode_plan(pool: KVPool, batch, num_q_heads, q_len, max_seq_len) -> dict:
    buf = (_c_i32 * len(PLAN_FIELDS))()
    _check(_lib.atlas_paged_gqa_decode_plan(pool.handle, batch, num_q_heads, q_len, max_seq_len,
                                            buf, len(PLAN_FIELDS)),
           "atlas_paged_gqa_decode_plan")
    return dict(zip(PLAN_FIELDS, (int(x) for x in buf)))


def default_sm_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
