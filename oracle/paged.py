"""The paged FP8 KV cache, as plain array indexing.  Test infrastructure only.

Layouts (the pages give none; these are the readings the whole build uses).
Token position ``p`` of sequence ``b`` lives in physical page
``block_table[b, p // ps]`` at slot ``p % ps``.  Inside a page, one of three
orders:

* ``"tok"`` (token-major): ``uint8[P, Hkv, ps, D]`` -- page, KV head, slot,
  head dimension.  The K pages use it.
* ``"grp16"`` (16-slot groups, head-dim-major inside a group):
  ``uint8[P, Hkv, ps // 16, D, 16]`` -- page, KV head, group of 16 slots,
  head dimension, byte position of the slot inside the group.  The V pages
  use it: the values of 16 consecutive tokens for one head dimension are
  adjacent bytes, and every 16-token piece of a page is one contiguous block.
  Inside a group the slots are interleaved: slot t sits at byte
  ``GROUP_POS[t] = 4*((t % 8) // 2) + 2*(t // 8) + t % 2``, so that bytes
  4c..4c+3 hold slots 2c, 2c+1, 2c+8, 2c+9.
* ``"dim"`` (head-dim-major): ``uint8[P, Hkv, D, ps]``; the same as
  ``"grp16"`` when ps = 16.
* ``"ksw"`` (token-major, chunk-permuted): ``uint8[P, Hkv, ps, 128]`` -- the
  token-major order with each token row cut into eight 16-byte chunks, and
  chunk j of slot s stored at chunk position ``j XOR (s % 8)``.  The K pages
  use it when D = 128 (the permutation is the 128-byte swizzle of the
  tensor-core operand layout, so a page copied verbatim is ready to use);
  with D = 64 K pages are plain ``"tok"``.

The block table is the fixed-size-block pool of the Atlas deep-dive
(ainews.cool, "Memory architecture" paragraph: KV blocks preallocated in
fixed sizes); the FP8 codes are those of the GB10 page's "paged FP8 KV cache"
(ainews.surl.tw).  The layouts are spelled out only in :func:`slot_of`,
:func:`ksw_chunk`, :func:`_store` and :func:`gather_codes`.
"""

import numpy as np

from . import e4m3

LAYOUTS = ("tok", "grp16", "dim", "ksw")
GROUP = 16
GROUP_POS = np.array([4 * ((t % 8) // 2) + 2 * (t // 8) + t % 2 for t in range(GROUP)])


def ksw_chunk(slot: int, j: int) -> int:
    """Chunk position of logical 16-byte chunk ``j`` of slot ``slot`` in the
    ``"ksw"`` order."""
    return j ^ (slot % 8)


def k_layout(head_dim: int) -> str:
    """In-page order of the K pages for a head dimension."""
    return "ksw" if head_dim == 128 else "tok"


def slot_of(block_table, b: int, pos: int, page_size: int):
    """(physical page, slot) of token position ``pos`` of sequence ``b``."""
    return int(block_table[b, pos // page_size]), pos % page_size


def _store(out, page, slot, codes, layout):
    """Write one token's codes ``[Hkv, D]`` into ``page`` at ``slot``."""
    if layout == "tok":
        out[page, :, slot, :] = codes
    elif layout == "grp16":
        out[page, :, slot // GROUP, :, GROUP_POS[slot % GROUP]] = codes
    elif layout == "dim":
        out[page, :, :, slot] = codes
    elif layout == "ksw":
        for j in range(8):
            c = ksw_chunk(slot, j)
            out[page, :, slot, 16 * c:16 * c + 16] = codes[:, 16 * j:16 * j + 16]
    else:
        raise ValueError(layout)


def append(pages, new, scale, block_table, start_pos, page_size, layout="tok"):
    """Return a copy of ``pages`` with the new tokens quantised and written.

    ``new``: float32 ``[B, n_new, Hkv, D]`` (bf16 inputs are passed as their
    exact float32 values); ``scale``: float32 ``[Hkv]``; ``start_pos[b]`` is the
    position of the first new token of sequence b.  Element (b, t, h, d) is
    encoded as ``E4M3(fp32(x) / fp32(scale[h]))`` and stored for token position
    ``start_pos[b] + t`` in the given page layout.
    """
    out = np.array(pages, dtype=np.uint8, copy=True)
    new = np.asarray(new, dtype=np.float32)
    scale = np.asarray(scale, dtype=np.float32)
    B, n_new = new.shape[0], new.shape[1]
    for b in range(B):
        for t in range(n_new):
            page, slot = slot_of(block_table, b, int(start_pos[b]) + t, page_size)
            _store(out, page, slot, e4m3.encode(new[b, t], scale[:, None]), layout)
    return out


def gather_codes(pages, block_table, b: int, length: int, page_size: int, layout="tok"):
    """Contiguous codes ``uint8[length, Hkv, D]`` of sequence ``b``'s first
    ``length`` tokens, re-assembled page by page."""
    pages = np.asarray(pages)
    n_pages = (length + page_size - 1) // page_size
    ids = np.asarray(block_table[b, :n_pages], dtype=np.int64)
    blocks = pages[ids]
    if layout == "tok":                       # [n_pages, Hkv, ps, D]
        seq = blocks.transpose(0, 2, 1, 3)
    elif layout == "grp16":                   # [n_pages, Hkv, ps/16, D, 16]
        blocks = blocks[..., GROUP_POS]        # byte positions -> slot order
        seq = blocks.transpose(0, 2, 4, 1, 3)  # [n_pages, ps/16, 16, Hkv, D]
        seq = seq.reshape(seq.shape[0], seq.shape[1] * GROUP, seq.shape[3], seq.shape[4])
    elif layout == "dim":                     # [n_pages, Hkv, D, ps]
        seq = blocks.transpose(0, 3, 1, 2)
    elif layout == "ksw":                     # [n_pages, Hkv, ps, 128], chunks permuted
        un = np.empty_like(blocks)
        for slot in range(blocks.shape[2]):
            for j in range(8):
                c = ksw_chunk(slot, j)
                un[:, :, slot, 16 * j:16 * j + 16] = blocks[:, :, slot, 16 * c:16 * c + 16]
        seq = un.transpose(0, 2, 1, 3)
    else:
        raise ValueError(layout)
    hkv = seq.shape[2]
    seq = seq.reshape(n_pages * page_size, hkv, seq.shape[3])
    return seq[:length]


def gather_dequant(pages, scale, block_table, b: int, length: int, page_size: int,
                   layout="tok"):
    """Dequantised float64 ``[length, Hkv, D]``: ``decode(code) * scale[h]``."""
    codes = gather_codes(pages, block_table, b, length, page_size, layout)
    scale = np.asarray(scale, dtype=np.float32).astype(np.float64)
    return e4m3.decode(codes) * scale[None, :, None]


def append_tokscale(pages, scales, new, block_table, start_pos, page_size, layout="tok"):
    """Finer-grained scales: like :func:`append`, but each new token's row of
    each KV head is quantised with its own dynamic scale (``e4m3.row_scale``),
    stored in ``scales`` float32 ``[P, Hkv, ps]`` at the token's (page, head,
    slot).  Returns ``(pages', scales')``."""
    out = np.array(pages, dtype=np.uint8, copy=True)
    sc = np.array(scales, dtype=np.float32, copy=True)
    new = np.asarray(new, dtype=np.float32)
    B, n_new = new.shape[0], new.shape[1]
    for b in range(B):
        for t in range(n_new):
            page, slot = slot_of(block_table, b, int(start_pos[b]) + t, page_size)
            codes, s = e4m3.encode_rows(new[b, t])          # [Hkv, D], [Hkv]
            _store(out, page, slot, codes, layout)
            sc[page, :, slot] = s
    return out, sc


def gather_dequant_tokscale(pages, scales, block_table, b: int, length: int, page_size: int,
                            layout="tok"):
    """Dequantised float64 ``[length, Hkv, D]`` with per-token scales:
    ``decode(code) * scales[page, h, slot]``."""
    codes = gather_codes(pages, block_table, b, length, page_size, layout)
    n_pages = (length + page_size - 1) // page_size
    ids = np.asarray(block_table[b, :n_pages], dtype=np.int64)
    s = np.asarray(scales, dtype=np.float32)[ids]                 # [n_pages, Hkv, ps]
    s = s.transpose(0, 2, 1).reshape(n_pages * page_size, -1)[:length]
    return e4m3.decode(codes) * s.astype(np.float64)[:, :, None]
