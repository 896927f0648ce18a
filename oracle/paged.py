"""The paged FP8 KV cache, as plain array indexing.  Test infrastructure only.

Layout (the pages give none; this is the reading the whole build uses):
pages are ``uint8[P, Hkv, ps, D]`` -- physical page, KV head, slot in page,
head dimension.  Token position ``p`` of sequence ``b`` lives in physical page
``block_table[b, p // ps]`` at slot ``p % ps``.  The block table is the
fixed-size-block pool of the Atlas deep-dive (ainews.cool, "Memory
architecture" paragraph: KV blocks preallocated in fixed sizes); the FP8 codes
are those of the GB10 page's "paged FP8 KV cache" (ainews.surl.tw).

The only place the layout is spelled out is :func:`slot_of`; everything else
goes through it, so another layout would change that one function.
"""

import numpy as np

from . import e4m3


def slot_of(block_table, b: int, pos: int, page_size: int):
    """(physical page, slot) of token position ``pos`` of sequence ``b``."""
    return int(block_table[b, pos // page_size]), pos % page_size


def append(pages, new, scale, block_table, start_pos, page_size):
    """Return a copy of ``pages`` with the new tokens quantised and written.

    ``new``: float32 ``[B, n_new, Hkv, D]`` (bf16 inputs are passed as their
    exact float32 values); ``scale``: float32 ``[Hkv]``; ``start_pos[b]`` is the
    position of the first new token of sequence b.  Element (b, t, h, d) is
    encoded as ``E4M3(fp32(x) / fp32(scale[h]))`` and stored at
    ``pages[page, h, slot, d]`` with ``(page, slot) = slot_of(b, start_pos[b] + t)``.
    """
    out = np.array(pages, dtype=np.uint8, copy=True)
    new = np.asarray(new, dtype=np.float32)
    scale = np.asarray(scale, dtype=np.float32)
    B, n_new = new.shape[0], new.shape[1]
    for b in range(B):
        for t in range(n_new):
            page, slot = slot_of(block_table, b, int(start_pos[b]) + t, page_size)
            out[page, :, slot, :] = e4m3.encode(new[b, t], scale[:, None])
    return out


def gather_codes(pages, block_table, b: int, length: int, page_size: int):
    """Contiguous codes ``uint8[length, Hkv, D]`` of sequence ``b``'s first
    ``length`` tokens, re-assembled page by page."""
    pages = np.asarray(pages)
    n_pages = (length + page_size - 1) // page_size
    ids = np.asarray(block_table[b, :n_pages], dtype=np.int64)
    blocks = pages[ids]                       # [n_pages, Hkv, ps, D]
    seq = blocks.transpose(0, 2, 1, 3)        # [n_pages, ps, Hkv, D]
    seq = seq.reshape(n_pages * page_size, pages.shape[1], pages.shape[3])
    return seq[:length]


def gather_dequant(pages, scale, block_table, b: int, length: int, page_size: int):
    """Dequantised float64 ``[length, Hkv, D]``: ``decode(code) * scale[h]``."""
    codes = gather_codes(pages, block_table, b, length, page_size)
    scale = np.asarray(scale, dtype=np.float32).astype(np.float64)
    return e4m3.decode(codes) * scale[None, :, None]
