"""Rotary position embedding of the new tokens' Q and K, then the FP8 append
of K and V, as the plain definition.  Test infrastructure only.

The deep-dive page (Atlas: Rust/CUDA LLM inference engine, ainews.cool,
"Kernel fusion" paragraph) fuses the per-block steps into one kernel; the
step in front of paged decode is: take the QKV projection output of the new
tokens, rotate Q and K by their positions, quantise K and V to FP8 with the
per-KV-head scales and write them into the pages, and hand the rotated Q to
the attention.

Readings where the pages are silent:
  * layout of the projection output: per token, the Hq query heads, then the
    Hkv key heads, then the Hkv value heads, each D wide (bf16);
  * rotation convention: "rotate half" -- element i < D/2 pairs with element
    i + D/2; with c = cos[pos, i], s = sin[pos, i]
        out[i]       = x[i] * c - x[i + D/2] * s
        out[i + D/2] = x[i + D/2] * c + x[i] * s
    i.e. the complex number x[i] + j x[i + D/2] multiplied by e^(j theta);
  * the angles come as an input table cos_sin float32 [max_pos, D] (cos in
    columns 0 .. D/2 - 1, sin in D/2 .. D - 1), so both sides rotate with the
    same float32 values;
  * arithmetic: float32, each product and the sum / difference rounded to
    nearest separately (no fused multiply-add), so the rotated value -- and
    the FP8 code decided from it -- is one exact float32 number;
  * the rotated Q is handed on as bf16, rounded to nearest even.
"""

import numpy as np

from . import e4m3, paged


def rotate(x, cos, sin):
    """Rotate-half RoPE of float32 ``x`` ``[..., D]`` with float32 ``cos``,
    ``sin`` ``[..., D/2]`` (broadcast), in float32 with separately rounded
    products and sums."""
    x = np.asarray(x, dtype=np.float32)
    cos = np.asarray(cos, dtype=np.float32)
    sin = np.asarray(sin, dtype=np.float32)
    h = x.shape[-1] // 2
    x1, x2 = x[..., :h], x[..., h:]
    o1 = np.subtract(np.multiply(x1, cos, dtype=np.float32), np.multiply(x2, sin, dtype=np.float32),
                     dtype=np.float32)
    o2 = np.add(np.multiply(x2, cos, dtype=np.float32), np.multiply(x1, sin, dtype=np.float32),
                dtype=np.float32)
    return np.concatenate([o1, o2], axis=-1)


def bf16_round(x) -> np.ndarray:
    """float32 -> nearest bf16 value (ties to even), returned as float32.
    Written on the bit pattern: add 0x7FFF plus the lowest kept bit, then
    drop the low 16 bits (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    keep = (u >> 16) & 1
    r = ((u + 0x7FFF + keep) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def split_qkv(qkv, num_q_heads, num_kv_heads):
    """``[B, n_new, Hq + 2 Hkv, D]`` -> (q, k, v) views."""
    q = qkv[:, :, :num_q_heads]
    k = qkv[:, :, num_q_heads:num_q_heads + num_kv_heads]
    v = qkv[:, :, num_q_heads + num_kv_heads:]
    return q, k, v


def rope_append(k_pages, v_pages, qkv, num_q_heads, num_kv_heads, cos_sin, k_scale, v_scale,
                block_table, start_pos, page_size, k_layout="tok", v_layout="tok"):
    """Returns ``(q_out, k_pages', v_pages')``.  ``qkv``: float32 ``[B, n_new,
    Hq + 2 Hkv, D]`` (the exact bf16 values); new token t of sequence b has
    position ``start_pos[b] + t``.  q_out: float32 ``[B, n_new, Hq, D]`` holding
    bf16 values (the rotated Q rounded to bf16)."""
    qkv = np.asarray(qkv, dtype=np.float32)
    B, n_new, _, D = qkv.shape
    q, k, v = split_qkv(qkv, num_q_heads, num_kv_heads)
    pos = np.asarray(start_pos, dtype=np.int64)[:, None] + np.arange(n_new)[None, :]   # [B, n_new]
    table = np.asarray(cos_sin, dtype=np.float32)
    cos = table[pos, :D // 2][:, :, None, :]     # [B, n_new, 1, D/2]
    sin = table[pos, D // 2:][:, :, None, :]
    q_rot = rotate(q, cos, sin)
    k_rot = rotate(k, cos, sin)
    q_out = bf16_round(q_rot)
    kp = paged.append(k_pages, k_rot, k_scale, block_table, start_pos, page_size, layout=k_layout)
    vp = paged.append(v_pages, v, v_scale, block_table, start_pos, page_size, layout=v_layout)
    return q_out, kp, vp


__all__ = ["rotate", "bf16_round", "split_qkv", "rope_append", "e4m3"]
