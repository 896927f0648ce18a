"""CPU oracle for the paged FP8 KV decode / MTP-verify attention path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, table or constant generator with the CUDA library, and it never
takes an input or an expected value from the CUDA path.

What it computes, and where the sources say so:

* ``e4m3``  -- the OCP OFP8 E4M3 ("FN") code: decode of all 256 codes and
  round-to-nearest-even, saturating encode of ``fp32(x) / fp32(scale)``.
  The Atlas pages only say "FP8 with per-group scales" (Atlas deep-dive,
  ainews.cool, "Quantisation" paragraph) and "paged FP8 KV cache" (Atlas vs
  vLLM on a single GB10, ainews.surl.tw, deployment-path paragraph); the bit
  format is the public OCP definition.
* ``paged``  -- the paged cache: the page-append scatter (token position p of
  sequence b lands in page ``block_table[b][p // ps]``, slot ``p % ps``) and
  the contiguous re-assembly of a sequence's K/V from its pages.  The
  fixed-size-block pool is the memory design of the Atlas deep-dive
  ("Memory architecture" paragraph).
* ``attention`` -- plain masked scaled-dot-product attention in float64 over
  the re-assembled, dequantised K/V, with grouped-query head sharing and the
  MTP-verify causal mask among the q_len new rows (Atlas deep-dive,
  "Attention" paragraph: dedicated MQA/GQA kernels; GB10 page: MTP with
  K = 4 drafts).

* ``acceptance`` -- greedy acceptance of MTP draft tokens: the target's
  choice at each new position is the first maximum of the verify logits;
  leading drafts equal to it are accepted, and the target at the first
  position not covered is emitted (GB10 page: MTP with K = 4; the
  speculative-decoding fusion page, blog.hotdry.top: the draft -> verify ->
  accept loop).

Every function is pinned by ``tests/test_oracle_*.py`` against something
other than itself (closed forms, brute force, invariants, torch's own
float8 and SDPA routines).  No function here is "parity unpinned".
"""

from . import e4m3, paged, attention, acceptance  # noqa: F401
