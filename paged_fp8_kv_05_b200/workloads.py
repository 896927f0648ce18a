"""Seeded synthetic inputs for the paged FP8 decode / verify path.

This module only draws random inputs and lays them out; it holds none of the
method's arithmetic (no FP8 coding, no attention).  Both the CUDA path and the
CPU oracle take their inputs from here, so the two see identical values.

Recipe (all draws from ``numpy.random.default_rng`` on children of
``numpy.random.SeedSequence(seed)``; one child per purpose, in this order:
lengths, page table, q, k, v, outlier rows, fragmentation, sharp shaping):

* context lengths ``L_b`` per the workload (uniform integers, or
  ``floor(exp(U[ln lo, ln hi]))`` for the log-uniform mix);
* Q ``N(0, 1)`` float32, rounded to bf16 (round-to-nearest-even);
* K and V ``N(0, 1)`` float32 ``[sum L_b, Hkv, D]``; optionally a Bernoulli
  fraction of K rows (one row = one token of one KV head) multiplied by a
  factor *before* the scales are taken (outlier keys);
* optional sharp-attention shaping of the same draws, before the scales are
  taken: Q multiplied by a gain (score standard deviation = gain); "needle"
  keys, a K row replaced by a multiple of one query row of its group, at
  seeded positions (one inside the MTP drafts when q_len > 1); or a "ramp", K
  rows of one query head per KV head set to ``c_t * q`` so that its scores
  rise linearly along the context;
* per-KV-head scales ``amax_h / 448`` in float32, the amax over every token of
  the generated tensor (new tokens included): one static scale per KV head and
  tensor;
* page table: sequences take consecutive runs of a seeded permutation of the
  pool ("perm"), or pages come off a LIFO free list that was first churned by
  8 rounds of allocating phantom sequences and freeing a random half of them
  ("frag": ids reused, non-monotone, non-contiguous).  Unused table entries
  are -1.

The five named workloads are the decode shapes the Atlas pages benchmark
(LLaMA-3-8B at batch 32; a 27B-class MTP K = 4 verify at high concurrency)
plus a tiny case, a long-context case and a ragged MQA case; no dataset is
involved.
"""

from dataclasses import dataclass, field
import math

import numpy as np
import torch

FP8_MAX = 448.0

# name -> shape recipe
CONFIGS = {
    0: dict(name="tiny paged GQA decode", batch=2, num_q_heads=8, num_kv_heads=2,
            head_dim=64, page_size=16, q_len=1, num_pages=64,
            lengths=("fixed", [37, 100]), table="perm"),
    1: dict(name="LLaMA-3-8B-shaped decode layer", batch=32, num_q_heads=32,
            num_kv_heads=8, head_dim=128, page_size=16, q_len=1, num_pages=16384,
            lengths=("uniform", 1024, 4096), table="perm"),
    2: dict(name="MTP-verify on a 27B-class GQA shape", batch=128, num_q_heads=40,
            num_kv_heads=8, head_dim=128, page_size=16, q_len=5, num_pages=16384,
            lengths=("uniform", 128, 1152), table="perm"),
    3: dict(name="long-context split-KV decode", batch=4, num_q_heads=32,
            num_kv_heads=8, head_dim=128, page_size=16, q_len=1, num_pages=40960,
            lengths=("uniform", 65536, 131072), table="perm",
            outlier_frac=0.01, outlier_gain=8.0),
    4: dict(name="ragged MQA high-concurrency decode", batch=256, num_q_heads=64,
            num_kv_heads=1, head_dim=128, page_size=64, q_len=1, num_pages=40000,
            lengths=("loguniform", 256, 8192), table="frag"),
}


@dataclass
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    q_len: int
    num_pages: int
    seq_lens: np.ndarray          # int32 [B]
    block_table: np.ndarray       # int32 [B, max_blocks], -1 where unused
    q: torch.Tensor               # bf16 [B, q_len, Hq, D] (CPU)
    k: np.ndarray                 # float32 [sum L, Hkv, D]
    v: np.ndarray                 # float32 [sum L, Hkv, D]
    k_scale: np.ndarray           # float32 [Hkv]
    v_scale: np.ndarray           # float32 [Hkv]
    cu_seqlens: np.ndarray        # int64 [B + 1]
    meta: dict = field(default_factory=dict)

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max()) if self.batch else 0

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def q_f64(self) -> np.ndarray:
        return self.q.float().numpy().astype(np.float64)

    def seq_k(self, b: int) -> np.ndarray:
        return self.k[self.cu_seqlens[b]:self.cu_seqlens[b + 1]]

    def seq_v(self, b: int) -> np.ndarray:
        return self.v[self.cu_seqlens[b]:self.cu_seqlens[b + 1]]

    def new_tokens(self, which: str) -> np.ndarray:
        """float32 ``[B, q_len, Hkv, D]``: the last q_len tokens of every
        sequence (the tokens a decode / verify step appends)."""
        src = self.k if which == "k" else self.v
        idx = np.concatenate([np.arange(self.cu_seqlens[b + 1] - self.q_len,
                                        self.cu_seqlens[b + 1])
                              for b in range(self.batch)]) if self.batch else np.zeros(0, np.int64)
        return src[idx].reshape(self.batch, self.q_len, self.num_kv_heads, self.head_dim)

    def kv_bytes(self) -> int:
        """FP8 bytes of K and V over the valid tokens."""
        return int(self.seq_lens.astype(np.int64).sum()) * self.num_kv_heads * self.head_dim * 2


def _lengths(rng, spec, batch):
    kind = spec[0]
    if kind == "fixed":
        return np.asarray(spec[1], dtype=np.int64)
    if kind == "uniform":
        return rng.integers(spec[1], spec[2], size=batch, endpoint=True).astype(np.int64)
    if kind == "loguniform":
        u = rng.uniform(math.log(spec[1]), math.log(spec[2]), size=batch)
        return np.floor(np.exp(u)).astype(np.int64)
    raise ValueError(kind)


def _table_perm(rng, lengths, page_size, num_pages):
    need = [(int(L) + page_size - 1) // page_size for L in lengths]
    if sum(need) > num_pages:
        raise ValueError("pool too small for the drawn lengths")
    perm = rng.permutation(num_pages)
    width = max(need) if need else 0
    table = np.full((len(lengths), max(width, 1)), -1, dtype=np.int32)
    at = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[at:at + n]
        at += n
    return table


def _table_frag(rng, lengths, page_size, num_pages, length_spec, rounds=8, per_round=64):
    """Churn a LIFO free list with phantom sequences, then allocate."""
    free = list(range(num_pages - 1, -1, -1))      # pop() yields 0, 1, 2, ...
    live = []
    for _ in range(rounds):
        for L in _lengths(rng, length_spec, per_round):
            n = (int(L) + page_size - 1) // page_size
            if n > len(free):
                break
            live.append([free.pop() for _ in range(n)])
        order = rng.permutation(len(live))
        drop = set(order[: len(live) // 2].tolist())
        keep = []
        for i, pages in enumerate(live):
            if i in drop:
                free.extend(reversed(pages))
            else:
                keep.append(pages)
        live = keep
    need = [(int(L) + page_size - 1) // page_size for L in lengths]
    if sum(need) > len(free):
        raise ValueError("pool too small after fragmentation")
    width = max(need) if need else 0
    table = np.full((len(lengths), max(width, 1)), -1, dtype=np.int32)
    for b, n in enumerate(need):
        table[b, :n] = [free.pop() for _ in range(n)]
    return table


def _shape_scores(rng, q, k, L, cu, num_kv_heads, q_len, needles, needle_gain, ramp):
    """Sharp-attention shaping of the K draws (in place).  Pure input layout:
    K rows become multiples of query rows, chosen by the seeded ``rng``.

    * ``needles`` per sequence and KV head: position t (uniform over the
      context; the first one inside the last q_len positions when q_len > 1),
      a q-head of the group and a query row that sees t; the K row becomes
      ``needle_gain * q`` of that row.
    * ``ramp`` > 0: for every sequence and KV head, the K rows become
      ``(ramp * t * sqrt(D) / |q|^2) * q`` for q the last query row of the
      group's first q-head, so that this row's score ``q . k_t / sqrt(D)`` is
      ``ramp * t`` (before FP8 rounding): it rises along the whole context.
    """
    B = len(L)
    Hq, D = q.shape[2], q.shape[3]
    G = Hq // num_kv_heads
    for b in range(B):
        n = int(L[b])
        base = int(cu[b])
        for h in range(num_kv_heads):
            for j in range(needles):
                if j == 0 and q_len > 1:
                    t = int(rng.integers(n - q_len, n))
                else:
                    t = int(rng.integers(0, n))
                i_min = max(0, t - (n - q_len))
                i = int(rng.integers(i_min, q_len))
                hq = h * G + int(rng.integers(0, G))
                k[base + t, h, :] = np.float32(needle_gain) * q[b, i, hq, :]
            if ramp > 0:
                qr = q[b, q_len - 1, h * G, :].astype(np.float64)
                nq = float(qr @ qr)
                if nq > 0:
                    c = ramp * np.arange(n, dtype=np.float64) * np.sqrt(D) / nq
                    k[base:base + n, h, :] = (c[:, None] * qr[None, :]).astype(np.float32)


def make_workload(*, batch, num_q_heads, num_kv_heads, head_dim, page_size, q_len,
                  num_pages, lengths, table="perm", outlier_frac=0.0,
                  outlier_gain=8.0, seed=0, name="custom", q_gain=1.0, needles=0,
                  needle_gain=1.0, ramp=0.0) -> Workload:
    """Draw one workload.  ``lengths`` is ``("fixed", [..])``,
    ``("uniform", lo, hi)`` (inclusive) or ``("loguniform", lo, hi)``.
    ``q_gain``, ``needles``/``needle_gain`` and ``ramp`` shape the draws for
    sharp attention (see :func:`_shape_scores`)."""
    (s_len, s_tab, s_q, s_k, s_v, s_out, s_frag,
     s_sharp) = np.random.SeedSequence(seed).spawn(8)
    L = _lengths(np.random.default_rng(s_len), lengths, batch)
    assert len(L) == batch
    if table == "perm":
        bt = _table_perm(np.random.default_rng(s_tab), L, page_size, num_pages)
    elif table == "frag":
        bt = _table_frag(np.random.default_rng(s_frag), L, page_size, num_pages, lengths)
    else:
        raise ValueError(table)

    qf = np.random.default_rng(s_q).standard_normal(
        (batch, q_len, num_q_heads, head_dim), dtype=np.float32)
    if q_gain != 1.0:
        qf *= np.float32(q_gain)
    q = torch.from_numpy(qf).to(torch.bfloat16)

    total = int(L.sum())
    k = np.random.default_rng(s_k).standard_normal((total, num_kv_heads, head_dim),
                                                   dtype=np.float32)
    v = np.random.default_rng(s_v).standard_normal((total, num_kv_heads, head_dim),
                                                   dtype=np.float32)
    cu = np.zeros(batch + 1, dtype=np.int64)
    cu[1:] = np.cumsum(L)
    if (needles > 0 or ramp > 0) and total:
        qv = q.float().numpy()     # the exact bf16 values
        _shape_scores(np.random.default_rng(s_sharp), qv, k, L, cu, num_kv_heads, q_len,
                      needles, needle_gain, ramp)
    n_out = 0
    if outlier_frac > 0 and total:
        rows = np.random.default_rng(s_out).random((total, num_kv_heads)) < outlier_frac
        k[rows] *= np.float32(outlier_gain)
        n_out = int(rows.sum())

    def scale_of(x):
        if x.shape[0] == 0:
            return np.ones(num_kv_heads, dtype=np.float32)
        amax = np.abs(x).max(axis=(0, 2)).astype(np.float32)
        amax = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
        return (amax / np.float32(FP8_MAX)).astype(np.float32)

    return Workload(name=name, batch=batch, num_q_heads=num_q_heads,
                    num_kv_heads=num_kv_heads, head_dim=head_dim, page_size=page_size,
                    q_len=q_len, num_pages=num_pages, seq_lens=L.astype(np.int32),
                    block_table=bt, q=q, k=k, v=v, k_scale=scale_of(k),
                    v_scale=scale_of(v), cu_seqlens=cu,
                    meta=dict(seed=seed, outlier_rows=n_out, table=table, q_gain=q_gain,
                              needles=needles, needle_gain=needle_gain, ramp=ramp))


def config_workload(index: int, seed: int = 0) -> Workload:
    """One of the five named workloads, drawn with ``seed``."""
    c = dict(CONFIGS[index])
    name = c.pop("name")
    return make_workload(seed=seed, name=name, **c)


def workload_tag(index: int) -> str:
    c = CONFIGS[index]
    return (f"{c['name']}: B={c['batch']} Hq={c['num_q_heads']} Hkv={c['num_kv_heads']} "
            f"D={c['head_dim']} ps={c['page_size']} q_len={c['q_len']} lengths={c['lengths']}")


def make_verify_logits(*, batch, num_drafts, vocab, seed=0, dtype=torch.bfloat16, ties=False):
    """Synthetic verify-step logits and MTP drafts for greedy acceptance.

    ``logits`` ``[B, K + 1, V]``: N(0, 1) draws (rounded to ``dtype``) with one
    planted token per row whose logit is 8.0 (far above the draws); with
    ``ties`` a second token of every row gets the same 8.0.  ``drafts``
    int32 ``[B, K]``: each sequence draws an agreement length a in 0..K; draft
    i is the row's planted token for i < a, and a different token at i = a
    (the tokens after it are random).  Pure input construction: the planted
    tokens are chosen, never computed from the logits."""
    s_log, s_tok, s_len, s_rest = np.random.SeedSequence(seed).spawn(4)
    K1 = num_drafts + 1
    x = np.random.default_rng(s_log).standard_normal((batch, K1, vocab), dtype=np.float32)
    rt = np.random.default_rng(s_tok)
    planted = rt.integers(0, vocab, size=(batch, K1))
    rows = np.arange(batch)[:, None], np.arange(K1)[None, :]
    x[rows[0], rows[1], planted] = 8.0
    second = None
    if ties:
        second = rt.integers(0, vocab, size=(batch, K1))
        x[rows[0], rows[1], second] = 8.0
    a = np.random.default_rng(s_len).integers(0, num_drafts + 1, size=batch)
    rr = np.random.default_rng(s_rest)
    drafts = rr.integers(0, vocab, size=(batch, max(num_drafts, 0))).astype(np.int32)
    for b in range(batch):
        drafts[b, :a[b]] = planted[b, :a[b]]
        if a[b] < num_drafts and vocab > 1:
            drafts[b, a[b]] = (planted[b, a[b]] + 1 + rr.integers(0, vocab - 1)) % vocab
    logits = torch.from_numpy(x).to(dtype)
    return logits, drafts, dict(planted=planted, agree=a, second=second)


def make_rope_inputs(*, batch, n_new, num_q_heads, num_kv_heads, head_dim, max_pos,
                     rope_base=500000.0, seed=0):
    """Synthetic QKV projection output of the new tokens and a rotary table.

    ``qkv`` bf16 ``[B, n_new, Hq + 2 Hkv, D]``: N(0, 1) draws rounded to bf16
    (query heads, then key heads, then value heads).  ``cos_sin`` float32
    ``[max_pos, D]``: the cos (columns 0 .. D/2 - 1) and sin (the rest) of the
    angles ``pos * rope_base ** (-2 i / D)`` -- the LLaMA-style frequency
    schedule (rope_base 500000 as in LLaMA-3), evaluated in float64 and
    rounded to float32; an input table, the same for both sides."""
    (s_x,) = np.random.SeedSequence(seed).spawn(1)
    x = np.random.default_rng(s_x).standard_normal(
        (batch, n_new, num_q_heads + 2 * num_kv_heads, head_dim), dtype=np.float32)
    qkv = torch.from_numpy(x).to(torch.bfloat16)
    inv = float(rope_base) ** (-np.arange(head_dim // 2, dtype=np.float64) * 2.0 / head_dim)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * inv[None, :]
    cos_sin = np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)
    return qkv, cos_sin


def make_packed_queries(*, q_lens, num_q_heads, head_dim, seed=0):
    """Packed bf16 queries for ragged verify / prefill: ``q`` ``[sum q_lens,
    Hq, D]`` N(0, 1) rounded to bf16, and ``cu_q_lens`` int32 ``[B + 1]``
    (exclusive prefix sums of ``q_lens``)."""
    (s_q,) = np.random.SeedSequence(seed).spawn(1)
    ql = np.asarray(q_lens, dtype=np.int64)
    cu = np.zeros(len(ql) + 1, np.int32)
    cu[1:] = np.cumsum(ql)
    x = np.random.default_rng(s_q).standard_normal((int(cu[-1]), num_q_heads, head_dim),
                                                    dtype=np.float32)
    return torch.from_numpy(x).to(torch.bfloat16), cu
