"""Put a drawn workload on the GPU and run the path through the C ABI.

Host-side plumbing only (uploads, pool creation, per-sequence cache fill,
one decode step); the arithmetic happens in ``libatlas_kv.so``.
"""

import numpy as np
import torch

from . import atlas_kv as ak
from .workloads import Workload


class DeviceWorkload:
    """A workload resident in HBM: page pool, block table, lengths, q, out.

    ``fill`` pre-sets every page byte (0x7F is an E4M3 NaN: slots the path
    must never read then poison the result if it does).
    """

    def __init__(self, w: Workload, device="cuda", fill=0x7F, min_split_tokens=256,
                 fill_cache=True, max_batch=None, max_q_len=None, token_scales=False):
        self.w = w
        self.device = torch.device(device)
        self.pool = ak.KVPool(w.num_pages, w.page_size, w.num_kv_heads, w.head_dim,
                              w.k_scale, w.v_scale, max_batch=max_batch or max(w.batch, 1),
                              max_q_len=max(max_q_len or 0, w.q_len), num_q_heads=w.num_q_heads,
                              max_seq_len=max(w.max_seq_len, w.q_len), device=self.device,
                              min_split_tokens=min_split_tokens, fill=fill)
        self.block_table = torch.from_numpy(np.ascontiguousarray(w.block_table)).to(self.device)
        self.seq_lens = torch.from_numpy(w.seq_lens.astype(np.int32)).to(self.device)
        self.q = w.q.to(self.device).contiguous()
        self.out = torch.empty_like(self.q)
        self.start_new = torch.from_numpy(
            (w.seq_lens.astype(np.int64) - w.q_len).astype(np.int32)).to(self.device)
        self.k_new = torch.from_numpy(w.new_tokens("k")).to(self.device).contiguous()
        self.v_new = torch.from_numpy(w.new_tokens("v")).to(self.device).contiguous()
        # finer-grained mode: one dynamic scale per (token, KV head)
        self.scales = ak.TokenScales(self.pool) if token_scales else None
        if fill_cache:
            self.fill_prefix()
            self.append_new()
            torch.cuda.synchronize(self.device)

    def fill_prefix(self):
        """Append every token before the q_len new ones, one sequence per call."""
        w = self.w
        zero = torch.zeros(1, dtype=torch.int32, device=self.device)
        for b in range(w.batch):
            n = int(w.seq_lens[b]) - w.q_len
            if n <= 0:
                continue
            kb = torch.from_numpy(w.seq_k(b)[:n]).to(self.device).unsqueeze(0).contiguous()
            vb = torch.from_numpy(w.seq_v(b)[:n]).to(self.device).unsqueeze(0).contiguous()
            if self.scales is not None:
                ak.atlas_fp8_kv_append_tokscale(self.pool, self.scales, kb, vb,
                                                self.block_table[b:b + 1], zero)
            else:
                ak.atlas_fp8_kv_append(self.pool, kb, vb, self.block_table[b:b + 1], zero)

    def append_new(self, stream=None):
        """A0: quantise and scatter the step's q_len new tokens of every sequence."""
        if self.scales is not None:
            ak.atlas_fp8_kv_append_tokscale(self.pool, self.scales, self.k_new, self.v_new,
                                            self.block_table, self.start_new, stream=stream)
            return
        ak.atlas_fp8_kv_append(self.pool, self.k_new, self.v_new, self.block_table,
                               self.start_new, stream=stream)

    def decode(self, stream=None, out=None):
        """A1-A9: attention of the q_len new rows over the paged cache."""
        if self.scales is not None:
            return ak.atlas_paged_gqa_decode_tokscale(
                self.pool, self.scales, self.q, self.block_table, self.seq_lens,
                max(self.w.max_seq_len, self.w.q_len), out=self.out if out is None else out,
                stream=stream)
        return ak.atlas_paged_gqa_decode(self.pool, self.q, self.block_table, self.seq_lens,
                                         max(self.w.max_seq_len, self.w.q_len),
                                         out=self.out if out is None else out, stream=stream)

    def step(self, stream=None, out=None):
        """One fused step (A0-A9 in one kernel): append the q_len new tokens
        and decode."""
        return ak.atlas_paged_gqa_append_decode(
            self.pool, self.k_new, self.v_new, self.q, self.block_table, self.seq_lens,
            max(self.w.max_seq_len, self.w.q_len), out=self.out if out is None else out,
            stream=stream)

    def plan(self):
        return ak.atlas_paged_gqa_decode_plan(self.pool, self.w.batch, self.w.num_q_heads,
                                              self.w.q_len, max(self.w.max_seq_len, self.w.q_len))
