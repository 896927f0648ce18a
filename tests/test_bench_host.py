"""CPU: host-side pieces of bench.py that need no GPU.

The end-to-end leg stages a step's inputs (q, the new K and V, the lengths,
the block table) in one buffer at 256-byte-aligned offsets and hands the
C ABI views into its device copy: the views must reproduce every input
exactly, with its dtype and shape, contiguous and aligned.
"""

import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from paged_fp8_kv_05_b200 import workloads  # noqa: E402


def test_staged_views_reproduce_every_input():
    for index in (0, 2):
        w = workloads.config_workload(index)
        parts = [w.q.contiguous(), torch.from_numpy(w.new_tokens("k")),
                 torch.from_numpy(w.new_tokens("v")),
                 torch.from_numpy(w.seq_lens.astype(np.int32)),
                 torch.from_numpy(np.ascontiguousarray(w.block_table))]
        buf, offs = bench.stage_inputs(parts)
        assert all(o % 256 == 0 for o in offs)
        assert offs == sorted(offs) and buf.numel() % 256 == 0
        nbytes = [t.numel() * t.element_size() for t in parts]
        assert all(offs[i] + nbytes[i] <= offs[i + 1] for i in range(len(parts) - 1))
        assert offs[-1] + nbytes[-1] <= buf.numel()
        copy = buf.clone()  # stands in for the device copy
        for t, v in zip(parts, bench.staged_views(copy, parts, offs)):
            assert v.dtype == t.dtype and v.shape == t.shape and v.is_contiguous()
            assert torch.equal(v, t)
            assert (v.data_ptr() - copy.data_ptr()) % 256 == 0
