"""GPU: greedy MTP acceptance is bit-exact with the oracle (targets,
accepted counts, next tokens), on the 27B-class verify shape and on edge
cases: unaligned rows (scalar path), no drafts, ties, a one-token vocabulary,
and two calls in a row (the completion counters are left at zero)."""

import numpy as np
import pytest
import torch

from oracle import acceptance
from paged_fp8_kv_05_b200 import build, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ak():
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv
    return atlas_kv


CASES = [
    # (batch, K, vocab, dtype, ties)
    (128, 4, 151936, torch.bfloat16, False),   # MTP K = 4 at concurrency 128
    (7, 4, 1001, torch.float32, False),        # odd vocabulary: unaligned rows
    (5, 7, 32000, torch.bfloat16, True),       # ties: the lower token id wins
    (3, 0, 50, torch.float32, False),          # no drafts: next token = target 0
    (4, 4, 1, torch.bfloat16, False),          # one-token vocabulary
    (33, 4, 4099, torch.bfloat16, True),
]


@pytest.mark.parametrize("case", CASES)
def test_greedy_accept_bit_exact(ak, case):
    B, K, V, dtype, ties = case
    logits, drafts, meta = workloads.make_verify_logits(batch=B, num_drafts=K, vocab=V,
                                                        seed=B + K, dtype=dtype, ties=ties)
    pool = ak.KVPool(4, 16, 1, 64, [1.0], [1.0], max_batch=B, max_q_len=1, num_q_heads=1,
                     max_seq_len=16)
    lg = logits.cuda().contiguous()
    dr = torch.from_numpy(drafts).cuda().contiguous()
    n_ref, next_ref, tg_ref = acceptance.greedy_accept(logits.float().numpy(), drafts)
    for call in range(2):
        n, nxt, tg = ak.atlas_mtp_greedy_accept(pool, lg, dr)
        torch.cuda.synchronize()
        assert np.array_equal(tg.cpu().numpy(), tg_ref), f"targets, call {call}"
        assert np.array_equal(n.cpu().numpy(), n_ref), f"accepted counts, call {call}"
        assert np.array_equal(nxt.cpu().numpy(), next_ref), f"next tokens, call {call}"
    assert pool.device_error() == 0
    if V > 1 and not ties:                        # the planted tokens are the targets
        assert np.array_equal(tg_ref, meta["planted"])
        assert np.array_equal(n_ref, np.minimum(meta["agree"], K))
