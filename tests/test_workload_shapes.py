"""CPU checks of the seeded generator's sharp-attention shaping: the inputs
the sharp GPU parity cases use are what those cases claim (scores computed
here in float64 from the quantised cache, never from GPU output)."""

import numpy as np

from oracle import paged
from paged_fp8_kv_05_b200 import workloads

from parity import oracle_pages


def _w(**kw):
    base = dict(batch=3, num_q_heads=16, num_kv_heads=4, head_dim=128, page_size=16, q_len=1,
                num_pages=3 * 160 + 8, lengths=("uniform", 1024, 2500), table="perm", seed=41)
    base.update(kw)
    return workloads.make_workload(**base)


def _scores(w, b, h, i, hq):
    kp, _ = oracle_pages(w, "k")
    K = paged.gather_dequant(kp, w.k_scale, w.block_table, b, int(w.seq_lens[b]), w.page_size)
    return K[:, h, :] @ w.q_f64()[b, i, hq, :] / np.sqrt(w.head_dim)


def test_unshaped_draws_are_unchanged_by_the_options():
    a, b = _w(), _w(q_gain=1.0, needles=0, ramp=0.0)
    assert np.array_equal(a.k, b.k) and np.array_equal(a.v, b.v)
    assert np.array_equal(a.q.float().numpy(), b.q.float().numpy())


def test_q_gain_scales_the_score_spread():
    w1, w8 = _w(), _w(q_gain=8.0)
    s1 = _scores(w1, 0, 1, 0, 5)
    s8 = _scores(w8, 0, 1, 0, 5)
    assert 0.8 < s1.std() < 1.2 and 6.4 < s8.std() < 9.6


def test_ramp_moves_the_reference_on_every_unit():
    """Along each sequence the running maximum of the shaped row's scores
    (base 2) rises by more than 0.5 on at least 95 % of the 32-token units
    (FP8 rounding of K makes single steps noisy), so a softmax reference that
    moves only by more than 0.5 moves on nearly every unit."""
    w = _w(ramp=0.03)
    G = w.num_q_heads // w.num_kv_heads
    for b in range(w.batch):
        L = int(w.seq_lens[b])
        for h in range(w.num_kv_heads):
            s = _scores(w, b, h, w.q_len - 1, h * G) * np.log2(np.e)
            full = L // 32 * 32                      # whole units only
            unit_max = np.maximum.accumulate([s[u:u + 32].max() for u in range(0, full, 32)])
            assert np.mean(np.diff(unit_max) > 0.5) >= 0.95, (b, h)


def test_needles_dominate_their_row_and_one_sits_in_the_drafts():
    w = _w(needles=2, needle_gain=1.0, q_len=5, num_q_heads=40, num_kv_heads=8,
           lengths=("uniform", 128, 1152), num_pages=3 * 72 + 8)
    q = w.q.float().numpy()
    G = w.num_q_heads // w.num_kv_heads
    for b in range(w.batch):
        L = int(w.seq_lens[b])
        k = w.seq_k(b)
        for h in range(w.num_kv_heads):
            # rows of this head equal to some query row of the group
            hits = [t for t in range(L)
                    if any(np.array_equal(k[t, h], q[b, i, h * G + g])
                           for i in range(w.q_len) for g in range(G))]
            assert len(hits) >= 1
            assert any(t >= L - w.q_len for t in hits)
