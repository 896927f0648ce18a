"""GPU: finer-grained FP8 scales, one dynamic scale per (token, KV head)
computed at append.  The append is bit-exact with the oracle (codes, scales,
the per-head V bound) and decode over such a cache matches the oracle's
attention with per-token dequantisation, on the LLaMA-3-8B-shaped decode and
on the long-context workload whose 1 % x8 outlier keys are what a per-head
scale handles worst."""

import numpy as np
import pytest
import torch

from oracle import attention, paged
from paged_fp8_kv_05_b200 import build, workloads

from parity import assert_close, k_token_major, record_parity, v_token_major

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ak():
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv
    return atlas_kv


def _oracle_cache(w):
    P, Hkv, ps, D = w.num_pages, w.num_kv_heads, w.page_size, w.head_dim
    out = {}
    for which, src in (("k", w.k), ("v", w.v)):
        pages = np.zeros((P, Hkv, ps, D), np.uint8)
        sc = np.zeros((P, Hkv, ps), np.float32)
        written = np.zeros((P, Hkv, ps), bool)
        for b in range(w.batch):
            L = int(w.seq_lens[b])
            seq = src[w.cu_seqlens[b]:w.cu_seqlens[b + 1]][None]
            pages, sc = paged.append_tokscale(pages, sc, seq, w.block_table[b:b + 1],
                                              np.array([0]), ps)
            t = np.arange(L)
            written[w.block_table[b, t // ps], :, t % ps] = True
        out[which] = (pages, sc, written)
    return out


@pytest.mark.parametrize("cfg,batch", [(1, 8), (3, None)])
def test_tokscale_append_bit_exact_and_decode(ak, cfg, batch):
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload
    c = dict(workloads.CONFIGS[cfg])
    c.pop("name")
    if batch:
        c["batch"] = batch
    w = workloads.make_workload(seed=0, **c)
    dw = DeviceWorkload(w, token_scales=True)
    assert dw.pool.device_error() == 0
    ref = _oracle_cache(w)
    for which, dev_pages, dev_sc in (("k", dw.pool.k_pages, dw.scales.k),
                                     ("v", dw.pool.v_pages, dw.scales.v)):
        pages, sc, written = ref[which]
        got = dev_pages.cpu().numpy()
        got = k_token_major(got) if which == "k" else v_token_major(got)
        assert np.array_equal(got[written], pages[written]), f"{which} codes"
        assert np.array_equal(dev_sc.cpu().numpy()[written], sc[written]), f"{which} scales"
    vb = dw.scales.v_bound.cpu().numpy()
    assert np.array_equal(vb, ref["v"][1].max(axis=(0, 2)))
    out = dw.decode().float().cpu().numpy()
    assert dw.pool.device_error() == 0
    kp, ksc, _ = ref["k"]
    vp, vsc, _ = ref["v"]
    want = attention.paged_gqa_decode_tokscale(w.q_f64(), kp, vp, ksc, vsc, w.block_table,
                                               w.seq_lens, w.q_len, w.page_size)
    max_abs, rel = assert_close(out, want, f"per-token scales, config {cfg}")
    record_parity(f"per-token scales, config {cfg} (batch {w.batch})", max_abs, rel)


def test_tokscale_verify_shape_and_splits(ak):
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload
    w = workloads.make_workload(batch=6, num_q_heads=40, num_kv_heads=8, head_dim=128,
                                page_size=16, q_len=5, num_pages=600,
                                lengths=("uniform", 100, 1100), seed=7, outlier_frac=0.02)
    dw = DeviceWorkload(w, token_scales=True, min_split_tokens=64)
    ref = _oracle_cache(w)
    kp, ksc, _ = ref["k"]
    vp, vsc, _ = ref["v"]
    want = attention.paged_gqa_decode_tokscale(w.q_f64(), kp, vp, ksc, vsc, w.block_table,
                                               w.seq_lens, w.q_len, w.page_size)
    for split in (0, 128):
        dw.pool.set_split_tokens(split)
        out = dw.decode(out=torch.empty_like(dw.q)).float().cpu().numpy()
        assert dw.pool.device_error() == 0
        max_abs, rel = assert_close(out, want, f"per-token scales, verify, split {split}")
        record_parity(f"per-token scales, verify shape, split {split or 'auto'}", max_abs, rel)


def test_tokscale_needs_head_dim_128(ak):
    pool = ak.KVPool(4, 16, 1, 64, [1.0], [1.0], max_batch=1, max_q_len=1, num_q_heads=1,
                     max_seq_len=16)
    sc = ak.TokenScales(pool)
    q = torch.zeros(1, 1, 1, 64, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    sl = torch.ones(1, dtype=torch.int32, device="cuda")
    with pytest.raises(ak.AtlasError) as e:
        ak.atlas_paged_gqa_decode_tokscale(pool, sc, q, bt, sl, 1)
    assert e.value.status == ak.ATLAS_ERR_UNSUPPORTED
