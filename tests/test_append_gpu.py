"""GPU: the FP8 page append is bit-exact with the oracle's encoder and
scatter, and writes nothing else."""

import numpy as np
import pytest
import torch

from oracle import e4m3, paged
from paged_fp8_kv_05_b200 import build, workloads

from parity import k_token_major, oracle_pages, v_token_major

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ak():
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv
    return atlas_kv


def _pool(ak, P, Hkv, ps, D, ks, vs, fill=0x7F):
    return ak.KVPool(P, ps, Hkv, D, ks, vs, max_batch=4, max_q_len=8, num_q_heads=Hkv,
                     max_seq_len=64, fill=fill)


@pytest.mark.parametrize("cfg", [0, 1, 4])
def test_cache_fill_bit_exact(ak, cfg):
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload
    w = workloads.config_workload(cfg)
    dw = DeviceWorkload(w)
    assert dw.pool.device_error() == 0
    for which, dev in (("k", dw.pool.k_pages), ("v", dw.pool.v_pages)):
        want, written = oracle_pages(w, which)           # token-major [P, Hkv, ps, D]
        got = dev.cpu().numpy()
        if which == "v":                                 # V pages: 16-slot groups
            got = v_token_major(got)
        else:                                            # K rows: chunk-permuted at D = 128
            got = k_token_major(got)
        assert np.array_equal(got[written], want[written]), f"{which}: codes differ"
        assert np.all(got[~written] == 0x7F), f"{which}: stray writes"


def _special_values():
    finite = np.concatenate([np.arange(0x7F), np.arange(0x80, 0xFF)]).astype(np.uint8)
    vals = e4m3.decode(finite)
    table = e4m3.decode(np.arange(0x7F, dtype=np.uint8))
    mids = (table[:-1] + table[1:]) / 2
    mids32 = mids.astype(np.float32)
    extra = np.array([0.0, -0.0, 448.0, 449.0, 463.99, 464.0, 480.0, 1e6, -1e6, np.inf, -np.inf,
                      2.0 ** -10, -(2.0 ** -10), 1.5 * 2.0 ** -10, 1e-30, -1e-30, 1e-45, 3e-39],
                     np.float32)
    ys = np.concatenate([vals.astype(np.float32), mids32, -mids32,
                         np.nextafter(mids32, np.float32(np.inf)),
                         np.nextafter(mids32, np.float32(-np.inf)), extra]).astype(np.float32)
    return ys


@pytest.mark.parametrize("scale", [1.0, 0.5, 0.0123, 3.7])
def test_special_values_bit_exact(ak, scale):
    ys = _special_values()
    D, Hkv, ps = 64, 1, 16
    n = (len(ys) + D - 1) // D
    x = np.zeros(n * D, np.float32)
    with np.errstate(over="ignore"):
        x[:len(ys)] = (ys.astype(np.float64) * scale).astype(np.float32)
    x = x.reshape(1, n, Hkv, D)
    P = (n + ps - 1) // ps
    pool = _pool(ak, P, Hkv, ps, D, [scale], [scale])
    bt = torch.arange(P, dtype=torch.int32, device="cuda").reshape(1, P)
    start = torch.zeros(1, dtype=torch.int32, device="cuda")
    xt = torch.from_numpy(x).cuda()
    ak.atlas_fp8_kv_append(pool, xt, xt, bt, start)
    got = paged.gather_codes(pool.k_pages.cpu().numpy(), bt.cpu().numpy(), 0, n, ps)
    want = e4m3.encode(x[0], np.float32(scale))
    assert np.array_equal(got, want)
    assert pool.device_error() == 0


def test_division_cases_bit_exact(ak):
    from test_oracle_e4m3 import DIVISION_CASES
    D = 64
    for xb, sb in DIVISION_CASES:
        x = np.full((1, 1, 1, D), np.uint32(xb).view(np.float32), np.float32)
        s = np.uint32(sb).view(np.float32)
        pool = _pool(ak, 1, 1, 16, D, [s], [s])
        bt = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        xt = torch.from_numpy(x).cuda()
        ak.atlas_fp8_kv_append(pool, xt, xt, bt, st)
        got = pool.k_pages[0, 0, 0].cpu().numpy()
        assert np.all(got == e4m3.encode(x[0, 0, 0], s))


def test_bf16_input_and_ragged_positions(ak):
    rng = np.random.default_rng(7)
    B, n_new, Hkv, D, ps, P = 3, 37, 2, 128, 16, 40
    xf = (rng.standard_normal((B, n_new, Hkv, D)) * 3).astype(np.float32)
    xb = torch.from_numpy(xf).to(torch.bfloat16)
    x_exact = xb.float().numpy()
    ks = np.array([0.011, 0.02], np.float32)
    vs = np.array([0.007, 0.03], np.float32)
    pool = _pool(ak, P, Hkv, ps, D, ks, vs)
    table = rng.permutation(P)[:B * 8].reshape(B, 8).astype(np.int32)
    start = np.array([0, 5, 63], np.int32)          # mid-page starts, page crossings
    bt = torch.from_numpy(table).cuda()
    st = torch.from_numpy(start).cuda()
    kt = xb.cuda().contiguous()
    vt = (xb * -0.5).cuda().contiguous()
    ak.atlas_fp8_kv_append(pool, kt, vt, bt, st)
    assert pool.device_error() == 0
    init_k = np.full((P, Hkv, ps, D), 0x7F, np.uint8)
    init_v = np.full((P, Hkv, ps // 16, D, 16), 0x7F, np.uint8)
    want_k = paged.append(init_k, x_exact, ks, table, start, ps, layout=paged.k_layout(D))
    want_v = paged.append(init_v, (vt.float().cpu().numpy()), vs, table, start, ps, layout="grp16")
    assert np.array_equal(pool.k_pages.cpu().numpy(), want_k)
    assert np.array_equal(pool.v_pages.cpu().numpy(), want_v)


def test_out_of_range_rows_are_skipped_and_flagged(ak):
    B, n_new, Hkv, D, ps, P = 2, 4, 1, 64, 16, 4
    pool = _pool(ak, P, Hkv, ps, D, [0.01], [0.01])
    x = torch.randn(B, n_new, Hkv, D, device="cuda")
    bt = torch.tensor([[0, -1], [5, 1]], dtype=torch.int32, device="cuda")   # -1 and 5 invalid
    st = torch.tensor([14, 0], dtype=torch.int32, device="cuda")
    before_k = pool.k_pages.clone()
    ak.atlas_fp8_kv_append(pool, x, x, bt, st)
    err = pool.device_error()
    assert err & ak.DEVERR_APPEND
    after = pool.k_pages.cpu().numpy()
    changed = np.argwhere(np.any(after != before_k.cpu().numpy(), axis=-1))
    # only sequence 0, positions 14 and 15 (page 0, slots 14-15) may be written
    assert sorted(map(tuple, changed.tolist())) == [(0, 0, 14), (0, 0, 15)]
    assert pool.device_error() == 0                    # reading clears the word
    st_bad = torch.tensor([-3, 40], dtype=torch.int32, device="cuda")  # negative / past table
    ak.atlas_fp8_kv_append(pool, x, x, bt, st_bad)
    assert pool.device_error() & ak.DEVERR_APPEND
