"""GPU parity in the sharp-attention regime.

The named workloads draw q, K and V from N(0, 1), so every score is ~N(0, 1)
and the softmax over thousands of keys is nearly flat.  The kernel's own
shortcuts matter most when it is not: probabilities carried as two E4M3
parts, a per-row softmax reference that moves only when a score exceeds it by
more than 0.5 (base 2), accumulation through FP8 tensor-core MMAs.  These
cases sharpen the softmax on the shapes of the LLaMA-3-8B decode, the
27B-class MTP verify and the ragged MQA workloads (batch reduced so the float64
oracle finishes in seconds):

* q multiplied by 4 and by 8 (score standard deviation 4 and 8);
* planted "needle" keys, a K row equal to a query row of its group (score
  about |q|^2 / sqrt(D) = 11 against N(0, 1) neighbours), one of them inside
  the MTP drafts for the verify shape;
* a "ramp": K rows proportional to one query row with a coefficient rising
  along the context, so that row's scores grow by ~1.4 (base 2) per 32-token
  unit and its softmax reference has to move on nearly every unit.

Each case runs on the warp-MMA kernel in both partitions and on the
tensor-core kernel, with the automatic split length and with 128-token
splits (segments cut into many parts, merged by log-sum-exp), and is
compared element by element with the oracle at max-abs 1e-2, rel-L2 5e-3.
"""

import functools

import pytest
import torch

from paged_fp8_kv_05_b200 import build, workloads

from parity import assert_close, oracle_decode, record_parity

pytestmark = pytest.mark.gpu

SHAPES = {
    "llama8b-decode": dict(batch=6, num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=16,
                           q_len=1, num_pages=6 * 256 + 16, lengths=("uniform", 1024, 4096),
                           table="perm"),
    "mtp-verify": dict(batch=12, num_q_heads=40, num_kv_heads=8, head_dim=128, page_size=16,
                       q_len=5, num_pages=12 * 72 + 16, lengths=("uniform", 128, 1152),
                       table="perm"),
    "ragged-mqa": dict(batch=10, num_q_heads=64, num_kv_heads=1, head_dim=128, page_size=64,
                       q_len=1, num_pages=12000, lengths=("loguniform", 256, 8192),
                       table="frag"),
}
VARIANTS = {
    "score-std-4": dict(q_gain=4.0),
    "score-std-8": dict(q_gain=8.0),
    "needles": dict(needles=2, needle_gain=1.0),
    "ramp": dict(ramp=0.03),
}


@functools.lru_cache(maxsize=None)
def _workload(shape, variant):
    return workloads.make_workload(seed=41, name=f"{shape}/{variant}", **SHAPES[shape],
                                   **VARIANTS[variant])


@functools.lru_cache(maxsize=None)
def _oracle(shape, variant):
    return oracle_decode(_workload(shape, variant))


@pytest.fixture(scope="module")
def ak():
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv
    return atlas_kv


# (ATLAS_OPT_KERNEL, ATLAS_OPT_PARTITION): warp-MMA kernel in its grid and
# balanced partitions, and the tensor-core kernel
KERNELS = {"warp-grid": (1, 1), "warp-balanced": (1, 2), "tcgen05": (2, 0)}


@pytest.mark.parametrize("split", [0, 128])
@pytest.mark.parametrize("kernel", list(KERNELS))
@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("shape", list(SHAPES))
def test_sharp_attention(ak, shape, variant, kernel, split):
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload
    w = _workload(shape, variant)
    dw = DeviceWorkload(w, min_split_tokens=64)
    kern, partition = KERNELS[kernel]
    dw.pool.set_option(ak.OPT_KERNEL, kern)
    dw.pool.set_option(ak.OPT_PARTITION, partition)
    dw.pool.set_split_tokens(split)
    got = dw.decode().float().cpu().numpy()
    assert dw.pool.device_error() == 0
    case = f"sharp {shape} {variant} {kernel} split {split or 'auto'}"
    max_abs, rel = assert_close(got, _oracle(shape, variant), case)
    record_parity(case, max_abs, rel)
