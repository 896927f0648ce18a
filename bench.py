#!/usr/bin/env python
"""Benchmark of the paged FP8 decode step on B200.

One step = the whole hot path over one batch: the FP8 append of the step's
q_len new K/V tokens per sequence (quantise + scatter into the pages) and the
paged decode / verify attention over every sequence's full context, run as
one fused kernel (atlas_paged_gqa_append_decode).  By default one run times
the four workloads the HBM-roofline target names, each for K steps after W
warm-up steps: the long-context split-KV decode (B=4, Hq=32, Hkv=8, D=128,
context U[65536, 131072]; the headline, the largest single-GPU workload), the
LLaMA-3-8B-shaped decode layer, the 27B-class MTP verify (q_len 5) and the
ragged MQA decode.  The headline's numbers fill the top-level keys; every
workload's record sits under ``per_config``.  ``--config I`` times workload I
alone.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--impl ours|reference]

Timing: L2 is flushed before every step, outside the CUDA events that bracket
the step (the step is one kernel, so the event pair on its stream times that
kernel): a 256 MiB write, then a read of another 256 MiB buffer, so that the
step starts from a cold L2 holding no dirty lines of the flush (the write
alone would leave ~126 MB of write-backs to land inside the timed step).  Under torchrun every rank runs an
independent replica (the path has no exchange step), the timed region is
bracketed by a barrier and a device synchronise, and the max over ranks is
taken.  Rank 0 prints one JSON line.
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged FP8 decode attention HBM GB/s (frac of B200 roofline); tokens/s/layer"
FALLBACK_HBM_GBS = 6650.0
# The workloads the HBM-roofline target names, timed in one run; the headline
# is the largest one that fits one GPU (the long-context split-KV decode).
TARGETS = (3, 1, 2, 4)
HEADLINE = 3
FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=None,
                    help="time one named workload only (default: workloads 1-4, headline 3)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--split-tokens", type=int, default=0, help="override the split size")
    ap.add_argument("--stages", type=int, default=0, help="override the K/V staging depth")
    ap.add_argument("--waves", type=int, default=0, help="CTAs per resident CTA slot")
    ap.add_argument("--partition", type=int, default=0, help="0 auto, 1 grid, 2 balanced")
    ap.add_argument("--rows-per-cta", type=int, default=0, help="query rows per CTA (0 auto)")
    ap.add_argument("--kernel", type=int, default=0,
                    help="0 auto, 1 FP8 warp-MMA kernel, 2 tensor-core (tcgen05) kernel")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the records of the rows after the core path")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    return ap.parse_args()


# ------------------------------------------------------------------ helpers

def algorithmic_bytes(w):
    """Bytes the step must move at minimum: FP8 K+V of valid tokens, scales,
    bf16 q in and out, block-table entries of valid pages and seq_lens (decode);
    float32 new K/V in and FP8 codes out (append)."""
    L = w.seq_lens.astype(np.int64)
    decode = (int(L.sum()) * w.num_kv_heads * w.head_dim * 2 + 2 * w.num_kv_heads * 4
              + 2 * w.batch * w.q_len * w.num_q_heads * w.head_dim * 2
              + 4 * int(((L + w.page_size - 1) // w.page_size).sum()) + 4 * w.batch)
    n_new = w.batch * w.q_len * w.num_kv_heads * w.head_dim * 2
    append = n_new * 4 + n_new * 1 + 4 * w.batch + 4 * w.batch
    return decode, append


def algorithmic_flops(w):
    return 4 * int(w.seq_lens.astype(np.int64).sum()) * w.q_len * w.num_q_heads * w.head_dim


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# The decode kernel and its launch path: the kernel, the shared device helpers
# and planner, the ABI layer that plans and launches it.
DECODE_SOURCES = ("atlas_internal.cuh", "atlas_kv.cu", "decode_fp8.cu", "decode_tc.cu")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_fp8_kv_05_b200", "csrc")
    for name in DECODE_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(config_index):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.txt")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash()
    for line in open(path):
        parts = line.split()
        if len(parts) >= 3 and parts[0] == f"config{config_index}" and parts[1] == want:
            try:
                return int(parts[2])
            except ValueError:
                return None
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return world, rank, local, dist
    return 1, 0, local, None


def max_over_ranks(x, dist, device):
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_config(w, index, bytes_decode, bytes_append, args):
    from paged_fp8_kv_05_b200.workloads import workload_tag
    return {"workload": workload_tag(index), "batch": w.batch, "q_len": w.q_len,
            "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "page_size": w.page_size,
            "mean_context": float(w.seq_lens.mean()), "max_context": int(w.max_seq_len),
            "decode_bytes_per_step": bytes_decode, "append_bytes_per_step": bytes_append,
            "l2": "flushed before every step, outside the events: 256 MiB write, then "
                  "256 MiB read of another buffer (cold L2, no dirty lines)",
            "parallelism": f"replicas x{args.gpus}"}


# ------------------------------------------------------------------ CPU oracle legs

def oracle_pair_timer(w):
    """Returns (run(b, h) -> seconds, nbytes(b, h)) for one step of the oracle
    on one (sequence, KV head) pair: the oracle append of the pair's q_len new
    tokens, then the float64 decode of the head's G q-heads.  The attention of
    one KV head never reads another head's pages, so a pair is an exact slice
    of the step; the oracle runs unmodified on head-sliced arrays."""
    from oracle import attention, e4m3, paged
    ps, Hkv, D, G = w.page_size, w.num_kv_heads, w.head_dim, w.group
    kp = np.zeros((w.num_pages, Hkv, ps, D), np.uint8)
    vp = np.zeros_like(kp)
    filled = set()
    q64 = w.q_f64()
    newk, newv = w.new_tokens("k"), w.new_tokens("v")

    def prepare(b, h):
        if (b, h) in filled:
            return
        L = int(w.seq_lens[b])
        t = np.arange(L)
        pg = w.block_table[b, t // ps]
        kp[pg, h, t % ps, :] = e4m3.encode(w.seq_k(b)[:, h, :], w.k_scale[h])
        vp[pg, h, t % ps, :] = e4m3.encode(w.seq_v(b)[:, h, :], w.v_scale[h])
        filled.add((b, h))

    def run(b, h):
        prepare(b, h)
        t0 = time.perf_counter()
        hs = slice(h, h + 1)
        start = w.seq_lens[b:b + 1] - w.q_len
        k2 = paged.append(kp[:, hs], newk[b:b + 1, :, hs], w.k_scale[hs], w.block_table[b:b + 1],
                          start, ps)
        v2 = paged.append(vp[:, hs], newv[b:b + 1, :, hs], w.v_scale[hs], w.block_table[b:b + 1],
                          start, ps)
        attention.paged_gqa_decode(q64[b:b + 1, :, h * G:(h + 1) * G], k2, v2, w.k_scale[hs],
                                   w.v_scale[hs], w.block_table[b:b + 1], w.seq_lens[b:b + 1],
                                   w.q_len, ps)
        return time.perf_counter() - t0

    def nbytes(b, h):
        return int(w.seq_lens[b]) * D * 2 + 2 * w.q_len * G * D * 2

    return run, nbytes


def oracle_prefix_timer(w):
    """Returns (run(b, h, n) -> seconds, nbytes(b, h, n)) for one step of the
    oracle on the first n context tokens of one (sequence, KV head) pair: the
    pair's pages up to token n copied into compact arrays (block table
    remapped), then the oracle append of q_len new tokens at n - q_len and the
    float64 decode over n tokens -- the same computation as a whole pair on a
    shorter context, for a step budget smaller than one whole pair."""
    from oracle import attention, e4m3, paged
    ps, Hkv, D, G = w.page_size, w.num_kv_heads, w.head_dim, w.group
    q64 = w.q_f64()
    newk, newv = w.new_tokens("k"), w.new_tokens("v")
    cache = {}

    def prepare(b, h, n):
        key = (b, h, n)
        if key not in cache:
            t = np.arange(n)
            npg = (n + ps - 1) // ps
            kp = np.zeros((npg, 1, ps, D), np.uint8)
            vp = np.zeros_like(kp)
            kp[t // ps, 0, t % ps, :] = e4m3.encode(w.seq_k(b)[:n, h, :], w.k_scale[h])
            vp[t // ps, 0, t % ps, :] = e4m3.encode(w.seq_v(b)[:n, h, :], w.v_scale[h])
            cache[key] = (kp, vp, np.arange(npg, dtype=np.int32)[None, :])
        return cache[key]

    def run(b, h, n):
        kp, vp, bt = prepare(b, h, n)
        hs = slice(h, h + 1)
        lens = np.array([n], np.int32)
        t0 = time.perf_counter()
        k2 = paged.append(kp, newk[b:b + 1, :, hs], w.k_scale[hs], bt, lens - w.q_len, ps)
        v2 = paged.append(vp, newv[b:b + 1, :, hs], w.v_scale[hs], bt, lens - w.q_len, ps)
        attention.paged_gqa_decode(q64[b:b + 1, :, h * G:(h + 1) * G], k2, v2, w.k_scale[hs],
                                   w.v_scale[hs], bt, lens, w.q_len, ps)
        return time.perf_counter() - t0

    def nbytes(b, h, n):
        return n * D * 2 + 2 * w.q_len * G * D * 2

    return run, nbytes


def _pairs(w):
    """(b, h) pairs in a fixed order that spreads over sequences first."""
    return [(b, h) for h in range(w.num_kv_heads) for b in range(w.batch)]


def cpu_baseline(w, seconds):
    """The oracle, as it stands, on a bounded sample of the workload: whole
    (sequence, KV head) pairs until `seconds` of CPU time are spent, on one
    host thread (BLAS limited to 1 thread; numpy elementwise is single-threaded)."""
    from threadpoolctl import threadpool_limits
    run, nbytes = oracle_pair_timer(w)
    pairs = _pairs(w)
    total_t, total_b, n = 0.0, 0, 0
    with threadpool_limits(1):
        run(*pairs[0])  # warm-up (untimed)
        while n < len(pairs) and total_t < seconds:
            total_t += run(*pairs[n])
            total_b += nbytes(*pairs[n])
            n += 1
    return {"value": total_b / total_t / 1e9, "unit": "GB/s", "cores": 1,
            "kind": "oracle",
            "tokens_per_s_per_layer": n * w.q_len / w.num_kv_heads / total_t,
            "sample": f"{n} of {len(pairs)} (sequence, KV head) pairs, one step each (oracle "
                      f"append of the new tokens + float64 decode of the head's {w.group} "
                      f"q-heads), {total_t:.1f} s on 1 host thread"}


def reference_arm(args):
    """--impl reference: the CPU oracle, timed as it stands, on the headline
    workload (or --config), same metric and config as our arm."""
    from threadpoolctl import threadpool_limits
    from paged_fp8_kv_05_b200 import workloads
    # No process group: rank 0 alone runs the CPU oracle, the others exit.
    if int(os.environ.get("RANK", "0")) != 0:
        return
    index = HEADLINE if args.config is None else args.config
    w = workloads.config_workload(index)
    run, nbytes = oracle_pair_timer(w)
    pairs = _pairs(w)
    # size each step so that warm-up + timed steps end within ~2 minutes
    budget = 120.0 / max(args.steps + args.warmup, 1)
    with threadpool_limits(1):
        t_one = max(run(*pairs[0]), 1e-3)
        times, bytes_, n_pairs, n_tok = [], [], 0, 0
        if t_one <= budget:  # whole pairs
            per_step = max(1, min(len(pairs), int(budget / t_one)))
            for i in range(args.warmup + args.steps):
                sel = [pairs[(i * per_step + j) % len(pairs)] for j in range(per_step)]
                dt = sum(run(b, h) for b, h in sel)
                if i >= args.warmup:
                    times.append(dt)
                    bytes_.append(sum(nbytes(b, h) for b, h in sel))
                    n_pairs += len(sel)
                    n_tok += sum(w.q_len for _ in sel)
            sample = (f"{per_step} (sequence, KV head) pair(s) per step of {len(pairs)}, "
                      f"float64 numpy on 1 host thread")
        else:  # one pair's first n context tokens per step
            prun, pbytes = oracle_prefix_timer(w)
            L_min = int(min(w.seq_lens[b] for b, _ in pairs))
            n = max(w.page_size, min(L_min, int(L_min * budget / t_one)))
            n = max(w.q_len, n // w.page_size * w.page_size)
            for i in range(args.warmup + args.steps):
                b, h = pairs[i % len(pairs)]
                dt = prun(b, h, n)
                if i >= args.warmup:
                    times.append(dt)
                    bytes_.append(pbytes(b, h, n))
                    n_pairs += 1
                    n_tok += w.q_len
            sample = (f"the first {n} context tokens of one (sequence, KV head) pair per step "
                      f"(a whole pair, {t_one:.1f} s, exceeds the step budget of {budget:.2f} s), "
                      f"float64 numpy on 1 host thread")
    T = sum(times)
    value = sum(bytes_) / T / 1e9
    b_dec, b_app = algorithmic_bytes(w)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * T / len(times), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator)",
            "tokens_per_s_per_layer": n_tok / w.num_kv_heads / T,
            "config": workload_config(w, index, b_dec, b_app, args),
            "cpu_baseline": {"kind": "oracle", "cores": 1, "value": value, "unit": "GB/s",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm

def append_throughput(w, device, flush_l2, ak, n_new=1024, calls=20):
    """A0 alone: one atlas_fp8_kv_append of n_new float32 tokens per sequence
    (the cache-fill shape), into a pool of its own so the workload's cache is
    untouched.  Bytes per call: 4 (f32 in) + 1 (code out) per element, plus
    the block-table entries and start positions.  Event-timed per call with
    the L2 flushed before each; reported beside the step, not in `value`."""
    B, Hkv, D, ps = w.batch, w.num_kv_heads, w.head_dim, w.page_size
    pages_per_seq = (n_new + ps - 1) // ps
    pool = ak.KVPool(B * pages_per_seq, ps, Hkv, D, w.k_scale, w.v_scale, max_batch=B,
                     max_q_len=1, num_q_heads=Hkv, max_seq_len=n_new, device=device)
    table = torch.arange(B * pages_per_seq, dtype=torch.int32, device=device).view(B, pages_per_seq)
    start = torch.zeros(B, dtype=torch.int32, device=device)
    gen = torch.Generator(device=device).manual_seed(7)
    k = torch.randn(B, n_new, Hkv, D, device=device, generator=gen)
    v = torch.randn(B, n_new, Hkv, D, device=device, generator=gen)
    stream = torch.cuda.current_stream(device)
    for _ in range(3):
        ak.atlas_fp8_kv_append(pool, k, v, table, start)
    times = []
    for _ in range(calls):
        flush_l2()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        ak.atlas_fp8_kv_append(pool, k, v, table, start)
        z.record(stream)
        z.synchronize()
        times.append(a.elapsed_time(z))
    if pool.device_error() != 0:
        raise SystemExit("device error flag set during the append timing")
    elems = 2 * B * n_new * Hkv * D
    nbytes = elems * (4 + 1) + 4 * B * pages_per_seq + 4 * B
    ms = sum(times) / len(times)
    peak, _ = load_peaks()
    return {"what": f"atlas_fp8_kv_append, {B} x {n_new} x {Hkv} x {D} float32 K and V",
            "us_per_call": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9,
            "frac": nbytes / (ms * 1e-3) / 1e9 / peak, "bytes_per_call": nbytes,
            "launches_per_call": 1}


def _time_calls(fn, flush_l2, device, calls=20, warm=3):
    """Mean event-timed duration (ms) of fn() over `calls` calls, L2 flushed
    before each (outside the events)."""
    stream = torch.cuda.current_stream(device)
    for _ in range(warm):
        fn()
    times = []
    for _ in range(calls):
        flush_l2()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        z.record(stream)
        z.synchronize()
        times.append(a.elapsed_time(z))
    return sum(times) / len(times)


def next_rows(device, flush_l2, ak):
    """The rows after the hot path's core: finer-grained scales (decode over a
    per-token-scaled cache, LLaMA-3-8B decode shape), fused RoPE + FP8 append
    (a 1024-token fill of that shape), ragged MTP verify (27B-class shape,
    q_len 1..5 per sequence, batch 128) and a 512-row prefill chunk over 4096
    tokens.  Each: one launch per call, event-timed with L2 flushed before
    every call; bytes are the algorithmic bytes of the call."""
    from paged_fp8_kv_05_b200 import workloads
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload
    peak, _ = load_peaks()
    out = {}

    def rec(what, ms, nbytes, extra=None):
        r = {"what": what, "us_per_call": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9,
             "frac": nbytes / (ms * 1e-3) / 1e9 / peak, "bytes_per_call": nbytes,
             "launches_per_call": 1}
        if extra:
            r.update(extra)
        return r

    # finer-grained scales: decode over a cache with one scale per (token, KV head)
    w = workloads.config_workload(1)
    dw = DeviceWorkload(w, device=device, token_scales=True)
    b_dec, _ = algorithmic_bytes(w)
    tok_bytes = b_dec + 2 * 4 * int(w.seq_lens.astype(np.int64).sum()) * w.num_kv_heads
    ms = _time_calls(lambda: dw.decode(), flush_l2, device)
    plain = DeviceWorkload(w, device=device)
    ms_plain = _time_calls(lambda: plain.decode(), flush_l2, device)
    out["token_scales"] = rec("atlas_paged_gqa_decode_tokscale, " + workloads.workload_tag(1),
                              ms, tok_bytes, {"per_head_scales_us": ms_plain * 1e3,
                                              "per_head_kernel": plain.plan()["kernel"]})
    del dw, plain

    # fused RoPE + quantise + append of a 1024-token fill, LLaMA-3-8B heads
    B, n_new, Hq, Hkv, D, ps = 32, 1024, 32, 8, 128, 16
    qkv, cos_sin = workloads.make_rope_inputs(batch=B, n_new=n_new, num_q_heads=Hq,
                                              num_kv_heads=Hkv, head_dim=D, max_pos=n_new, seed=2)
    pool = ak.KVPool(B * n_new // ps, ps, Hkv, D, np.full(Hkv, 0.01, np.float32),
                     np.full(Hkv, 0.01, np.float32), max_batch=B, max_q_len=1, num_q_heads=Hq,
                     max_seq_len=n_new, device=device)
    table = torch.arange(B * n_new // ps, dtype=torch.int32, device=device).view(B, -1)
    start = torch.zeros(B, dtype=torch.int32, device=device)
    d_qkv, d_cs = qkv.to(device).contiguous(), torch.from_numpy(cos_sin).to(device)
    q_out = torch.empty(B, n_new, Hq, D, dtype=torch.bfloat16, device=device)
    ms = _time_calls(lambda: ak.atlas_rope_fp8_kv_append(pool, d_qkv, Hq, d_cs, table, start,
                                                         q_out=q_out), flush_l2, device)
    elems = B * n_new * (Hq + 2 * Hkv) * D
    nbytes = elems * 2 + B * n_new * Hq * D * 2 + B * n_new * 2 * Hkv * D + B * n_new * D * 4
    out["rope_append"] = rec(f"atlas_rope_fp8_kv_append, bf16 QKV {B} x {n_new} x "
                             f"({Hq} + 2 x {Hkv}) x {D}", ms, nbytes)
    del pool, d_qkv, q_out

    # ragged MTP verify and a prefill chunk (packed rows)
    for name, mk, qls in (
            ("ragged_verify",
             lambda: workloads.make_workload(batch=128, num_q_heads=40, num_kv_heads=8,
                                             head_dim=128, page_size=16, q_len=1,
                                             num_pages=16384, lengths=("uniform", 128, 1152),
                                             seed=13),
             lambda: np.random.default_rng(13).integers(1, 6, size=128)),
            ("prefill_512_over_4096",
             lambda: workloads.make_workload(batch=8, num_q_heads=32, num_kv_heads=8,
                                             head_dim=128, page_size=16, q_len=1,
                                             num_pages=8 * 256 + 8,
                                             lengths=("fixed", [4096] * 8), seed=14),
             lambda: np.full(8, 512))):
        w = mk()
        q_lens = qls()
        q, cu = workloads.make_packed_queries(q_lens=q_lens, num_q_heads=w.num_q_heads,
                                              head_dim=w.head_dim, seed=5)
        dw = DeviceWorkload(w, device=device, max_q_len=int(q_lens.max()))
        dq, dcu = q.to(device).contiguous(), torch.from_numpy(cu).to(device)
        o = torch.empty_like(dq)
        ms = _time_calls(lambda: ak.atlas_paged_gqa_decode_varlen(
            dw.pool, dq, dcu, dw.block_table, dw.seq_lens, int(q_lens.max()), w.max_seq_len,
            out=o), flush_l2, device)
        L = w.seq_lens.astype(np.int64)
        nbytes = (int(L.sum()) * w.num_kv_heads * w.head_dim * 2 + 2 * dq.numel() * 2
                  + 4 * int(((L + 15) // 16).sum()))
        flops = 4 * int(sum(int(L[b]) * int(q_lens[b]) for b in range(w.batch))) * w.num_q_heads * w.head_dim
        out[name] = rec(f"atlas_paged_gqa_decode_varlen, {w.batch} sequences, q_len "
                        f"{int(q_lens.min())}..{int(q_lens.max())}", ms, nbytes,
                        {"tflops": flops / (ms * 1e-3) / 1e12,
                         "plan": ak.atlas_paged_gqa_decode_plan(dw.pool, w.batch, w.num_q_heads,
                                                                int(q_lens.max()),
                                                                w.max_seq_len)})
        del dw, dq, o
    torch.cuda.empty_cache()
    return out


def accept_throughput(device, flush_l2, ak, batch=128, num_drafts=4, vocab=151936, calls=20):
    """Greedy MTP acceptance alone (the step after a verify decode): bf16
    verify logits [batch, K + 1, vocab] read once, plus the drafts in and the
    targets, accepted counts and next tokens out.  Event-timed per call with
    the L2 flushed before each; reported beside the decode step."""
    from paged_fp8_kv_05_b200 import workloads
    logits, drafts, _ = workloads.make_verify_logits(batch=batch, num_drafts=num_drafts,
                                                     vocab=vocab, seed=3)
    lg = logits.to(device).contiguous()
    dr = torch.from_numpy(drafts).to(device).contiguous()
    pool = ak.KVPool(4, 16, 1, 64, [1.0], [1.0], max_batch=batch, max_q_len=1, num_q_heads=1,
                     max_seq_len=16, device=device)
    n, nxt, tg = ak.atlas_mtp_greedy_accept(pool, lg, dr)
    stream = torch.cuda.current_stream(device)
    for _ in range(3):
        ak.atlas_mtp_greedy_accept(pool, lg, dr, targets=tg, n_accepted=n, next_token=nxt)
    times = []
    for _ in range(calls):
        flush_l2()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        ak.atlas_mtp_greedy_accept(pool, lg, dr, targets=tg, n_accepted=n, next_token=nxt)
        z.record(stream)
        z.synchronize()
        times.append(a.elapsed_time(z))
    if pool.device_error() != 0:
        raise SystemExit("device error flag set during the acceptance timing")
    nbytes = lg.numel() * lg.element_size() + dr.numel() * 4 + tg.numel() * 4 + 2 * batch * 4
    ms = sum(times) / len(times)
    peak, _ = load_peaks()
    return {"what": f"atlas_mtp_greedy_accept, bf16 logits {batch} x {num_drafts + 1} x {vocab}",
            "us_per_call": ms * 1e3, "gbs": nbytes / (ms * 1e-3) / 1e9,
            "frac": nbytes / (ms * 1e-3) / 1e9 / peak, "bytes_per_call": nbytes,
            "launches_per_call": 1}


def stage_inputs(parts, pin=False):
    """Pack tensors into one uint8 buffer, each at a 256-byte-aligned offset
    (the end-to-end leg's single host-to-device copy).  Returns the buffer
    (pinned if asked) and the offsets."""
    offs, n = [], 0
    for t in parts:
        offs.append(n)
        n = (n + t.numel() * t.element_size() + 255) // 256 * 256
    buf = torch.zeros(n, dtype=torch.uint8)
    if pin:
        buf = buf.pin_memory()
    for t, o in zip(parts, offs):
        nb = t.numel() * t.element_size()
        buf[o:o + nb].copy_(t.contiguous().reshape(-1).view(torch.uint8))
    return buf, offs


def staged_views(buf, parts, offs):
    """Views into a staging buffer (or its device copy) with the dtypes and
    shapes of `parts`."""
    return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
            for t, o in zip(parts, offs)]


def measure(index, args, device, dist, ak, flush_l2, local):
    """Time K fused steps (append + decode, one launch each) of one workload,
    then K_e2e steps end to end through the public API with pinned host
    buffers.  Returns the per-workload record."""
    from paged_fp8_kv_05_b200 import workloads
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload

    w = workloads.config_workload(index)
    dw = DeviceWorkload(w, device=device)
    if args.split_tokens:
        dw.pool.set_split_tokens(args.split_tokens)
    if args.stages:
        dw.pool.set_option(ak.OPT_STAGES, args.stages)
    if args.waves:
        dw.pool.set_option(ak.OPT_WAVES, args.waves)
    if args.partition:
        dw.pool.set_option(ak.OPT_PARTITION, args.partition)
    if args.rows_per_cta:
        dw.pool.set_option(ak.OPT_ROWS_PER_CTA, args.rows_per_cta)
    if args.kernel:
        dw.pool.set_option(ak.OPT_KERNEL, args.kernel)
    plan = dw.plan()
    b_dec, b_app = algorithmic_bytes(w)
    stream = torch.cuda.current_stream(device)

    for _ in range(args.warmup):
        flush_l2()
        dw.step()
    torch.cuda.synchronize(device)
    if dw.pool.device_error() != 0:
        raise SystemExit(f"device error flag set during warm-up (workload {index})")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(local) as clk:
        for k in range(K):
            flush_l2()
            e0, e1 = evs[k]
            e0.record(stream)
            dw.step()            # one kernel: FP8 append of the new tokens + decode
            e1.record(stream)
        torch.cuda.synchronize(device)
    if dist is not None:
        dist.barrier()
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    total_ms = max_over_ranks(sum(step_ms), dist, device)
    ms_per_step = total_ms / K
    assert plan["launches"] == 1

    # end to end through the public API from pinned host memory.  The step's
    # inputs (q, the new K and V, seq_lens, the block table) sit in one pinned
    # staging buffer, each at a 256-byte-aligned offset, and go to the device
    # in one copy (as a serving loop stages a step's small inputs); the call
    # gets views into the device copy; the output comes back in one copy.
    parts = [w.q.contiguous(), torch.from_numpy(w.new_tokens("k")),
             torch.from_numpy(w.new_tokens("v")),
             torch.from_numpy(w.seq_lens.astype(np.int32)),
             torch.from_numpy(np.ascontiguousarray(w.block_table))]
    stage_h, offs = stage_inputs(parts, pin=True)
    stage_d = torch.empty(stage_h.numel(), dtype=torch.uint8, device=device)
    q_d, k_d, v_d, sl_d, bt_d = staged_views(stage_d, parts, offs)
    out_h = torch.empty(w.q.shape, dtype=torch.bfloat16).pin_memory()
    out_d = torch.empty_like(dw.q)
    h2d = stage_h.numel()
    d2h = out_h.numel() * out_h.element_size()
    K_e2e = min(K, 200)
    e2e_ms = []
    for k in range(K_e2e + 3):
        flush_l2()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        stage_d.copy_(stage_h, non_blocking=True)
        ak.atlas_paged_gqa_append_decode(dw.pool, k_d, v_d, q_d, bt_d, sl_d, w.max_seq_len,
                                         out=out_d)
        out_h.copy_(out_d, non_blocking=True)
        z.record(stream)
        z.synchronize()
        if k >= 3:
            e2e_ms.append(a.elapsed_time(z))
    e2e_total = max_over_ranks(sum(e2e_ms), dist, device)
    if dw.pool.device_error() != 0:
        raise SystemExit(f"device error flag set during timing (workload {index})")

    world = 1 if dist is None else dist.get_world_size()
    peak, peak_kind = load_peaks()
    step_bytes = b_dec + b_app
    achieved = step_bytes / (ms_per_step * 1e-3) / 1e9
    rec = {
        "workload": workloads.workload_tag(index),
        "config": workload_config(w, index, b_dec, b_app, args),
        "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "us_per_step": ms_per_step * 1e3,
        "value": world * achieved, "unit": "GB/s",
        "tokens_per_s_per_layer": world * w.batch * w.q_len / (ms_per_step * 1e-3),
        "plan": plan,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "frac_of_8tbs": achieved / 8000.0,
                     "kernel": ("paged_decode_tc_kernel" if plan["kernel"] == 3 else
                                "paged_decode_fp8_kernel") +
                               " (fused append + decode, one launch per step, launch-averaged "
                               "over the timed steps)",
                     "traffic": recorded_traffic(index),
                     "algorithmic_bytes": step_bytes,
                     "algorithmic_flops": algorithmic_flops(w)},
        "e2e": {"value": world * step_bytes / (e2e_total / K_e2e * 1e-3) / 1e9, "unit": "GB/s",
                "ms_per_step": e2e_total / K_e2e, "steps": K_e2e,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": K,
        "clocks": clk.summary(),
    }
    del dw
    torch.cuda.empty_cache()
    return w, rec


def ours(args):
    world, rank, local, dist = dist_setup(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from paged_fp8_kv_05_b200 import build
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv as ak

    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    flush_r = torch.ones(FLUSH_BYTES, dtype=torch.uint8, device=device)

    def flush_l2():
        flush.zero_()                        # evicts everything the last step left
        flush_r.sum(dtype=torch.int32)       # evicts the dirty lines of that write

    order = TARGETS if args.config is None else (args.config,)
    head = HEADLINE if args.config is None else args.config
    per, head_w, append_line = {}, None, None
    for index in order:
        w, rec = measure(index, args, device, dist, ak, flush_l2, local)
        per[str(index)] = rec
        if index == head:
            head_w = w
        if index == 1 or (append_line is None and index == order[-1]):
            append_line = append_throughput(w, device, flush_l2, ak)
        del w

    h = per[str(head)]
    line = {
        "metric": METRIC, "value": h["value"], "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": h["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3",
        "data": "synthetic (seeded generator; random N(0,1) q/K/V, no weights)",
        "config": h["config"],
        "tokens_per_s_per_layer": h["tokens_per_s_per_layer"],
        "step_us": h["us_per_step"],
        "plan": h["plan"],
        "roofline": h["roofline"],
        "e2e": h["e2e"],
        "gpu_launches": h["gpu_launches"],
        "clocks": h["clocks"],
        "per_config": per,
        "append": append_line,
        "accept": accept_throughput(device, flush_l2, ak),
    }
    if not args.no_next_rows:
        line["next_rows"] = next_rows(device, flush_l2, ak)
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(head_w, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
    else:
        ours(args)


if __name__ == "__main__":
    main()
