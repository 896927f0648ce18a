#!/usr/bin/env python
"""Benchmark of the paged FP8 decode step on B200.

One step = the whole hot path over one batch: the FP8 append of the step's
q_len new K/V tokens per sequence (quantise + scatter into the pages) and the
paged decode / verify attention over every sequence's full context, run as
one fused kernel (atlas_paged_gqa_append_decode).  The
default workload is the LLaMA-3-8B-shaped decode layer (B=32, Hq=32, Hkv=8,
D=128, page 16, context U[1024, 4096], q_len=1); ``--config`` selects another
of the five named workloads.

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
FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--split-tokens", type=int, default=0, help="override the split size")
    ap.add_argument("--stages", type=int, default=0, help="override the K/V staging depth")
    ap.add_argument("--waves", type=int, default=0, help="CTAs per resident CTA slot")
    ap.add_argument("--partition", type=int, default=0, help="0 auto, 1 grid, 2 balanced")
    ap.add_argument("--rows-per-cta", type=int, default=0, help="query rows per CTA (0 auto)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
DECODE_SOURCES = ("atlas_internal.cuh", "atlas_kv.cu", "decode_fp8.cu")


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

def oracle_step_timer(w):
    """Returns (run(sample_seqs) -> seconds, bytes(sample_seqs)) for the oracle
    decode step (append of the new tokens + decode) on chosen sequences."""
    from oracle import attention, e4m3, paged
    ps, Hkv, D = w.page_size, w.num_kv_heads, w.head_dim
    kp = np.zeros((w.num_pages, Hkv, ps, D), np.uint8)
    vp = np.zeros_like(kp)
    filled = set()
    q64 = w.q_f64()

    def prepare(seqs):
        for b in seqs:
            if b in filled:
                continue
            L = int(w.seq_lens[b])
            t = np.arange(L)
            pg = w.block_table[b, t // ps]
            kp[pg, :, t % ps, :] = e4m3.encode(w.seq_k(b), w.k_scale[None, :, None])
            vp[pg, :, t % ps, :] = e4m3.encode(w.seq_v(b), w.v_scale[None, :, None])
            filled.add(b)

    def run(seqs):
        prepare(seqs)
        t0 = time.perf_counter()
        sel = np.asarray(seqs)
        newk = w.new_tokens("k")[sel]
        newv = w.new_tokens("v")[sel]
        start = w.seq_lens[sel] - w.q_len
        k2 = paged.append(kp, newk, w.k_scale, w.block_table[sel], start, ps)
        v2 = paged.append(vp, newv, w.v_scale, w.block_table[sel], start, ps)
        attention.paged_gqa_decode(q64[sel], k2, v2, w.k_scale, w.v_scale, w.block_table[sel],
                                   w.seq_lens[sel], w.q_len, ps)
        return time.perf_counter() - t0

    def nbytes(seqs):
        L = w.seq_lens[np.asarray(seqs)].astype(np.int64)
        return int(L.sum()) * Hkv * D * 2 + 2 * len(seqs) * w.q_len * w.num_q_heads * D * 2

    return run, nbytes


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_baseline(w, seconds):
    run, nbytes = oracle_step_timer(w)
    seqs, total_t, total_b, tokens = [], 0.0, 0, 0
    b = 0
    run([0])  # warm-up (one sequence, untimed)
    while b < w.batch and total_t < seconds:
        total_t += run([b])
        total_b += nbytes([b])
        tokens += w.q_len
        seqs.append(b)
        b += 1
    return {"value": total_b / total_t / 1e9, "unit": "GB/s", "cores": blas_threads(),
            "kind": "oracle",
            "tokens_per_s_per_layer": tokens / total_t,
            "sample": f"{len(seqs)} of {w.batch} sequences (b=0..{len(seqs) - 1}), one step each "
                      f"(oracle append of the new tokens + float64 decode), "
                      f"{total_t:.1f} s, numpy elementwise single-threaded"}


def reference_arm(args):
    """--impl reference: the CPU oracle, timed as it stands, on this config."""
    from paged_fp8_kv_05_b200 import workloads
    # No process group: rank 0 alone runs the CPU oracle, the others exit.
    if int(os.environ.get("RANK", "0")) != 0:
        return
    w = workloads.config_workload(args.config)
    run, nbytes = oracle_step_timer(w)
    # size each step so that warm-up + timed steps end within ~2 minutes
    t_one = max(run([0]), 1e-3)
    budget = 120.0 / max(args.steps + args.warmup, 1)
    per_step = max(1, min(w.batch, int(budget / t_one)))
    order = [(i * per_step + j) % w.batch for i in range(args.steps + args.warmup)
             for j in range(per_step)]
    times, bytes_, toks = [], [], []
    for i in range(args.warmup + args.steps):
        seqs = sorted(set(order[i * per_step:(i + 1) * per_step]))
        dt = run(seqs)
        if i >= args.warmup:
            times.append(dt)
            bytes_.append(nbytes(seqs))
            toks.append(len(seqs) * w.q_len)
    T = sum(times)
    value = sum(bytes_) / T / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * T / len(times), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator)",
            "tokens_per_s_per_layer": sum(toks) / T,
            "config": {"workload": workloads.workload_tag(args.config), "oracle": "float64 numpy"},
            "cpu_baseline": {"kind": "oracle", "cores": blas_threads(), "value": value,
                             "unit": "GB/s",
                             "sample": f"{per_step} sequence(s) per step of {w.batch}"},
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


def ours(args):
    world, rank, local, dist = dist_setup(args)
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from paged_fp8_kv_05_b200 import build, workloads
    build.build()
    from paged_fp8_kv_05_b200 import atlas_kv as ak
    from paged_fp8_kv_05_b200.device_cache import DeviceWorkload

    w = workloads.config_workload(args.config)
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
    plan = dw.plan()
    b_dec, b_app = algorithmic_bytes(w)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    flush_r = torch.ones(FLUSH_BYTES, dtype=torch.uint8, device=device)

    def flush_l2():
        flush.zero_()                        # evicts everything the last step left
        flush_r.sum(dtype=torch.int32)       # evicts the dirty lines of that write
    stream = torch.cuda.current_stream(device)

    for _ in range(args.warmup):
        flush_l2()
        dw.step()
    torch.cuda.synchronize(device)
    if dw.pool.device_error() != 0:
        raise SystemExit("device error flag set during warm-up")

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
    launches = K         # the fused step is one launch (plan: 1 launch per call)
    assert plan["launches"] == 1

    # end to end through the public API with pinned host buffers
    q_h = w.q.clone().pin_memory()
    k_h = torch.from_numpy(w.new_tokens("k")).pin_memory()
    v_h = torch.from_numpy(w.new_tokens("v")).pin_memory()
    sl_h = torch.from_numpy(w.seq_lens.astype(np.int32)).pin_memory()
    bt_h = torch.from_numpy(np.ascontiguousarray(w.block_table)).pin_memory()
    out_h = torch.empty(w.q.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h, sl_h, bt_h))
    d2h = out_h.numel() * out_h.element_size()
    q_d = torch.empty_like(dw.q)
    k_d, v_d = torch.empty_like(dw.k_new), torch.empty_like(dw.v_new)
    sl_d = torch.empty_like(dw.seq_lens)
    bt_d = torch.empty_like(dw.block_table)
    out_d = torch.empty_like(dw.q)
    K_e2e = min(K, 200)
    e2e_ms = []
    for k in range(K_e2e + 5):
        flush_l2()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for dst, src in ((q_d, q_h), (k_d, k_h), (v_d, v_h), (sl_d, sl_h), (bt_d, bt_h)):
            dst.copy_(src, non_blocking=True)
        ak.atlas_paged_gqa_append_decode(dw.pool, k_d, v_d, q_d, bt_d, sl_d, w.max_seq_len,
                                         out=out_d)
        out_h.copy_(out_d, non_blocking=True)
        z.record(stream)
        z.synchronize()
        if k >= 5:
            e2e_ms.append(a.elapsed_time(z))
    e2e_total = max_over_ranks(sum(e2e_ms), dist, device)
    if dw.pool.device_error() != 0:
        raise SystemExit("device error flag set during timing")
    append_line = append_throughput(w, device, flush_l2, ak)

    peak, peak_kind = load_peaks()
    step_bytes = b_dec + b_app
    achieved = step_bytes / (ms_per_step * 1e-3) / 1e9
    value = world * step_bytes / (ms_per_step * 1e-3) / 1e9
    tokens = world * w.batch * w.q_len / (ms_per_step * 1e-3)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3",
        "data": "synthetic (seeded generator; random N(0,1) q/K/V, no weights)",
        "config": workload_config(w, args.config, b_dec, b_app, args),
        "tokens_per_s_per_layer": tokens,
        "step_us": ms_per_step * 1e3,
        "plan": plan,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "frac_of_8tbs": achieved / 8000.0,
                     "kernel": "paged_decode_fp8_kernel (fused append + decode, launch-averaged)",
                     "traffic": recorded_traffic(args.config),
                     "algorithmic_bytes": step_bytes,
                     "algorithmic_flops": algorithmic_flops(w)},
        "e2e": {"value": world * step_bytes / (e2e_total / K_e2e * 1e-3) / 1e9, "unit": "GB/s",
                "ms_per_step": e2e_total / K_e2e, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "append": append_line,
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
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
