"""CPU: the multi-process plumbing of bench.py with two `gloo` ranks.

The decode path shards by sequence with no exchange step, so `bench.py --gpus
N` runs N independent replicas: every rank joins one process group, times its
own steps, and the job time is the maximum over ranks.  These tests run that
plumbing (process-group setup from the torchrun environment, the max-over-ranks
reduction, the barrier, and the reference arm's rank-0-only rule) as two CPU
processes; nothing here touches a GPU.
"""

import json
import os
import socket
import subprocess
import sys
import textwrap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


_WORKER = textwrap.dedent("""
    import json, os, sys, types
    sys.path.insert(0, {root!r})
    import torch
    import bench
    args = types.SimpleNamespace(gpus=2)
    world, rank, local, dist = bench.dist_setup(args)
    # each rank reports a different step time; the job takes the slowest
    mine = 1.5 * (rank + 1)
    job = bench.max_over_ranks(mine, dist, torch.device("cpu"))
    dist.barrier()
    print(json.dumps({{"rank": rank, "world": world, "mine": mine, "job": job}}))
    dist.destroy_process_group()
""")


def _launch(nranks, code):
    port = _free_port()
    procs = []
    for r in range(nranks):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(nranks),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, cwd=ROOT,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                      text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err[-2000:]
        outs.append(out)
    return outs


def test_two_gloo_ranks_take_the_max_step_time():
    outs = _launch(2, _WORKER.format(root=ROOT))
    recs = sorted((json.loads(o.strip().splitlines()[-1]) for o in outs), key=lambda d: d["rank"])
    assert [d["rank"] for d in recs] == [0, 1]
    assert all(d["world"] == 2 for d in recs)
    assert all(d["job"] == 3.0 for d in recs)       # max(1.5, 3.0) on every rank


def test_reference_arm_runs_on_rank_zero_only():
    # rank 1 of a torchrun launch exits at once, without output and without
    # joining a process group (the oracle runs on rank 0's host cores alone)
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2",
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()), CUDA_VISIBLE_DEVICES="")
    res = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "1"], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=180)
    assert res.returncode == 0, res.stderr[-2000:]
    assert res.stdout.strip() == ""
