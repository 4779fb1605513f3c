"""The N > 1 host path on CPU: two gloo ranks (world size 2).

Each rank decodes its own sequences (weak scaling, no collective on the data
path); the job time is the max over ranks.  Runs without a GPU."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import bench
    from two_level_sparse_quest_b200 import workloads as W

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        base = W.WORKLOADS["gqa48k_bf16"].with_(ctx=512, k_b=4, k_t=32)
        w = bench.rank_workload(base, rank)
        inp = W.make_decode_inputs(w)
        t = bench.max_over_ranks(10.0 + rank)
        dist.barrier()
        out[rank] = (w.seed, float(W.to_f64(inp.K[0, 0, :4, :4], w.dtype).sum()), t)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_have_independent_work_and_max_time():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    (s0, k0, t0), (s1, k1, t1) = out[0], out[1]
    assert s0 != s1 and k0 != k1
    assert t0 == t1 == 11.0


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero():
    """`bench.py --impl reference` launched like the multi-GPU bench: rank 0
    times the oracle and prints the one JSON line; the other rank exits 0
    without work (no GPU, no process group needed)."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-3000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
