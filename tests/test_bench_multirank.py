"""The bench's multi-rank plumbing on CPU with the gloo backend, world size 2:
timing is the max over ranks, each rank draws its own seeded batch (weak
scaling, no data-path collective), and the aggregate divides all ranks' work
by that max time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, lr = bench.dist_env()
    assert (r, w, lr) == (rank, world, rank)
    dist = bench.init_dist(w, "gloo")
    bench.barrier(w)
    elapsed = 1.0 + rank          # rank 1 is the slow one
    t_max = bench.max_over_ranks(elapsed, w)
    seed = bench.rank_seed(r)
    import workloads as W
    x = W.activations_with_outliers(4, 256, seed=seed)
    flops_step = 10.0
    value = w * flops_step * 3 / t_max
    out[rank] = (t_max, seed, int(x.astype("int64").sum()), value)
    dist.destroy_process_group()


def test_two_rank_max_timing_and_weak_scaling():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    t0, s0, h0, v0 = out[0]
    t1, s1, h1, v1 = out[1]
    assert t0 == t1 == 2.0                 # both ranks see the slowest rank's time
    assert s0 != s1 and h0 != h1           # independent batches per rank
    assert v0 == v1 == 2 * 10.0 * 3 / 2.0  # whole-job throughput


def test_single_rank_helpers_are_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    assert bench.rank_seed(0) == 0


def test_reference_arm_line_on_cpu():
    """`bench.py --impl reference` (the oracle timed on the host cores) prints
    one JSON line with the contract's keys, on a one-row sample."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--ref-rows", "1"], capture_output=True, text=True, timeout=600, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and "workload" in d["config"]
