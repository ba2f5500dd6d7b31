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
