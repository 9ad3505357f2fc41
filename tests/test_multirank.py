"""Multi-rank host logic on CPU (gloo, world size 2): the weak-scaling partition used by bench.py.

Each rank owns an independent layer of the same shape (its own seed) and runs it end to end; the
only collective is the max over ranks of the timing scalar. Here each rank runs the oracle on its
own small layer, and the test checks that the ranks' problems are distinct, that every rank's
result equals what a single process computes for that rank's seed, and that the timing reduction
returns the slowest rank.
"""

import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from temporal_block_sparse_b200 import workload as wl

BASE = wl.small_workload(1, 2, 2, 6, 8, 64, steps=2, locality=3.0, tau=-2.0, seed_offset=40)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_result(rank):
    w = bench.rank_workload(BASE, rank)
    q, k, v = wl.Trajectory(w, device="cpu").current()
    r = oracle.lite_attention_forward(*(x.float().numpy().astype(np.float64) for x in (q, k, v)), None,
                                      tau=-2.0, tile=8)
    return q, r


def _worker(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, r = _rank_result(rank)
        slowest = bench.max_over_ranks(10.0 + rank, dist, torch.device("cpu"))
        qs = [torch.zeros_like(q) for _ in range(world)]
        dist.all_gather(qs, q)
        np.save(os.path.join(outdir, f"lse{rank}.npy"), r.lse)
        np.save(os.path.join(outdir, f"mask{rank}.npy"), r.mask_out)
        distinct = not torch.equal(qs[0], qs[1])
        with open(os.path.join(outdir, f"ok{rank}"), "w") as f:
            f.write(f"{slowest} {int(distinct)}")
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_partition():
    port = _free_port()
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(2, port, d), nprocs=2, join=True, start_method="spawn")
        for rank in range(2):
            slowest, distinct = open(os.path.join(d, f"ok{rank}")).read().split()
            assert float(slowest) == 11.0 and distinct == "1"
            _, ref = _rank_result(rank)
            np.testing.assert_array_equal(np.load(os.path.join(d, f"lse{rank}.npy")), ref.lse)
            np.testing.assert_array_equal(np.load(os.path.join(d, f"mask{rank}.npy")), ref.mask_out)


def test_single_process_needs_no_collective():
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    assert bench.rank_workload(BASE, 0).seed == BASE.seed
    assert bench.rank_workload(BASE, 3).seed != BASE.seed
