"""Multi-rank host logic on CPU (gloo, world size 2): the head partition of one layer used by
bench.py --gpus N.

Every (b, h) slice of a layer is independent, so the layer splits across ranks by heads with no
data-path collective: rank r keeps heads [r*H/N, (r+1)*H/N) of every batch entry, its own Skip-Mask
rows, and writes o and lse for those heads. Here each rank runs the oracle on its head slice over
two denoising steps (mask carried from step to step), the slices are gathered, and the result must
equal a single process running the whole layer bit for bit. The timing reduction returns the
slowest rank.
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
from temporal_block_sparse_b200 import sharding
from temporal_block_sparse_b200 import workload as wl

LAYER = wl.small_workload(2, 4, 2, 6, 8, 64, steps=2, locality=3.0, tau=-2.0, seed_offset=40)  # N=96


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _np(x):
    return x.float().numpy().astype(np.float64)


def _run(rank, world):
    """Two steps of the layer restricted to this rank's heads (the whole layer for world == 1)."""
    tr = wl.Trajectory(LAYER, device="cpu")
    mask = None
    outs, lses = [], []
    for _ in range(2):
        q, k, v = (sharding.shard_heads(x, rank, world, dim=2) for x in tr.current())
        r = oracle.lite_attention_forward(_np(q), _np(k), _np(v), mask, tau=-2.0, tile=16)
        mask = r.mask_out
        outs.append(r.out)
        lses.append(r.lse)
        tr.advance()
    return np.stack(outs), np.stack(lses), mask


def _worker(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        o, lse, mask = _run(rank, world)
        slowest = bench.max_over_ranks(10.0 + rank, dist, torch.device("cpu"))
        # gather the slices (inspection only; the benchmark's data path has no collective)
        parts = [None] * world
        dist.all_gather_object(parts, (o, lse, mask))
        if rank == 0:
            np.save(os.path.join(outdir, "o.npy"), np.concatenate([p[0] for p in parts], axis=3))
            np.save(os.path.join(outdir, "lse.npy"), np.concatenate([p[1] for p in parts], axis=2))
            np.save(os.path.join(outdir, "mask.npy"), np.concatenate([p[2] for p in parts], axis=1))
        with open(os.path.join(outdir, f"ok{rank}"), "w") as f:
            f.write(f"{slowest} {o.shape[3]}")
    finally:
        dist.destroy_process_group()


def test_two_ranks_split_one_layer_by_heads():
    port = _free_port()
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(2, port, d), nprocs=2, join=True, start_method="spawn")
        for rank in range(2):
            slowest, heads = open(os.path.join(d, f"ok{rank}")).read().split()
            assert float(slowest) == 11.0 and int(heads) == LAYER.H // 2
        o_ref, lse_ref, mask_ref = _run(0, 1)
        assert mask_ref.any()  # the steps flag tiles, so the carried mask matters
        np.testing.assert_array_equal(np.load(os.path.join(d, "o.npy")), o_ref)
        np.testing.assert_array_equal(np.load(os.path.join(d, "lse.npy")), lse_ref)
        np.testing.assert_array_equal(np.load(os.path.join(d, "mask.npy")), mask_ref)


def test_head_ranges_cover_the_layer_once():
    for H, world in ((40, 1), (40, 2), (40, 4), (40, 5), (40, 8), (4, 2)):
        ranges = [sharding.head_range(H, r, world) for r in range(world)]
        assert ranges[0][0] == 0 and ranges[-1][1] == H
        assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
        assert len({h1 - h0 for h0, h1 in ranges}) == 1
    with pytest.raises(ValueError):
        sharding.head_range(40, 0, 3)
    with pytest.raises(ValueError):
        sharding.head_range(40, 2, 2)
    x = torch.arange(2 * 3 * 4 * 5).reshape(2, 3, 4, 5)
    assert sharding.shard_heads(x, 0, 1, dim=2) is x
    assert torch.equal(sharding.shard_heads(x, 1, 2, dim=2), x[:, :, 2:4])


def test_single_process_needs_no_collective():
    assert bench.max_over_ranks(3.5, None, None) == 3.5
