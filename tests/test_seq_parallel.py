"""Sequence parallelism over K/V splits on CPU (gloo, world size 2).

LiteAttention README, SeqParallelLiteAttention: each call attends to one K/V split, named by its
split index, with a skip state per split; partial results combine by their LSE. Here every rank
holds one token shard of q, k, v; seq_parallel_forward all-gathers the K/V shards, runs one
partial attention per split and merges them. The per-split attention and the merge are the
oracle's (the CUDA versions of both are covered by the GPU parity tests), so this checks the
exchange, the split bookkeeping and the composition:
  * step 0 (fresh masks) equals full attention of the rank's queries over all tokens;
  * at later steps each split's mask equals what a single process computes for
    (queries of this rank, keys of that split) over the same steps;
  * the rank's own split is processed first.
"""

import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from temporal_block_sparse_b200 import workload as wl
from temporal_block_sparse_b200.attention import seq_parallel_forward, split_order

WORLD = 2
N_SHARD = 200  # ragged: 3 full tiles of 64 plus 8 rows
TAU = -2.0
STEPS = 3
BASE = wl.small_workload(1, 2, 5, 8, 10, 64, steps=STEPS, locality=5.0, tau=TAU, seed_offset=77)  # N = 400


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _np(x):
    return x.double().numpy()


def _steps_qkv():
    tr = wl.Trajectory(BASE, device="cpu")
    out = []
    for _ in range(STEPS):
        q, k, v = tr.current()
        out.append(tuple(x.float() for x in (q, k, v)))
        tr.advance()
    return out


class OracleSplits:
    """Per-split skip state with the oracle as the attention (the host-side stand-in for
    SeqParallelLiteAttention in this CPU test)."""

    def __init__(self, world):
        self.masks = [None] * world
        self.calls = []

    def __call__(self, q, k, v, s):
        self.calls.append(s)
        r = oracle.lite_attention_forward(_np(q), _np(k), _np(v), self.masks[s], tau=TAU)
        self.masks[s] = r.mask_out
        return torch.from_numpy(r.out), torch.from_numpy(r.lse)


def _merge(parts):
    o, l = oracle.lse_merge([(o.numpy(), l.numpy()) for o, l in parts])
    return torch.from_numpy(o), torch.from_numpy(l)


def _worker(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        attn = OracleSplits(world)
        sl = slice(rank * N_SHARD, (rank + 1) * N_SHARD)
        for t, (q, k, v) in enumerate(_steps_qkv()):
            o, lse = seq_parallel_forward(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(),
                                          attn, merge=_merge)
            np.save(os.path.join(outdir, f"o{rank}_{t}.npy"), o.numpy())
            np.save(os.path.join(outdir, f"lse{rank}_{t}.npy"), lse.numpy())
            for s in range(world):
                np.save(os.path.join(outdir, f"mask{rank}_{s}_{t}.npy"), attn.masks[s])
        np.save(os.path.join(outdir, f"calls{rank}.npy"), np.array(attn.calls))
    finally:
        dist.destroy_process_group()


def test_split_order_starts_with_own_split():
    assert split_order(0, 4) == [0, 1, 2, 3]
    assert split_order(2, 4) == [2, 3, 0, 1]
    assert split_order(1, 2) == [1, 0]


def test_two_ranks_seq_parallel_matches_single_process():
    port = _free_port()
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(WORLD, port, d), nprocs=WORLD, join=True, start_method="spawn")
        qkv = _steps_qkv()
        # step 0: fresh masks, nothing skipped -> full attention over all tokens
        q, k, v = qkv[0]
        full = oracle.lite_attention_forward(_np(q), _np(k), _np(v), None, tau=-np.inf)
        for r in range(WORLD):
            sl = slice(r * N_SHARD, (r + 1) * N_SHARD)
            np.testing.assert_allclose(np.load(os.path.join(d, f"o{r}_0.npy")), full.out[:, sl], rtol=1e-10,
                                       atol=1e-12)
            np.testing.assert_allclose(np.load(os.path.join(d, f"lse{r}_0.npy")), full.lse[:, :, sl], rtol=1e-12)
            assert list(np.load(os.path.join(d, f"calls{r}.npy"))[:WORLD]) == split_order(r, WORLD)
        # every step: per-split masks and outputs equal a single-process run of the same splits
        for r in range(WORLD):
            qs = slice(r * N_SHARD, (r + 1) * N_SHARD)
            masks = [None] * WORLD
            flagged_any = False
            for t, (q, k, v) in enumerate(qkv):
                parts = []
                for s in range(WORLD):
                    ks = slice(s * N_SHARD, (s + 1) * N_SHARD)
                    res = oracle.lite_attention_forward(_np(q[:, qs]), _np(k[:, ks]), _np(v[:, ks]), masks[s],
                                                        tau=TAU)
                    masks[s] = res.mask_out
                    parts.append((res.out, res.lse))
                    got = np.load(os.path.join(d, f"mask{r}_{s}_{t}.npy"))
                    np.testing.assert_array_equal(got, res.mask_out)
                    flagged_any |= bool(res.mask_out.any())
                o, l = oracle.lse_merge(parts)
                np.testing.assert_allclose(np.load(os.path.join(d, f"o{r}_{t}.npy")), o, rtol=1e-10, atol=1e-12)
                np.testing.assert_allclose(np.load(os.path.join(d, f"lse{r}_{t}.npy")), l, rtol=1e-12)
            assert flagged_any, "the case must exercise per-split flags"
