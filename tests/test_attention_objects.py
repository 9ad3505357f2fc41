"""Host-side checks of the per-layer attention objects (CPU; they raise before any library call)."""

import pytest
import torch

from temporal_block_sparse_b200.attention import LiteAttention, SeqParallelLiteAttention, split_order


def _qkv(B=1, N=8, H=1, d=64):
    x = torch.zeros((B, N, H, d), dtype=torch.bfloat16)
    return x, x, x


def test_batch_beyond_max_batch_size_is_refused():
    attn = LiteAttention(max_batch_size=2)
    with pytest.raises(ValueError):
        attn(*_qkv(B=3))


def test_seq_parallel_checks_split_index_and_node_count():
    with pytest.raises(ValueError):
        SeqParallelLiteAttention(num_nodes=0)
    attn = SeqParallelLiteAttention(num_nodes=2)
    for bad in (-1, 2, 5):
        with pytest.raises(IndexError):
            attn(*_qkv(), split_idx=bad)


def test_state_before_first_call():
    attn = LiteAttention(threshold=-3.0)
    assert attn.skipped_fraction() is None
    attn.reset_skip_state()  # no state yet: a no-op
    attn.set_threshold(-5.0)
    assert attn.threshold == -5.0
    attn.enable_skip_optimization(False)
    assert not attn.enable_skipping
    sp = SeqParallelLiteAttention(num_nodes=3)
    assert [sp.skipped_fraction(i) for i in range(3)] == [None, None, None]


def test_split_order_is_a_rotation():
    for world in (1, 2, 3, 8):
        for rank in range(world):
            order = split_order(rank, world)
            assert sorted(order) == list(range(world)) and order[0] == rank
