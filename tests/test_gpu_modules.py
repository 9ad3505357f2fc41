"""LiteAttention / SeqParallelLiteAttention objects on the GPU vs the oracle (needs a B200).

The objects keep one Skip-Mask pair per layer (per K/V split for the sequence-parallel one) and
swap it after every call. Across steps the oracle is teacher-forced with the object's own mask
state, so a near-threshold flip cannot cascade.
"""

import numpy as np
import pytest
import torch

import oracle
from temporal_block_sparse_b200 import lite_attn as la
from temporal_block_sparse_b200 import workload as wl
from temporal_block_sparse_b200.attention import LiteAttention, SeqParallelLiteAttention

from gpu_parity import assert_within, compare, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

TAU = -2.0


@pytest.fixture(autouse=True)
def _clean_state():
    la.load()
    yield
    assert la.lite_get_device_status() == 0


def _mask_np(m):
    return None if m is None else m.cpu().numpy().view(np.uint32).copy()


def test_lite_attention_keeps_state_across_steps():
    w = wl.small_workload(1, 3, 6, 8, 16, 128, steps=4, locality=4.0, tau=TAU, seed_offset=300)
    tr = wl.Trajectory(w, device="cuda")
    attn = LiteAttention(threshold=TAU)
    before = None
    flagged = 0
    for t in range(w.steps):
        q, k, v = tr.current()
        o, lse = attn(q, k, v, return_softmax_lse=True)
        after = attn._state.cur  # the mask this call wrote
        ref = oracle.lite_attention_forward(to_np(q), to_np(k), to_np(v), before, tau=TAU)
        rep = compare(o, lse, after, ref)
        assert_within(rep)
        flagged += rep.flagged
        got = _mask_np(after)
        if before is not None:
            assert ((got & before) == before).all()  # the skipped set only grows
        before = got
        tr.advance()
    assert flagged > 0
    assert 0.0 < attn.skipped_fraction() < 1.0


def test_disabled_skipping_is_dense_and_leaves_state():
    w = wl.small_workload(1, 2, 4, 8, 16, 128, steps=2, locality=4.0, tau=TAU, seed_offset=301)
    q, k, v = wl.Trajectory(w, device="cuda").current()
    attn = LiteAttention(threshold=0.0)
    attn(q, k, v)
    state = attn._state.cur.clone()
    attn.enable_skip_optimization(False)
    o, lse = attn(q, k, v, return_softmax_lse=True)
    assert torch.equal(attn._state.cur, state)
    assert_within(compare(o, lse, None, oracle.lite_attention_forward(to_np(q), to_np(k), to_np(v), None,
                                                                     tau=-np.inf), check_mask=False))
    attn.reset_skip_state()
    assert attn.skipped_fraction() == 0.0


def test_must_do_list_through_the_object():
    w = wl.small_workload(1, 2, 4, 8, 16, 128, steps=2, locality=4.0, tau=TAU, seed_offset=302)
    q, k, v = wl.Trajectory(w, device="cuda").current()
    N = q.shape[1]
    must_do = [N - 1, N - 100, 150, 140]  # key tiles 3 and 1
    attn = LiteAttention(threshold=0.0)
    o, lse = attn(q, k, v, return_softmax_lse=True, must_do_list=must_do)
    ref = oracle.lite_attention_forward(to_np(q), to_np(k), to_np(v), None, tau=0.0, must_do=must_do)
    assert_within(compare(o, lse, attn._state.cur, ref))


def test_seq_parallel_object_on_one_gpu():
    """Three K/V splits of one clip, attended in turn with their split index and merged by LSE."""
    w = wl.small_workload(1, 2, 6, 8, 16, 128, steps=3, locality=4.0, tau=TAU, seed_offset=303)
    tr = wl.Trajectory(w, device="cuda")
    N = w.N  # 768
    cuts = [0, 250, 500, N]  # ragged splits
    attn = SeqParallelLiteAttention(num_nodes=3, threshold=TAU)
    masks = [None] * 3
    for t in range(w.steps):
        q, k, v = tr.current()
        parts, refs = [], []
        for s, (a, e) in enumerate(zip(cuts, cuts[1:])):
            ks, vs = k[:, a:e].contiguous(), v[:, a:e].contiguous()
            o_s, l_s = attn(q, ks, vs, split_idx=s)
            ref = oracle.lite_attention_forward(to_np(q), to_np(ks), to_np(vs), masks[s], tau=TAU)
            assert_within(compare(o_s, l_s, attn._states[s].cur, ref))
            masks[s] = _mask_np(attn._states[s].cur)
            parts.append((o_s, l_s))
            refs.append((ref.out, ref.lse))
        o, lse = la.lite_lse_merge(parts)
        ro, rl = oracle.lse_merge(refs)
        assert_within(compare(o, lse, None, oracle.ForwardResult(ro, rl, None, {}), check_mask=False))
        tr.advance()
    with pytest.raises(IndexError):
        attn(q, k, v, split_idx=3)
