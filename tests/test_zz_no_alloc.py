"""lite_attn_fwd_noalloc against lite_attn_fwd (needs a B200).

The no-allocation entry point is for callers that may not allocate device memory (a runtime that
owns nearly all of it, or a loop that cannot afford an allocator call per layer). It must give the
same results as lite_attn_fwd while keeping its scratch in the library's fixed device array. Two
calls in a row check that the array's leftover contents from the previous call do no harm. This file
is collected last so that a run stopping at the first failure has already run every other test.
"""

import numpy as np
import pytest
import torch

from temporal_block_sparse_b200 import lite_attn as la
from temporal_block_sparse_b200 import workload as wl

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

O_MAX_ABS = 2e-2
LSE_ABS = 1e-3


def _two_steps(w):
    tr = wl.Trajectory(w, device="cuda")
    B, N, H, d = w.B, w.N, w.H, w.d
    ref_in = la.new_mask(B, H, N, d)
    new_in = la.new_mask(B, H, N, d)
    for step in range(2):
        q, k, v = tr.current()
        tau = w.tau(step)
        ref_out, new_out = torch.empty_like(ref_in), torch.empty_like(new_in)
        o_ref, lse_ref = la.lite_attn_fwd(q, k, v, ref_in, ref_out, tau=tau)
        o_new = torch.empty_like(q)
        lse_new = torch.empty_like(lse_ref)
        la.lite_attn_fwd_noalloc(q, k, v, o_new, lse_new, new_in, new_out, tau=tau)
        assert la.lite_get_device_status() == 0
        assert (o_new.float() - o_ref.float()).abs().max().item() <= O_MAX_ABS
        assert (lse_new - lse_ref).abs().max().item() <= LSE_ABS
        assert torch.equal(new_out, ref_out)
        ref_in, new_in = ref_out, new_out
        tr.advance()
    return ref_in


def test_noalloc_matches_fwd_on_two_calls_small_ragged_layer():
    w = wl.small_workload(2, 3, 3, 9, 11, 128, steps=2, locality=3.0, tau=-2.0, seed_offset=31)  # N=297
    _two_steps(w)


def test_noalloc_matches_fwd_on_two_calls_480p_layer():
    w = wl.WORKLOADS["480p"]
    base = wl.Workload(w.name, w.B, w.H, w.frames, w.grid_h, w.grid_w, w.d, w.steps, w.locality, w.drift,
                       wl._tau_const(-1.0), seed_offset=w.seed_offset)
    mask = _two_steps(base)
    assert mask.any()  # tau=-1 flags tiles, so the second call reads a non-empty mask


def test_noalloc_refuses_layers_beyond_its_scratch():
    w = wl.WORKLOADS["720p"]  # needs ~28 MB of scratch
    q = torch.zeros((1, w.N, w.H, w.d), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    with pytest.raises(la.LiteAttnError) as e:
        la.lite_attn_fwd_noalloc(q, q, q, o, None, None, None, tau=-3.0)
    assert e.value.status == la.LITE_ERR_SCRATCH_LIMIT
    assert la.lite_get_device_status() == 0
