"""lite_attn_fwd_noalloc against lite_attn_fwd (needs a B200).

The no-allocation entry point is for callers that may not allocate device memory: a serving
runtime that has reserved nearly all of it for its own pool (any library allocation would fail or
evict the caller's data), or a denoising loop that cannot afford an allocator call per layer. Its
scratch lives in the library's fixed device array, so it must give exactly the results of
lite_attn_fwd -- both run the same kernels on the same inputs -- while allocating nothing. Two calls
in a row check that the array's leftover contents from the previous call do no harm. This file is
collected last so that a run stopping at the first failure has already run every other test.
"""

import os
import subprocess
import sys

import pytest
import torch

from temporal_block_sparse_b200 import lite_attn as la
from temporal_block_sparse_b200 import workload as wl

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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
        # the same kernels on the same inputs: identical bits, so leftover scratch cannot hide
        assert torch.equal(o_new, o_ref)
        assert torch.equal(lse_new, lse_ref)
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


def test_noalloc_wrapper_refuses_bad_buffers():
    """Buffers the C side cannot check (a host mask, a short or mistyped o / lse) are refused
    before the call."""
    w = wl.small_workload(1, 2, 2, 8, 8, 128, steps=1, seed_offset=32)  # N=128
    q, k, v = wl.Trajectory(w, device="cuda").current()
    B, N, H, d = q.shape
    m = la.new_mask(B, H, N, d)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    bad = [
        dict(mask_in=m.cpu()),
        dict(mask_out=torch.zeros((B, H, 2, 1), dtype=torch.int32, device="cuda")),
        dict(o=torch.empty((B, N, H, d), dtype=torch.float16, device="cuda")),
        dict(o=torch.empty((B, N - 1, H, d), dtype=torch.bfloat16, device="cuda")),
        dict(lse=torch.empty((B, H, N - 1), dtype=torch.float32, device="cuda")),
        dict(lse=torch.empty((B, H, N), dtype=torch.float64, device="cuda")),
    ]
    for kw in bad:
        args = dict(o=o, lse=lse, mask_in=m, mask_out=m)
        args.update(kw)
        with pytest.raises(ValueError):
            la.lite_attn_fwd_noalloc(q, k, v, args["o"], args["lse"], args["mask_in"], args["mask_out"], tau=-3.0)


CHILD = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
from temporal_block_sparse_b200 import lite_attn as la
from temporal_block_sparse_b200 import workload as wl
torch.cuda.set_device(0)
for shape in ((1, 2, 2, 8, 8), (1, 4, 3, 9, 11)):
    w = wl.small_workload(*shape, 128, steps=1, seed_offset=33)
    q, k, v = wl.Trajectory(w, device="cuda").current()
    B, N, H, d = q.shape
    m_in, m_out = la.new_mask(B, H, N, d), la.new_mask(B, H, N, d)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    for _ in range(2):
        la.lite_attn_fwd_noalloc(q, k, v, o, lse, m_in, m_out, tau=-2.0)
    assert la.lite_get_device_status() == 0
    assert la.scratch_pool_bytes() == 0, la.scratch_pool_bytes()
la.lite_attn_fwd(q, k, v, m_in, m_out, tau=-2.0)
torch.cuda.synchronize()
assert la.scratch_pool_bytes() > 0  # the hook does see the pool once a pooled call has run
print("noalloc allocated nothing")
"""


def test_noalloc_allocates_nothing_in_a_fresh_process():
    """In a process where only lite_attn_fwd_noalloc runs, the library's scratch pool is never
    created (it reserves nothing); one pooled lite_attn_fwd call afterwards does create it."""
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "noalloc allocated nothing" in r.stdout
