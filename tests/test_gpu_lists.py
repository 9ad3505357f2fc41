"""Attention over caller-supplied Skip-Lists, and the attention kernel's list checks (needs a B200).

lite_attn_fwd_list runs the schedule and the attention kernel on lists the caller passes (the
compaction step skipped). It must reproduce lite_attn_fwd on the mask those lists describe bit for
bit. Malformed lists must stop the kernel with LITE_ERR_CHECK in the device status word and leave
the context usable. Every malformed case here stays inside the buffers the kernel may touch even
without the checks: list entries below 32 * W (so a flag would land in the row's own mask words),
counts read from a list buffer padded past its last row, stray bits above the index.
"""

import pytest
import torch

from temporal_block_sparse_b200 import lite_attn as la
from temporal_block_sparse_b200 import workload as wl

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(autouse=True)
def _clean_state():
    la.load()
    yield
    assert la.lite_get_device_status() == 0


def _layer(B=2, H=3, frames=3, gh=9, gw=37, seed=51):  # N = 999: ragged last tile, T = 8
    w = wl.small_workload(B, H, frames, gh, gw, 128, steps=1, locality=3.0, tau=-2.0, seed_offset=seed)
    return w, wl.Trajectory(w, device="cuda").current()


@pytest.mark.parametrize("density,tau", [(0.0, -2.0), (0.5, -2.0), (0.9, 0.0), (0.5, float("-inf"))])
def test_lists_reproduce_the_mask_path(density, tau):
    w, (q, k, v) = _layer()
    B, N, H, d = q.shape
    _, T, _ = la.lite_mask_geometry(N, d)
    mask = wl.random_mask(B, H, T, density, seed=int(density * 10) + 3).cuda()
    lst, counts = la.lite_mask_to_list(mask, B, H, N, d)
    out_mask = torch.empty_like(mask)
    o_ref, lse_ref = la.lite_attn_fwd(q, k, v, mask, out_mask, tau=tau)
    out_list = mask.clone()
    o, lse = la.lite_attn_fwd_list(q, k, v, lst, counts, out_list, tau=tau)
    assert la.lite_get_device_status() == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    assert torch.equal(out_list, out_mask)


def test_tagged_entries_are_never_flagged():
    w, (q, k, v) = _layer(seed=52)
    B, N, H, d = q.shape
    lst, counts = la.lite_mask_to_list(None, B, H, N, d)
    tagged = torch.where(lst >= 0, lst | 0x4000, lst)
    m0 = la.new_mask(B, H, N, d)
    m_plain = m0.clone()
    la.lite_attn_fwd_list(q, k, v, lst, counts, m_plain, tau=0.0)
    assert m_plain.any()  # tau = 0 flags tiles of this layer
    m_tag = m0.clone()
    o_t, lse_t = la.lite_attn_fwd_list(q, k, v, tagged, counts, m_tag, tau=0.0)
    o_p, lse_p = la.lite_attn_fwd_list(q, k, v, lst, counts, m0.clone(), tau=0.0)
    assert la.lite_get_device_status() == 0
    assert not m_tag.any()
    assert torch.equal(o_t, o_p) and torch.equal(lse_t, lse_p)


def _corrupt(kind, lst, counts, T):
    """One malformed list (row 0 of head (0, 0), or the very last row) in a buffer padded by two
    rows, so that a count past T still reads inside the allocation."""
    lst = lst.clone()
    counts = counts.clone()
    flat = lst.view(-1, T)
    rows = counts.numel()
    if kind == "ascending pair":
        flat[0, 0], flat[0, 1] = flat[0, 1].item(), flat[0, 0].item()
    elif kind == "repeated entry":
        flat[0, 1] = flat[0, 0]
    elif kind == "index at T":
        flat[0, 0] = T  # below 32 * W: its flag bit would still sit in the row's own word
    elif kind == "stray bit":
        flat[0, 2] = flat[0, 2] | 0x2000
    elif kind == "count past T":
        counts.view(-1)[rows - 1] = T + 1  # the last row: entry T is read from the padding
    elif kind == "negative count":
        counts.view(-1)[5] = -1
    return lst, counts


@pytest.mark.parametrize("kind", ["ascending pair", "repeated entry", "index at T", "stray bit", "count past T",
                                  "negative count"])
def test_malformed_lists_stop_the_kernel_with_check_status(kind):
    w, (q, k, v) = _layer(B=1, H=2, seed=53)
    B, N, H, d = q.shape
    _, T, W = la.lite_mask_geometry(N, d)
    assert T == 8 and W == 1
    lst, counts = la.lite_mask_to_list(None, B, H, N, d)
    padded = torch.full(((B * H * T + 2) * T,), 0, dtype=torch.int16, device="cuda")
    padded[: lst.numel()] = lst.view(-1)
    bad_list, bad_counts = _corrupt(kind, padded, counts, T)
    mask_out = la.new_mask(B, H, N, d)
    la.lite_attn_fwd_list(q, k, v, bad_list, bad_counts, mask_out, tau=-2.0)
    assert la.lite_get_device_status() == la.LITE_ERR_CHECK
    # the context survives: a well-formed call right after runs and reports no error
    o, lse = la.lite_attn_fwd_list(q, k, v, padded, counts, la.new_mask(B, H, N, d), tau=-2.0)
    o_ref, lse_ref = la.lite_attn_fwd(q, k, v, None, None, tau=-2.0)
    assert la.lite_get_device_status() == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
