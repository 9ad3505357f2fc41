"""The work order and the pairing of query tiles change only which CTA processes which query tile
(needs a B200).

Results (o, lse, mask) are bit-identical with the schedule on and off and for every pairing stride
(each query tile walks its own Skip-List whatever tile it shares a CTA with); the per-CTA timing hook
accounts for every live tile exactly once.
"""

import numpy as np
import pytest
import torch

from temporal_block_sparse_b200 import lite_attn as la
from temporal_block_sparse_b200 import workload as wl

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(autouse=True)
def _clean_state():
    la.load()
    yield
    la.lite_set_option(la.LITE_OPT_SCHEDULE, 1)
    la.lite_set_option(la.LITE_OPT_PAIR_STRIDE, 0)
    la.lite_set_option(la.LITE_OPT_MAX_CTAS, 0)
    la.lite_set_cta_timing(None)
    assert la.lite_get_device_status() == 0


def _masked_step(seed):
    w = wl.small_workload(2, 3, 8, 16, 16, 128, steps=2, locality=5.0, tau=-2.0, seed_offset=seed)  # N = 2048
    tr = wl.Trajectory(w, device="cuda")
    q, k, v = tr.current()
    B, N, H, d = q.shape
    m0 = la.new_mask(B, H, N, d)
    m1 = torch.empty_like(m0)
    la.lite_attn_fwd(q, k, v, m0, m1, tau=-2.0)  # a non-uniform mask for the next step
    tr.advance()
    return tr.current(), m1


def test_schedule_off_gives_identical_results():
    (q, k, v), m_in = _masked_step(61)
    outs = []
    for sched in (1, 0):
        la.lite_set_option(la.LITE_OPT_SCHEDULE, sched)
        m_out = torch.empty_like(m_in)
        o, lse = la.lite_attn_fwd(q, k, v, m_in, m_out, tau=-2.0)
        torch.cuda.synchronize()
        outs.append((o.clone(), lse.clone(), m_out.clone()))
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])
    assert torch.equal(outs[0][2], outs[1][2])


def test_cta_timing_counts_every_live_tile():
    (q, k, v), m_in = _masked_step(62)
    B, N, H, d = q.shape
    _, T, _ = la.lite_mask_geometry(N, d)
    _, counts = la.lite_mask_to_list(m_in, B, H, N, d)
    live = int(counts.sum().item())
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    buf = torch.zeros((sms, 3), dtype=torch.int64, device="cuda")
    la.lite_set_cta_timing(buf)
    la.lite_attn_fwd(q, k, v, m_in, torch.empty_like(m_in), tau=-2.0)
    torch.cuda.synchronize()
    la.lite_set_cta_timing(None)
    rec = buf.cpu().numpy()
    used = rec[:, 1] > 0
    # the kernel's work items are pairs of query tiles of one head
    assert used.sum() == min(sms, B * H * ((T + 1) // 2))
    assert (rec[used, 1] >= rec[used, 0]).all()
    assert int(rec[used, 2].sum()) == live


def test_head_dim_64_runs_two_ctas_per_sm():
    """With d = 64 a CTA holds half of the SM's TMEM columns, so the persistent grid has two CTAs
    per SM and they run side by side: every CTA takes work, the CTAs start together (not in two
    waves), and their tiles add up to the layer's."""
    w = wl.small_workload(1, 8, 8, 32, 64, 64, locality=2.0, seed_offset=64)  # N = 16384, 512 items
    q, k, v = wl.Trajectory(w, device="cuda").current()
    B, N, H, d = q.shape
    _, T, _ = la.lite_mask_geometry(N, d)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    buf = torch.zeros((2 * sms + 8, 3), dtype=torch.int64, device="cuda")
    la.lite_set_cta_timing(buf)
    la.lite_attn_fwd(q, k, v, None, None, tau=-3.0)
    torch.cuda.synchronize()
    la.lite_set_cta_timing(None)
    rec = buf.cpu().numpy()
    used = rec[:, 1] > 0
    assert used.sum() == 2 * sms
    assert (rec[used, 2] > 0).all()
    assert int(rec[used, 2].sum()) == B * H * T * T  # no mask: every tile is live
    starts, ends = rec[used, 0], rec[used, 1]
    # a second wave would start only when the first CTAs ran out of work
    assert starts.max() - starts.min() < 0.25 * (ends.max() - starts.min())


@pytest.mark.parametrize("d", [64, 128])
def test_grid_size_gives_identical_results(d):
    """Every work item computes the same bits whichever CTA takes it: the full grid (two CTAs per
    SM at d = 64), an odd cap that leaves some SMs one CTA, and a single CTA."""
    w = wl.small_workload(1, 16, 8, 32, 32, d, steps=2, locality=4.0, tau=-2.0, seed_offset=70 + d)  # 512 items
    tr = wl.Trajectory(w, device="cuda")
    q, k, v = tr.current()
    B, N, H, _ = q.shape
    m0 = la.new_mask(B, H, N, d)
    m_in = torch.empty_like(m0)
    la.lite_attn_fwd(q, k, v, m0, m_in, tau=-2.0)  # a grown, uneven mask for the compared step
    tr.advance()
    q, k, v = tr.current()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    runs = [_run_with(q, k, v, m_in, -2.0, LITE_OPT_MAX_CTAS=cap) for cap in (0, sms + 1, 1)]
    la.lite_set_option(la.LITE_OPT_MAX_CTAS, 0)
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            assert torch.equal(a, b)


def _run_with(q, k, v, m_in, tau, **opts):
    for name, val in opts.items():
        la.lite_set_option(getattr(la, name), val)
    m_out = torch.empty_like(m_in)
    o, lse = la.lite_attn_fwd(q, k, v, m_in, m_out, tau=tau)
    torch.cuda.synchronize()
    assert la.lite_get_device_status() == 0
    return o.clone(), lse.clone(), m_out.clone()


@pytest.mark.parametrize("layer", ["small", "480p"])
def test_pairing_stride_gives_identical_results(layer):
    """Fixed strides (1 = tiles 2k and 2k+1, several others, and strides larger than half the
    query tiles) and the stride picked from the mask give the same bits, with the schedule on and
    off. The 480p case runs six steps of its trajectory first, so the mask is the grown, uneven one
    where the picked stride differs from 1."""
    if layer == "small":
        (q, k, v), m_in = _masked_step(63)
        tau = -2.0
    else:
        w = wl.WORKLOADS["480p"]
        tr = wl.Trajectory(w, device="cuda")
        B, N, H, d = w.B, w.N, w.H, w.d
        m_in = la.new_mask(B, H, N, d)
        m_out = torch.empty_like(m_in)
        for t in range(6):
            q, k, v = tr.current()
            la.lite_attn_fwd(q, k, v, m_in, m_out, tau=w.tau(t))
            m_in, m_out = m_out, m_in
            tr.advance()
        q, k, v = tr.current()
        tau = w.tau(6)
    ref = _run_with(q, k, v, m_in, tau, LITE_OPT_PAIR_STRIDE=1, LITE_OPT_SCHEDULE=1)
    for stride in (0, 2, 3, 12, 28, 64, 4096):
        for sched in (1, 0):
            got = _run_with(q, k, v, m_in, tau, LITE_OPT_PAIR_STRIDE=stride, LITE_OPT_SCHEDULE=sched)
            for a, b in zip(ref, got):
                assert torch.equal(a, b), (stride, sched)
