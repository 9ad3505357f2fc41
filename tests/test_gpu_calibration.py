"""Accumulated-error calibration on the GPU vs the oracle (needs a B200).

lite_dropped_mass is compared element by element with the oracle's 1 - exp(lse_live - lse_full) on the
same fp32 inputs, and end to end (GPU lse of the sparse and the dense pass) with the oracle's direct
sum of dense softmax probabilities over the skipped tiles. The GPU calibration of one step is checked
against the oracle's: its mask keeps the oracle-measured dropped mass within the budget, and its
threshold equals the oracle's unless the budget sits within measurement noise of the dropped mass at
one of the two thresholds.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import calibration as ocal
from temporal_block_sparse_b200 import calibration as gcal
from temporal_block_sparse_b200 import lite_attn as la
from temporal_block_sparse_b200 import workload as wl

from gpu_parity import to_np

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

NOISE = 3e-4  # dropped-mass error from the fp32 lse of two GPU passes (lse abs error <= 1e-4 each)


@pytest.fixture(autouse=True)
def _clean_state():
    la.load()
    yield
    assert la.lite_get_device_status() == 0


@pytest.mark.parametrize("shape", [(1, 1, 1), (1, 3, 7), (2, 5, 1001), (1, 40, 4096)])
def test_dropped_mass_kernel_matches_oracle(shape):
    g = torch.Generator(device="cuda")
    g.manual_seed(sum(shape))
    full = torch.randn(shape, generator=g, device="cuda") * 4
    gap = torch.rand(shape, generator=g, device="cuda") ** 3 * 12  # many small, some large drops
    live = full - gap
    live.view(-1)[::7] = float("-inf")          # rows with no live tile
    live.view(-1)[1::11] = full.view(-1)[1::11]  # rows that drop nothing
    row = torch.empty_like(full)
    la.lite_dropped_mass(live, full, row_mass=row)
    _, stats = la.lite_dropped_mass(live, full)
    want = ocal.dropped_mass(live.cpu().numpy(), full.cpu().numpy())
    got = row.cpu().numpy()
    np.testing.assert_allclose(got, want, atol=2e-6, rtol=1e-5)
    mx, tot = stats.tolist()
    assert mx == pytest.approx(want.max(), abs=2e-6)
    assert tot == pytest.approx(want.sum(), rel=1e-5, abs=1e-4)


def test_dropped_mass_kernel_unaligned_views():
    # buffers starting 4 bytes past a 16-byte boundary take the scalar path; 4097 rows leave a tail
    n = 4097
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    live_buf = torch.empty(n + 1, device="cuda")
    full_buf = torch.empty(n + 1, device="cuda")
    row_buf = torch.empty(n + 1, device="cuda")
    full = full_buf[1:].view(1, 1, n)
    live = live_buf[1:].view(1, 1, n)
    full.copy_(torch.randn((1, 1, n), generator=g, device="cuda"))
    live.copy_(full - torch.rand((1, 1, n), generator=g, device="cuda") * 3)
    row = row_buf[1:].view(1, 1, n)
    _, stats = la.lite_dropped_mass(live, full, row_mass=row)
    want = ocal.dropped_mass(live.cpu().numpy(), full.cpu().numpy())
    np.testing.assert_allclose(row.cpu().numpy(), want, atol=2e-6, rtol=1e-5)
    assert stats[0].item() == pytest.approx(want.max(), abs=2e-6)


def _step(seed=21, frames=6, gh=8, gw=16, d=64, H=2, locality=5.0):
    w = wl.small_workload(1, H, frames, gh, gw, d, steps=2, locality=locality, tau=-2.0, seed_offset=seed)
    return wl.Trajectory(w, device="cuda").current()


@pytest.mark.parametrize("d", [64, 128])
def test_dropped_mass_through_attention(d):
    q, k, v = _step(seed=22, d=d, gw=16 if d == 64 else 32)
    B, N, H, _ = q.shape
    m_in = la.new_mask(B, H, N, d)
    m_out = torch.empty_like(m_in)
    la.lite_attn_fwd(q, k, v, m_in, m_out, tau=-1.0)
    _, lse_live = la.lite_attn_fwd(q, k, v, m_out, None, tau=float("-inf"))
    _, lse_full = la.lite_attn_dense(q, k, v)
    row = torch.empty_like(lse_full)
    la.lite_dropped_mass(lse_live, lse_full, row_mass=row)
    mask = m_out.cpu().numpy().view(np.uint32)
    assert mask.any()
    want = ocal.dropped_mass_direct(to_np(q), to_np(k), mask)
    np.testing.assert_allclose(row.cpu().numpy(), want, atol=NOISE)


@pytest.mark.parametrize("eps", [1e-3, 1e-2])
def test_calibrate_step_matches_oracle(eps):
    q, k, v = _step(seed=23)
    B, N, H, d = q.shape
    res = gcal.calibrate_step(q, k, v, la.new_mask(B, H, N, d), eps, tau_lo=-12.0, tau_hi=0.0, iters=6)
    qn, kn, vn = to_np(q), to_np(k), to_np(v)
    _, lse_full = oracle.dense_attention(qn, kn, vn)
    ref = ocal.calibrate_step(qn, kn, vn, None, eps, tau_lo=-12.0, tau_hi=0.0, iters=6, lse_full=lse_full)
    # the GPU's mask keeps the true dropped mass within the budget (up to measurement noise)
    if res.mask_out is not None:
        got_mask = res.mask_out.cpu().numpy().view(np.uint32)
        true_max, _ = ocal.mask_dropped(qn, kn, vn, got_mask, lse_full)
        assert true_max <= eps + NOISE
        assert abs(true_max - res.dropped_max) <= NOISE
    if res.tau != ref.tau:
        # only a budget within noise of the dropped mass at one of the two thresholds may split them
        near = []
        for tau in (res.tau, ref.tau):
            if math.isfinite(tau):
                m = oracle.lite_attention_forward(qn, kn, vn, None, tau=tau).mask_out
                near.append(abs(ocal.mask_dropped(qn, kn, vn, m, lse_full)[0] - eps))
            up = min(0.0, tau + 12.0 / 2 ** 6) if math.isfinite(tau) else -12.0
            m = oracle.lite_attention_forward(qn, kn, vn, None, tau=up).mask_out
            near.append(abs(ocal.mask_dropped(qn, kn, vn, m, lse_full)[0] - eps))
        assert min(near) <= NOISE, (res.tau, ref.tau, near)


def test_calibrate_schedule_keeps_budgets():
    w = wl.small_workload(1, 2, 6, 8, 16, 64, steps=4, locality=5.0, tau=-2.0, seed_offset=24)
    tr = wl.Trajectory(w, device="cuda")

    def steps():
        for _ in range(w.steps):
            yield tr.current()
            tr.advance()

    eps = 5e-3
    out = gcal.calibrate_schedule(steps(), w.steps, eps, early_step_ratio=0.5)
    budgets = gcal.error_budgets(w.steps, 0.5)
    assert len(out) == w.steps
    prev = None
    for t, r in enumerate(out):
        assert r.budget == pytest.approx(eps * budgets[t])
        m = r.mask_out.cpu().numpy().view(np.uint32)
        if math.isfinite(r.tau):
            assert r.dropped_max <= r.budget + NOISE
        else:
            # the carried-over mask already spends the budget: no new flags
            assert prev is not None and (m == prev).all()
        if prev is not None:
            assert ((m & prev) == prev).all()  # the mask only grows
        prev = m
    assert prev.any()
