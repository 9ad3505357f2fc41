"""Pins for the oracle of the accumulated-error calibration (CPU).

The pages state the calibration in words (skill page "Lite Attention Temporal Sparse", Architecture
Overview and Implementation Steps, Step 3; README "Error Calibration"); none prints a worked
example. The checks here pin the oracle to things that hold independently of its code:
  * the budget schedule's stated shape (0.5 at step 0, a linear rise over the first 30% of the
    steps, 1.0 afterwards) and values derived by hand from it;
  * dropped mass by two independent routes: the dense softmax summed over the skipped tiles, and
    1 - exp(lse_live - lse_full) from the oracle forward pass (a closed form);
  * the QK-Skip element bound: the mass newly dropped at a step stays below the number of newly
    flagged columns times exp(tau) (tau <= 0);
  * bisection properties: the chosen threshold meets the budget, a looser budget never gives a
    smaller threshold, and the threshold one resolution step higher violates the budget.
"""

import math

import numpy as np
import pytest

import oracle
from oracle import calibration as cal
from temporal_block_sparse_b200 import workload as wl


def _qkv(seed=0, H=2, frames=6, gh=8, gw=16, d=64, locality=5.0, tau=-2.0, steps=2):
    w = wl.small_workload(1, H, frames, gh, gw, d, steps=steps, locality=locality, tau=tau, seed_offset=seed)
    tr = wl.Trajectory(w, device="cpu")
    out = []
    for _ in range(steps):
        out.append(tuple(x.float().numpy().astype(np.float64) for x in tr.current()))
        tr.advance()
    return w, out


def _budget_pins(schedule):
    """The schedule's stated shape and values derived by hand from it, for a schedule function."""
    for T, ratio in ((10, 0.3), (50, 0.3), (7, 0.5), (20, 0.0), (1, 0.3)):
        b = np.asarray(schedule(T, ratio))
        n_early = int(T * ratio)
        assert len(b) == T
        assert np.all(np.diff(b) >= 0)                     # later steps never get a tighter budget
        assert np.all(b[n_early:] == 1.0)                  # "later steps tolerate more error": 1.0
        if n_early:
            assert b[0] == 0.5                             # the early ramp starts at 0.5
            assert np.all(b[:n_early] < 1.0)
            steps = np.diff(b[:n_early])
            assert np.allclose(steps, steps[0] if len(steps) else 0)  # linear
    # hand-derived: 10 steps, 3 early steps rising by 1/6 each
    assert np.allclose(schedule(10, 0.3), [0.5, 2 / 3, 5 / 6, 1, 1, 1, 1, 1, 1, 1])


def test_error_budget_schedule_shape():
    _budget_pins(cal.error_budgets)


@pytest.mark.parametrize("mistake", ["reversed ramp", "ramp from zero", "ramp over every step"])
def test_planted_mistake_in_budget_schedule_is_caught(monkeypatch, mistake):
    """A mistake planted in oracle.calibration.error_budgets itself fails the pins above."""
    right = cal.error_budgets

    def planted(num_steps, early_step_ratio=0.3):
        b = np.asarray(right(num_steps, early_step_ratio))
        if mistake == "reversed ramp":         # early steps get MORE tolerance
            return 1.5 - b
        if mistake == "ramp from zero":        # the 0.5 offset dropped
            return np.where(b < 1.0, 2 * b - 1.0, b)
        return np.asarray(right(num_steps, 1.0))  # early_step_ratio ignored

    monkeypatch.setattr(cal, "error_budgets", planted)
    with pytest.raises(AssertionError):
        _budget_pins(cal.error_budgets)


def _flagged_tile_max_p(q, k, mask_out):
    """Largest dense-softmax probability inside each flagged tile (numpy, float64, per head)."""
    B, N, H, d = q.shape
    t, T, _ = oracle.geometry(N, d)
    out = []
    for b in range(B):
        for h in range(H):
            s = (q[b, :, h] @ k[b, :, h].T) / math.sqrt(d)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            for i in range(T):
                for j in range(T):
                    if oracle.is_skipped(mask_out, b, h, i, j):
                        out.append(p[i * t:(i + 1) * t, j * t:(j + 1) * t].max())
    return np.asarray(out)


def test_tau_for_budget_bounds_the_flagged_elements():
    """tau_for_budget(base, b) is the threshold whose flags keep every element of a flagged tile
    below b * exp(base) under that step's dense softmax (pinned through the forward pass's flags and
    an independent softmax, not through the function's formula). A sign-flipped mapping flags
    tiles that break the bound on the same inputs."""
    _, steps = _qkv(seed=17, locality=5.0, H=2)
    q, k, v = steps[0]
    checked, caught = 0, 0
    for base, b in ((-3.0, 0.05), (-2.0, 0.1), (-1.0, 0.5)):
        tau = cal.tau_for_budget(base, b)
        r = oracle.lite_attention_forward(q, k, v, None, tau=tau)
        mx = _flagged_tile_max_p(q, k, r.mask_out)
        checked += len(mx)
        assert np.all(mx < b * math.exp(base))
        wrong = oracle.lite_attention_forward(q, k, v, None, tau=base - math.log(b))
        caught += int(np.any(_flagged_tile_max_p(q, k, wrong.mask_out) >= b * math.exp(base)))
    assert checked > 0 and caught > 0
    assert cal.tau_for_budget(-3.0, 1.0) == -3.0


def test_dropped_mass_two_routes_agree():
    w, steps = _qkv(seed=11)
    q, k, v = steps[0]
    r0 = oracle.lite_attention_forward(q, k, v, None, tau=-2.0)
    mask = r0.mask_out
    assert mask.any()
    _, lse_full = oracle.dense_attention(q, k, v)
    live = oracle.lite_attention_forward(q, k, v, mask, tau=-np.inf)
    via_lse = cal.dropped_mass(live.lse, lse_full)
    direct = cal.dropped_mass_direct(q, k, mask)
    np.testing.assert_allclose(via_lse, direct, atol=1e-12, rtol=1e-9)
    assert direct.max() > 0


def test_dropped_mass_special_cases():
    w, steps = _qkv(seed=12)
    q, k, v = steps[0]
    B, N, H, d = q.shape
    t, T, W = oracle.geometry(N, d)
    assert cal.dropped_mass_direct(q, k, None).max() == 0.0
    full = np.zeros((B, H, T, W), dtype=np.uint32)
    for j in range(T):
        full[..., j >> 5] |= np.uint32(1 << (j & 31))
    np.testing.assert_allclose(cal.dropped_mass_direct(q, k, full), 1.0, atol=1e-12)
    assert np.all(cal.dropped_mass(np.full((1, 1, 3), -np.inf), np.zeros((1, 1, 3))) == 1.0)
    assert np.all(cal.dropped_mass(np.zeros((1, 1, 3)), np.zeros((1, 1, 3))) == 0.0)


@pytest.mark.parametrize("tau", [-6.0, -3.0, -1.0])
def test_new_dropped_mass_within_the_qk_skip_bound(tau):
    w, steps = _qkv(seed=13, locality=5.0)
    q, k, v = steps[0]
    B, N, H, d = q.shape
    tile, T, _ = oracle.geometry(N, d)
    r = oracle.lite_attention_forward(q, k, v, None, tau=tau)
    dropped = cal.dropped_mass_direct(q, k, r.mask_out)  # starting from an empty mask: all new
    for (b, h, i), tr in r.tiles.items():
        cols = sum(min(N, (j + 1) * tile) - j * tile for j in tr.flagged)
        rows = slice(i * tile, min(N, (i + 1) * tile))
        assert np.all(dropped[b, h, rows] <= cols * math.exp(tau) + 1e-12)


def test_calibrate_step_properties():
    w, steps = _qkv(seed=14, locality=5.0)
    q, k, v = steps[0]
    _, lse_full = oracle.dense_attention(q, k, v)
    prev = -np.inf
    for eps in (1e-4, 1e-3, 1e-2, 1e-1):
        r = cal.calibrate_step(q, k, v, None, eps, tau_lo=-12.0, tau_hi=0.0, iters=6, lse_full=lse_full)
        assert r.dropped_max <= eps
        assert r.tau >= prev                                  # looser budget, never a smaller tau
        prev = r.tau
        if np.isfinite(r.tau) and r.tau < 0.0:
            # one bisection resolution above the chosen threshold breaks the budget
            up = oracle.lite_attention_forward(q, k, v, None, tau=r.tau + 12.0 / 2 ** 6)
            mx, _ = cal.mask_dropped(q, k, v, up.mask_out, lse_full)
            assert mx > eps
        # the returned mask is the forward pass's at the returned threshold
        if np.isfinite(r.tau):
            again = oracle.lite_attention_forward(q, k, v, None, tau=r.tau)
            np.testing.assert_array_equal(again.mask_out, r.mask_out)


def test_calibrate_step_keeps_mask_when_nothing_fits():
    w, steps = _qkv(seed=15, locality=5.0)
    q, k, v = steps[0]
    m = oracle.lite_attention_forward(q, k, v, None, tau=-1.0).mask_out
    base, _ = cal.mask_dropped(q, k, v, m, oracle.dense_attention(q, k, v)[1])
    assert base > 0
    r = cal.calibrate_step(q, k, v, m, base / 2, tau_lo=-12.0, tau_hi=0.0)
    assert r.tau == -np.inf
    np.testing.assert_array_equal(r.mask_out, m)
    assert math.isclose(r.dropped_max, base, rel_tol=1e-12)


def test_mean_criterion_is_looser_than_max():
    # mean <= max per row set, so for one budget the mean criterion admits a threshold at least as large
    w, steps = _qkv(seed=16, locality=5.0)
    q, k, v = steps[0]
    _, lse_full = oracle.dense_attention(q, k, v)
    for eps in (1e-4, 1e-3):
        rmax = cal.calibrate_step(q, k, v, None, eps, lse_full=lse_full, criterion="max")
        rmean = cal.calibrate_step(q, k, v, None, eps, lse_full=lse_full, criterion="mean")
        assert rmean.dropped_mean <= eps
        assert rmean.tau >= rmax.tau
    with pytest.raises(ValueError):
        cal.calibrate_step(q, k, v, None, 1e-3, lse_full=lse_full, criterion="median")
