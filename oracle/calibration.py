"""CPU oracle of the accumulated-error calibration of the QK-Skip threshold. TEST INFRASTRUCTURE ONLY.

Imported only by the test suite and the benchmark's CPU legs; the product path never uses it.

Sources (the LiteAttention pages):
  * "Lite Attention Temporal Sparse" skill page, Architecture Overview, "Accumulated-Error
    Calibration": each timestep gets its own error budget, early steps tolerating less error.
  * Same page, Implementation Steps, Step 3 ("Error Calibration"): a per-timestep tolerance
    multiplier that rises linearly from 0.5 over the early steps (the first early_step_ratio
    fraction of the trajectory, default 0.3) and is 1.0 afterwards.
  * LiteAttention README, contribution list, "Error Calibration": stricter error bounds for earlier
    timesteps, which have greater influence on the final output.
  * README, "QK-Skip Algorithm": once marked, a tile is skipped at every later step (the mask only
    grows), so the error a step's flags introduce is carried by every later step.

Readings where the pages are silent:
  * The multiplier scales the QK-Skip element bound exp(tau): a tile flagged with threshold tau has
    every element below exp(tau) under that step's softmax, so a budget multiplier b corresponds to
    tau + ln(b) (tau_for_budget).
  * The error of a Skip-Mask at a step is the softmax probability mass its skipped tiles hold under
    that step's dense softmax, per query row (dropped_mass_direct). It equals 1 - exp(lse_live -
    lse_dense), with lse_live the log-normaliser over the live tiles only (dropped_mass).
  * Calibrating step t means choosing the largest threshold whose resulting mask (mask_in OR the new
    flags) keeps the largest per-row dropped mass at that step's inputs within the step's budget
    eps * b_t (calibrate_step). The mask and its error accumulate over steps because the mask only
    grows; flags grow monotonically with tau, so the largest admissible tau is found by bisection.
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np

from .lite_attention import geometry, is_skipped, lite_attention_forward, dense_attention


def error_budgets(num_steps: int, early_step_ratio: float = 0.3) -> np.ndarray:
    """Per-step error-tolerance multipliers: the first n_early = floor(num_steps * early_step_ratio)
    steps rise linearly from 0.5 (step 0) towards 1.0 (0.5 + 0.5 * t / n_early), later steps 1.0."""
    n_early = int(num_steps * early_step_ratio)
    out = np.ones(num_steps)
    for t in range(min(n_early, num_steps)):
        out[t] = 0.5 + 0.5 * t / n_early
    return out


def tau_for_budget(tau_base: float, budget: float) -> float:
    """Threshold whose per-element bound exp(tau) is budget * exp(tau_base)."""
    return tau_base + math.log(budget)


def dropped_mass_direct(q, k, mask, scale: Optional[float] = None) -> np.ndarray:
    """Per query row, the dense-softmax probability held by the key tiles the mask skips.

    q [B, N, H, d], k [B, N, H, d] (values as float), mask uint32 [B, H, T, W] or None.
    Returns [B, H, N] in float64: sum over skipped columns c of exp(s_rc) / sum over all c of exp(s_rc).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    B, N, H, d = q.shape
    Nk = k.shape[1]
    if scale is None or not (scale > 0):
        scale = 1.0 / math.sqrt(d)
    t, Tq, _ = geometry(N, d)
    _, Tk, _ = geometry(Nk, d)
    out = np.zeros((B, H, N))
    if mask is None:
        return out
    for b in range(B):
        for h in range(H):
            s = scale * (q[b, :, h, :] @ k[b, :, h, :].T)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            for i in range(Tq):
                rows = slice(i * t, min(N, (i + 1) * t))
                for j in range(Tk):
                    if is_skipped(mask, b, h, i, j):
                        out[b, h, rows] += p[rows, j * t:min(Nk, (j + 1) * t)].sum(axis=1)
    return out


def dropped_mass(lse_live, lse_full) -> np.ndarray:
    """1 - exp(lse_live - lse_full) per row (1 where no tile is live), computed as -expm1."""
    a = np.asarray(lse_live, dtype=np.float64)
    f = np.asarray(lse_full, dtype=np.float64)
    with np.errstate(invalid="ignore"):
        m = -np.expm1(a - f)
    return np.where(np.isneginf(a), 1.0, np.clip(m, 0.0, 1.0))


@dataclass
class StepCalibration:
    tau: float              # chosen threshold (-inf: no new flags fit the budget)
    mask_out: np.ndarray    # mask_in | flags(tau)
    dropped_max: float      # largest per-row dropped mass of mask_out at this step's inputs
    dropped_mean: float
    evaluations: int        # forward passes with a candidate threshold


def mask_dropped(q, k, v, mask, lse_full, scale=None):
    """(max, mean) over rows of the dropped mass of `mask` at these inputs."""
    live = lite_attention_forward(q, k, v, mask, scale=scale, tau=-np.inf)
    m = dropped_mass(live.lse, lse_full)
    return float(m.max()), float(m.mean())


def calibrate_step(q, k, v, mask_in, eps: float, tau_lo: float = -12.0, tau_hi: float = 0.0,
                   iters: int = 6, scale=None, lse_full=None, criterion: str = "max") -> StepCalibration:
    """Largest tau in [tau_lo, tau_hi] (to the bisection's resolution) whose mask keeps the largest
    (criterion "max") or the mean ("mean") per-row dropped mass at these inputs <= eps. Bisection on
    tau: the flags, hence the mask and both statistics of its dropped mass, grow monotonically."""
    if criterion not in ("max", "mean"):
        raise ValueError("criterion is 'max' or 'mean'")
    pick = (lambda mx, mean: mx) if criterion == "max" else (lambda mx, mean: mean)
    if lse_full is None:
        _, lse_full = dense_attention(q, k, v, scale)
    evals = 0

    def trial(tau):
        nonlocal evals
        evals += 1
        r = lite_attention_forward(q, k, v, mask_in, scale=scale, tau=tau)
        mx, mean = mask_dropped(q, k, v, r.mask_out, lse_full, scale)
        return r.mask_out, mx, mean

    m_hi, d_hi, e_hi = trial(tau_hi)
    if pick(d_hi, e_hi) <= eps:
        return StepCalibration(tau_hi, m_hi, d_hi, e_hi, evals)
    m_lo, d_lo, e_lo = trial(tau_lo)
    if pick(d_lo, e_lo) > eps:
        # even the strictest candidate overshoots: add no flags at this step
        base = np.asarray(mask_in).copy() if mask_in is not None else None
        mx, mean = (0.0, 0.0) if base is None else mask_dropped(q, k, v, base, lse_full, scale)
        return StepCalibration(-np.inf, base, mx, mean, evals)
    lo, hi = tau_lo, tau_hi
    best = (tau_lo, m_lo, d_lo, e_lo)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        m, dm, em = trial(mid)
        if pick(dm, em) <= eps:
            lo, best = mid, (mid, m, dm, em)
        else:
            hi = mid
    return StepCalibration(best[0], best[1], best[2], best[3], evals)
