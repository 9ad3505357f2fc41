"""Accumulated-error calibration of the QK-Skip threshold over a denoising trajectory.

Sources: "Lite Attention Temporal Sparse" skill page, Architecture Overview ("Accumulated-Error
Calibration": variable error budgets per timestep, early steps tolerating less) and Implementation
Steps, Step 3 (a tolerance multiplier that rises linearly from 0.5 over the first 30% of the steps
and is 1.0 afterwards); LiteAttention README contribution list, "Error Calibration" (stricter bounds
for the earlier timesteps, which influence the final output more); README "QK-Skip Algorithm" (the
mask only grows, so a step's flags add error to every later step).

Definitions used here:
  * budget multiplier b_t per step (error_budgets); the error budget of step t is eps * b_t;
  * the error of a Skip-Mask at a step is, per query row, the probability mass its skipped tiles
    hold under that step's dense softmax: 1 - exp(lse_live - lse_full) (lite_dropped_mass);
  * calibrating step t picks the largest threshold in [tau_lo, tau_hi] whose mask (mask_in OR the
    flags it raises) keeps the largest (or the mean) per-row error at step t within eps * b_t. The flags grow
    monotonically with tau, so the threshold is found by bisection; each trial runs the sparse
    forward pass with the candidate threshold and then with its mask to measure the error. Each
    step's dense pass (for lse_full) is computed once.
  * tau_for_budget gives the static alternative: the multiplier scales the QK-Skip element bound
    exp(tau), i.e. tau_t = tau_base + ln(b_t).

Host-side control only: every tensor operation is a call into the CUDA library (lite_attn).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, Iterable, List, Optional, Tuple

import torch

from . import lite_attn as la


def error_budgets(num_steps: int, early_step_ratio: float = 0.3) -> List[float]:
    """Per-step tolerance multipliers: 0.5 + 0.5 * t / n_early over the first n_early =
    floor(num_steps * early_step_ratio) steps, 1.0 afterwards."""
    n_early = int(num_steps * early_step_ratio)
    return [0.5 + 0.5 * t / n_early if t < n_early else 1.0 for t in range(num_steps)]


def tau_for_budget(tau_base: float, budget: float) -> float:
    """Threshold whose per-element bound exp(tau) equals budget * exp(tau_base)."""
    return tau_base + math.log(budget)


@dataclass
class StepCalibration:
    tau: float                 # chosen threshold; -inf when no new flag fits the budget
    mask_out: torch.Tensor     # mask_in | flags(tau): the mask of the next step
    dropped_max: float         # largest per-row error of mask_out at this step's inputs
    dropped_mean: float
    evaluations: int           # threshold trials (each: one flagging pass and one measuring pass)
    budget: float = 0.0


class _Workspace:
    def __init__(self, q, k, v):
        B, N, H, d = q.shape
        self.o = torch.empty_like(q)
        self.lse_live = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
        self.lse_full = torch.empty_like(self.lse_live)
        self.stats = torch.empty(2, dtype=torch.float32, device=q.device)
        self.rows = B * H * N


def mask_error(q, k, v, mask, ws: _Workspace, scale=None) -> Tuple[float, float]:
    """(largest, mean) per-row error of `mask` at these inputs; ws.lse_full must hold the dense lse."""
    la.lite_attn_fwd(q, k, v, mask, None, scale=scale, tau=float("-inf"), o=ws.o, lse=ws.lse_live)
    la.lite_dropped_mass(ws.lse_live, ws.lse_full, stats=ws.stats)
    mx, tot = ws.stats.tolist()
    return mx, tot / ws.rows


def calibrate_step(q, k, v, mask_in: torch.Tensor, eps: float, tau_lo: float = -12.0, tau_hi: float = 0.0,
                   iters: int = 6, scale=None, ws: Optional[_Workspace] = None,
                   criterion: str = "max") -> StepCalibration:
    """Largest tau in [tau_lo, tau_hi] (to (tau_hi - tau_lo) / 2**iters) whose mask keeps the largest
    (criterion "max") or the mean ("mean") per-row dropped mass at these inputs <= eps. mask_in is
    not modified."""
    if criterion not in ("max", "mean"):
        raise ValueError("criterion is 'max' or 'mean'")
    pick = (lambda mx, mean: mx) if criterion == "max" else (lambda mx, mean: mean)
    if ws is None:
        ws = _Workspace(q, k, v)
        la.lite_attn_dense(q, k, v, scale=scale, o=ws.o, lse=ws.lse_full)
    evals = 0

    def trial(tau):
        nonlocal evals
        evals += 1
        m = torch.empty_like(mask_in)
        la.lite_attn_fwd(q, k, v, mask_in, m, scale=scale, tau=tau, o=ws.o, lse=ws.lse_live)
        mx, mean = mask_error(q, k, v, m, ws, scale)
        return m, mx, mean

    m_hi, d_hi, e_hi = trial(tau_hi)
    if pick(d_hi, e_hi) <= eps:
        return StepCalibration(tau_hi, m_hi, d_hi, e_hi, evals, eps)
    m_lo, d_lo, e_lo = trial(tau_lo)
    if pick(d_lo, e_lo) > eps:
        mx, mean = mask_error(q, k, v, mask_in, ws, scale)
        return StepCalibration(float("-inf"), mask_in.clone(), mx, mean, evals, eps)
    lo, hi = tau_lo, tau_hi
    best = (tau_lo, m_lo, d_lo, e_lo)
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        m, dm, em = trial(mid)
        if pick(dm, em) <= eps:
            lo, best = mid, (mid, m, dm, em)
        else:
            hi = mid
    return StepCalibration(best[0], best[1], best[2], best[3], evals, eps)


def calibrate_schedule(steps: Iterable[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]], num_steps: int, eps: float,
                       early_step_ratio: float = 0.3, tau_lo: float = -12.0, tau_hi: float = 0.0, iters: int = 6,
                       scale=None, mask: Optional[torch.Tensor] = None, criterion: str = "max",
                       on_step: Optional[Callable[[int, StepCalibration], None]] = None) -> List[StepCalibration]:
    """Calibrate a threshold for every step of a trajectory.

    steps yields (q, k, v) for steps 0 .. num_steps-1 (bf16 [B, N, H, d] on the GPU); eps is the base
    error budget (the largest, or with criterion "mean" the mean, per-row dropped softmax mass),
    scaled per step by error_budgets. The mask
    carries over from step to step as in a LiteAttention run (fresh when mask is None). Returns one
    StepCalibration per step; its tau is the step's calibrated threshold.
    """
    budgets = error_budgets(num_steps, early_step_ratio)
    out: List[StepCalibration] = []
    for t, (q, k, v) in enumerate(steps):
        if t >= num_steps:
            break
        B, N, H, d = q.shape
        if mask is None:
            mask = la.new_mask(B, H, N, d, device=q.device)
        ws = _Workspace(q, k, v)
        la.lite_attn_dense(q, k, v, scale=scale, o=ws.o, lse=ws.lse_full)
        r = calibrate_step(q, k, v, mask, eps * budgets[t], tau_lo, tau_hi, iters, scale, ws, criterion)
        out.append(r)
        if on_step is not None:
            on_step(t, r)
        mask = r.mask_out
    return out
