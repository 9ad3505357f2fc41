"""Shared comparison helpers for the GPU parity tests (GPU path vs the CPU oracle).

Tolerances: output max-abs error <= 2e-2 and relative RMS <= 1e-2; lse absolute error <= 1e-3;
Skip-Mask bit-exact except for tiles whose QK-Skip margin lies within 1e-3 of tau (those are counted
and returned, not failed).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

import oracle

O_MAX_ABS = 2e-2
O_REL_RMS = 1e-2
LSE_ABS = 1e-3
MARGIN_BAND = 1e-3


@dataclass
class Report:
    o_max_abs: float
    o_rel_rms: float
    lse_max_abs: float
    mask_mismatches: int  # tiles that differ (all within the margin band)
    flagged: int  # tiles the oracle flagged in the compared rows


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def compare(o, lse, mask_out, ref: oracle.ForwardResult, mask_in_np=None, check_mask=True) -> Report:
    """Compare GPU outputs with an oracle result (all rows, or the sampled query tiles of `ref`)."""
    o_np = to_np(o)
    rows = ~np.isnan(ref.out[..., 0])  # [B, N, H] rows the oracle computed
    diff = (o_np - ref.out)[rows]
    refv = ref.out[rows]
    o_max = float(np.abs(diff).max()) if diff.size else 0.0
    rel = float(np.sqrt((diff ** 2).mean()) / max(np.sqrt((refv ** 2).mean()), 1e-30)) if diff.size else 0.0
    lse_err = 0.0
    if lse is not None:
        l_np = to_np(lse)
        lrows = ~np.isnan(ref.lse)
        a, b = l_np[lrows], ref.lse[lrows]
        inf = np.isneginf(b)
        assert (np.isneginf(a) == inf).all(), "lse -inf pattern differs"
        if (~inf).any():
            lse_err = float(np.abs(a[~inf] - b[~inf]).max())
    mism = 0
    flagged = 0
    if check_mask and mask_out is not None:
        got = mask_out.cpu().numpy().view(np.uint32)
        for (b, h, i), t in ref.tiles.items():
            flagged += len(t.flagged)
            for w in range(got.shape[-1]):
                dbits = int(got[b, h, i, w]) ^ int(ref.mask_out[b, h, i, w])
                while dbits:
                    bit = (dbits & -dbits).bit_length() - 1
                    dbits &= dbits - 1
                    j = w * 32 + bit
                    margin = t.margins.get(j, math.inf)
                    assert abs(margin) <= MARGIN_BAND, f"mask differs at (b={b},h={h},i={i},j={j}), margin {margin}"
                    mism += 1
    return Report(o_max, rel, lse_err, mism, flagged)


def assert_within(rep: Report):
    assert rep.o_max_abs <= O_MAX_ABS, rep
    assert rep.o_rel_rms <= O_REL_RMS, rep
    assert rep.lse_max_abs <= LSE_ABS, rep
