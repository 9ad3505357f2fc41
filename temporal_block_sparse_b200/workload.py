"""Seeded synthetic inputs shaped like the video-DiT self-attention layers LiteAttention targets.

This module is shared by the CUDA path's harness (bench, tests) and by the CPU oracle's tests. It holds
no arithmetic of the attention method itself: it only draws q, k, v tensors and the per-step threshold
schedule.

Token order is frame-major, then latent row, then latent column: n = f*(Hs*Ws) + y*Ws + x.
q and k are N(0,1) "content" plus s times a shared per-token 3-D sinusoidal position embedding, so
scores favour nearby tokens and the attention is locally concentrated, as in the video DiTs the
LiteAttention README evaluates (Wan2.1 / Wan2.2, "Results"). v is N(0,1) content only.

Denoising drift: the content parts follow x_t = (1 - delta) * x_{t-1} + delta * eps_t with fresh
eps_t ~ N(0,1); the position term is re-added at every step. This is the literal reading of the
workload text; it is not variance preserving, so locality (and sparsity) rises over the steps.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, Iterator, List, Optional, Sequence

import torch


def _tau_const(v: float) -> Callable[[int, int], float]:
    return lambda t, steps: float(v)


def _tau_linear(a: float, b: float) -> Callable[[int, int], float]:
    # both endpoints included: tau_0 = a, tau_{steps-1} = b
    return lambda t, steps: float(a + (b - a) * (t / max(steps - 1, 1)))


@dataclass(frozen=True)
class Workload:
    """One synthetic attention layer followed over a denoising trajectory."""

    name: str
    B: int
    H: int
    frames: int
    grid_h: int
    grid_w: int
    d: int
    steps: int
    locality: float  # s, multiplies the position embedding (ignored when locality_range is set)
    drift: float  # delta in x_t = (1-delta) x_{t-1} + delta eps
    tau_schedule: Callable[[int, int], float] = field(compare=False, repr=False, default=_tau_const(-3.0))
    locality_range: Optional[Sequence[float]] = None  # per-(b,h) s ~ U[lo, hi] when set
    seed_offset: int = 0

    @property
    def N(self) -> int:
        return self.frames * self.grid_h * self.grid_w

    @property
    def seed(self) -> int:
        return 20251114 + self.seed_offset

    def tau(self, t: int) -> float:
        return self.tau_schedule(t, self.steps)

    def taus(self) -> List[float]:
        return [self.tau(t) for t in range(self.steps)]

    def dense_flop(self) -> float:
        """4 * B * H * N^2 * d: QK^T and PV, two flops per multiply-add."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.d


WORKLOADS = {
    # 4 frames x 16x16 latent grid, d=64, tile 64, 5 steps, tau=-3
    "tiny": Workload("tiny", 1, 1, 4, 16, 16, 64, 5, 2.0, 0.05, _tau_const(-3.0), seed_offset=1),
    # one layer at a 480p-like latent (21 frames x 30x52), tau linear -10 -> 0 over 10 steps
    "480p": Workload("480p", 1, 40, 21, 30, 52, 128, 10, 2.0, 0.05, _tau_linear(-10.0, 0.0), seed_offset=2),
    # the 480p latent at head dimension 64 (tile 64), tau=-3, 10 steps
    "480p_d64": Workload("480p_d64", 1, 40, 21, 30, 52, 64, 10, 2.0, 0.05, _tau_const(-3.0), seed_offset=6),
    # one layer at a Wan2.1-14B 720p-like latent (21 frames x 45x80), tau=-3, 50 steps, 3% drift
    "720p": Workload("720p", 1, 40, 21, 45, 80, 128, 50, 3.0, 0.03, _tau_const(-3.0), seed_offset=3),
    # threshold sweep on the 720p shape (tau fixed per run, set by the caller), 20 steps
    "sweep": Workload("sweep", 1, 40, 21, 45, 80, 128, 20, 3.0, 0.03, _tau_const(-3.0), seed_offset=4),
    # high-sparsity stress: B=2, per-(b,h) locality s ~ U[2,8], 30 steps
    "stress": Workload("stress", 2, 40, 21, 45, 80, 128, 30, 0.0, 0.03, _tau_const(-3.0),
                       locality_range=(2.0, 8.0), seed_offset=5),
}

SWEEP_TAUS = (-math.inf, -10.0, -3.0, 0.0)


def axis_split(d: int):
    """Split the head dimension into (frame, row, column) axes for the 3-D embedding.

    The row and column axes get 2*floor(d/6) dims each, the frame axis the rest
    (d=128 -> 44/42/42, d=64 -> 24/20/20). Every part is even, so sin/cos pairs fill it exactly.
    """
    dy = 2 * (d // 6)
    return d - 2 * dy, dy, dy


def _axis_embedding(pos: torch.Tensor, dims: int) -> torch.Tensor:
    half = dims // 2
    k = torch.arange(half, dtype=torch.float64)
    omega = torch.pow(10000.0, -2.0 * k / dims)
    ang = pos.to(torch.float64)[:, None] * omega[None, :]
    return torch.cat([torch.sin(ang), torch.cos(ang)], dim=1)


def position_embedding(frames: int, grid_h: int, grid_w: int, d: int) -> torch.Tensor:
    """[N, d] float32 3-D sinusoidal embedding, frame-major token order."""
    df, dy, dx = axis_split(d)
    n = torch.arange(frames * grid_h * grid_w)
    f = n // (grid_h * grid_w)
    y = (n // grid_w) % grid_h
    x = n % grid_w
    pe = torch.cat([_axis_embedding(f, df), _axis_embedding(y, dy), _axis_embedding(x, dx)], dim=1)
    return pe.to(torch.float32)


def small_workload(B: int, H: int, frames: int, grid_h: int, grid_w: int, d: int, steps: int = 3,
                   locality: float = 2.0, drift: float = 0.05, tau: float = -3.0, seed_offset: int = 100,
                   name: str = "custom") -> Workload:
    """A workload of arbitrary shape (ragged tails, several heads) built by the same recipe."""
    return Workload(name, B, H, frames, grid_h, grid_w, d, steps, locality, drift, _tau_const(tau),
                    seed_offset=seed_offset)


class Trajectory:
    """Draws the q, k, v of successive denoising steps of one workload.

    Tensors are [B, N, H, d] bf16 on `device`. The random stream is a torch.Generator seeded with
    the workload's seed on that device; CPU and CUDA generators give different (equally valid) draws.
    """

    def __init__(self, wl: Workload, device="cpu", dtype=torch.bfloat16):
        self.wl = wl
        self.device = torch.device(device)
        self.dtype = dtype
        self.gen = torch.Generator(device=self.device)
        self.gen.manual_seed(wl.seed)
        B, N, H, d = wl.B, wl.N, wl.H, wl.d
        pe = position_embedding(wl.frames, wl.grid_h, wl.grid_w, d).to(self.device)
        if wl.locality_range is not None:
            lo, hi = wl.locality_range
            s = lo + (hi - lo) * torch.rand((B, H), generator=self.gen, device=self.device, dtype=torch.float32)
        else:
            s = torch.full((B, H), wl.locality, device=self.device, dtype=torch.float32)
        self.locality = s  # [B, H]
        # s * PE broadcast to [B, N, H, d]
        self._pos = pe[None, :, None, :] * s[:, None, :, None]
        shape = (B, N, H, d)
        self._base = [torch.randn(shape, generator=self.gen, device=self.device, dtype=torch.float32)
                      for _ in range(3)]
        self.t = 0

    def current(self):
        q = (self._base[0] + self._pos).to(self.dtype)
        k = (self._base[1] + self._pos).to(self.dtype)
        v = self._base[2].to(self.dtype)
        return q, k, v

    def advance(self):
        dlt = self.wl.drift
        for x in self._base:
            eps = torch.randn(x.shape, generator=self.gen, device=self.device, dtype=torch.float32)
            x.mul_(1.0 - dlt).add_(eps, alpha=dlt)
        self.t += 1

    def __iter__(self) -> Iterator:
        for _ in range(self.wl.steps):
            yield self.current()
            self.advance()


def random_mask(B: int, H: int, T: int, density: float, seed: int, device="cpu", Tk=None) -> torch.Tensor:
    """A random skip mask [B, H, T, ceil(Tk/32)] int32 (uint32 bit patterns) for T query tiles and
    Tk key tiles (Tk = T by default); bits >= Tk are zero."""
    Tk = T if Tk is None else Tk
    W = (Tk + 31) // 32
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    bits = torch.rand((B, H, T, W * 32), generator=g) < density
    bits[..., Tk:] = False
    weights = (2 ** torch.arange(32, dtype=torch.int64))
    words = (bits.view(B, H, T, W, 32).to(torch.int64) * weights).sum(-1)
    words = torch.where(words >= 2 ** 31, words - 2 ** 32, words).to(torch.int32)
    return words.to(device)
