"""Per-layer attention objects over the C ABI: the Skip-Mask state that persists across denoising
steps, and sequence parallelism over K/V splits.

Sources (LiteAttention README, Python API): one LiteAttention object per attention layer, each
with its own skip state (sharing one across layers is wrong); enable_skip_optimization() turns the
skip test on and off (off: every tile is computed); reset_skip_state() clears the state for a new
video; must_do_list / must_skip_list key ranges; return_softmax_lse for combining partial
attentions; SeqParallelLiteAttention(num_nodes, ...) called with the index of the K/V split it
processes, one skip state per split.

Host bookkeeping only: every tensor operation runs in the CUDA library through lite_attn. The
state is a pair of mask buffers per (split, shape); each call reads one and writes the other (the
library copies mask_in into mask_out and ORs new flags), then the pair swaps.
"""

from __future__ import annotations

from typing import Callable, Dict, List, Optional, Sequence, Tuple

import torch

from . import lite_attn as la


class _SkipState:
    """The two mask buffers of one layer (or one K/V split of a layer)."""

    def __init__(self):
        self.key = None
        self.cur: Optional[torch.Tensor] = None
        self.nxt: Optional[torch.Tensor] = None

    def buffers(self, B: int, H: int, Nq: int, Nk: int, d: int, device) -> Tuple[torch.Tensor, torch.Tensor]:
        key = (B, H, Nq, Nk, d, str(device))
        if key != self.key:
            # a new shape starts from a fresh (all-live) mask
            self.cur = la.new_mask(B, H, Nq, d, device=device, Nk=Nk)
            self.nxt = torch.empty_like(self.cur)
            self.key = key
        return self.cur, self.nxt

    def swap(self):
        self.cur, self.nxt = self.nxt, self.cur

    def reset(self):
        if self.cur is not None:
            self.cur.zero_()

    def skipped_fraction(self) -> Optional[float]:
        if self.cur is None:
            return None
        B, H, Nq, Nk, d, _ = self.key
        _, Tk, _ = la.lite_mask_geometry(Nk, d)
        words = self.cur.to(torch.int64) & 0xFFFFFFFF
        bits = (words.unsqueeze(-1) >> torch.arange(32, device=words.device)) & 1
        return float(bits.flatten(-2)[..., :Tk].float().mean())


class LiteAttention:
    """One attention layer's LiteAttention: call it at every denoising step with that step's q, k, v.

    threshold: QK-Skip tau (natural-log units of scale * QK^T; README default -10).
    enable_skipping: False computes every tile and neither reads nor updates the skip state.
    """

    def __init__(self, enable_skipping: bool = True, threshold: float = -10.0, max_batch_size: int = 4):
        self.enable_skipping = bool(enable_skipping)
        self.threshold = float(threshold)
        self.max_batch_size = int(max_batch_size)
        self._state = _SkipState()

    def enable_skip_optimization(self, enable: bool = True):
        self.enable_skipping = bool(enable)

    def set_threshold(self, threshold: float):
        self.threshold = float(threshold)

    def reset_skip_state(self):
        self._state.reset()

    def skipped_fraction(self) -> Optional[float]:
        """Fraction of (query tile, key tile) pairs the current state skips (None before the first call)."""
        return self._state.skipped_fraction()

    def _run(self, state: _SkipState, q, k, v, scale, return_softmax_lse, must_do_list, must_skip_list):
        B, Nq, H, d = q.shape
        if B > self.max_batch_size:
            raise ValueError(f"batch {B} exceeds max_batch_size {self.max_batch_size}")
        Nk = k.shape[1]
        if not self.enable_skipping:
            if must_do_list or must_skip_list:
                o, lse = la.lite_attn_fwd_ex(q, k, v, None, None, must_do=must_do_list, must_skip=must_skip_list,
                                             scale=scale, tau=float("-inf"), return_lse=return_softmax_lse)
            else:
                o, lse = la.lite_attn_dense_ex(q, k, v, scale=scale, return_lse=return_softmax_lse)
        else:
            m_in, m_out = state.buffers(B, H, Nq, Nk, d, q.device)
            o, lse = la.lite_attn_fwd_ex(q, k, v, m_in, m_out, must_do=must_do_list, must_skip=must_skip_list,
                                         scale=scale, tau=self.threshold, return_lse=return_softmax_lse)
            state.swap()
        return (o, lse) if return_softmax_lse else o

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: Optional[float] = None,
                 return_softmax_lse: bool = False, must_do_list: Optional[Sequence[int]] = None,
                 must_skip_list: Optional[Sequence[int]] = None):
        """o [B, Nq, H, d] (and lse [B, H, Nq] with return_softmax_lse) for q [B, Nq, H, d], k, v [B, Nk, H, d]."""
        return self._run(self._state, q, k, v, scale, return_softmax_lse, must_do_list, must_skip_list)


class SeqParallelLiteAttention(LiteAttention):
    """LiteAttention for sequence parallelism: the keys and values come in num_nodes splits, each
    call attends the local queries to one split and keeps a separate skip state per split (the
    QK-Skip running maximum only sees that split's key tiles). The partial results combine with
    lite_lse_merge; seq_parallel_forward below does the exchange and the combine."""

    def __init__(self, num_nodes: int, enable_skipping: bool = True, threshold: float = -10.0,
                 max_batch_size: int = 4):
        super().__init__(enable_skipping, threshold, max_batch_size)
        if num_nodes < 1:
            raise ValueError("num_nodes >= 1")
        self.num_nodes = int(num_nodes)
        self._states = [_SkipState() for _ in range(self.num_nodes)]

    def reset_skip_state(self):
        for s in self._states:
            s.reset()

    def skipped_fraction(self, split_idx: int = 0) -> Optional[float]:
        return self._states[split_idx].skipped_fraction()

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, split_idx: int,
                 scale: Optional[float] = None, return_softmax_lse: bool = True,
                 must_do_list: Optional[Sequence[int]] = None, must_skip_list: Optional[Sequence[int]] = None):
        if not 0 <= split_idx < self.num_nodes:
            raise IndexError(f"split_idx {split_idx} outside [0, {self.num_nodes})")
        return self._run(self._states[split_idx], q, k, v, scale, return_softmax_lse, must_do_list, must_skip_list)


SplitAttn = Callable[[torch.Tensor, torch.Tensor, torch.Tensor, int], Tuple[torch.Tensor, torch.Tensor]]
Merge = Callable[[List[Tuple[torch.Tensor, torch.Tensor]]], Tuple[torch.Tensor, torch.Tensor]]


def split_order(rank: int, world: int) -> List[int]:
    """Order in which a rank processes the K/V splits: its own first (no wait on the exchange),
    then the others in ring order."""
    return [(rank + s) % world for s in range(world)]


def seq_parallel_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, split_attn: SplitAttn,
                         merge: Merge = None, group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Sequence-parallel attention of this rank's queries against the keys / values of all ranks.

    q, k, v: this rank's token shard, [B, n, H, d] each (every rank holds the same n). The K and V
    shards of all ranks are all-gathered into local memory (asynchronously: the rank's own split is
    computed while the exchange runs), each split s gives a partial (o_s, lse_s) =
    split_attn(q, k_s, v_s, s), and the partials are merged by their LSE. Returns (o, lse) for
    this rank's queries. split_attn is normally a SeqParallelLiteAttention with return_softmax_lse;
    merge defaults to lite_lse_merge (at most 8 splits).
    """
    import torch.distributed as dist

    if merge is None:
        merge = la.lite_lse_merge
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if world == 1:
        return merge([split_attn(q, k, v, 0)])
    # gathered as [world * B, n, H, d] (concatenated along dim 0, the form every backend takes),
    # which is the same memory as [world, B, n, H, d]
    B = k.shape[0]
    k_cat = torch.empty((world * B,) + tuple(k.shape[1:]), dtype=k.dtype, device=k.device)
    v_cat = torch.empty_like(k_cat)
    hk = dist.all_gather_into_tensor(k_cat, k.contiguous(), group=group, async_op=True)
    hv = dist.all_gather_into_tensor(v_cat, v.contiguous(), group=group, async_op=True)
    k_all = k_cat.view((world,) + tuple(k.shape))
    v_all = v_cat.view((world,) + tuple(k.shape))
    parts: Dict[int, Tuple[torch.Tensor, torch.Tensor]] = {}
    order = split_order(rank, world)
    parts[order[0]] = split_attn(q, k, v, order[0])
    hk.wait()
    hv.wait()
    for s in order[1:]:
        parts[s] = split_attn(q, k_all[s], v_all[s], s)
    return merge([parts[s] for s in range(world)])
