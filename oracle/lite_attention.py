"""CPU oracle for the LiteAttention forward pass. TEST INFRASTRUCTURE ONLY.

This module is the slow, plain statement of what the block-sparse attention path computes. Only the
test suite, the smoke check and the benchmark's CPU-baseline leg may import it; the product path
never does, and it shares no code with the CUDA library (it only reads the same buffer layouts).

Sources (the LiteAttention pages):
  * LiteAttention README (moonmath-ai/LiteAttention, GitHub), "QK-Skip Algorithm": the Skip-Mask is
    updated at every timestep, the skipped set only grows, and a marked tile's whole attention
    iteration is bypassed at the following timesteps.
  * Same README, contribution list, "Full-Stage Elimination": a skipped tile costs no QK product, no
    softmax and no PV product.
  * Same README, must_do_list convention: the kernel walks key positions in reverse order, i.e.
    the key tiles of a query tile are visited from the highest index down.
  * Same README, Python API: thresholds are negative log-domain numbers (default -10; -6, -3 and 0
    in the examples and the threshold ablation table); thresholds above 0 are a debug-only setting.
  * "Lite Attention Temporal Sparse" skill page, Core Concept: a tile is flagged when its local
    maximum QK score is far below the cumulative maximum.
  * arXiv 2511.11062 abstract: tiles found non-essential at step t stay so at t + delta.
  * "Online normalizer calculation for softmax" (cited by the paper): the running-max softmax gives
    exactly the plain softmax; the oracle therefore states the output by its plain definition.

The QK-Skip predicate in symbols (the plainest reading that agrees with the README): for query tile i
with valid rows r, visit its live key tiles j in descending order; with m_r the maximum of
s = scale * q_r . k_c over the live tiles visited before j (m_r = -inf before the first one),
    loc_r = max over valid columns c of tile j of s_rc,
    tile j is flagged  <=>  for every valid row r: loc_r - m_r < tau,
then m_r <- max(m_r, loc_r). Flags are OR-ed into the mask that the next step reads.

Precision: inputs are bf16 values (exact in float64). Scores, softmax and output are float64. The
flag decision is an integer outcome decided by floating point, so it is taken in float32, the
precision of the GPU kernel's scores: each score is rounded to float32 and the max / difference /
compare run in float32. Margins (max_r delta_r - tau) are reported so that tiles within rounding
distance of tau can be told apart from real disagreements.

Layouts (those of the C ABI): q [B, Nq, H, d], k and v [B, Nk, H, d] (Nq = Nk = N for self
attention); lse [B, H, Nq] natural log; masks uint32 [B, H, Tq, Wk] with bit (j & 31) of word
(j >> 5) set meaning "skip key tile j"; Tq = ceil(Nq / tile), Tk = ceil(Nk / tile),
Wk = ceil(Tk / 32). Tile = 64 for d = 64 and 128 for d = 128.

Partial attentions (README, "Both LiteAttention and SeqParallelLiteAttention support returning the
softmax log-sum-exp (LSE) values for combining results from multiple partial attention
computations"): outputs over disjoint key sets combine by their LSE -- lse = log sum_p exp(lse_p),
o = sum_p exp(lse_p - lse) o_p -- which is the softmax over the union of the key sets.

Key-token ranges (README, must_do_list / must_skip_list): a list [start_0, end_0, start_1, end_1,
...] with start_i > end_i > start_{i+1} names the key tokens end_i + 1 .. start_i (start inclusive,
end exclusive, counted downwards because the kernel iterates in reverse). A key tile holding any
must-do token is always live and never flagged; a key tile lying entirely inside must-skip ranges
is always skipped; must-do wins where both apply.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

NEG_INF = -math.inf


def tile_for_head_dim(d: int) -> int:
    """Square tile edge used for head dim d (64 -> 64, 128 -> 128)."""
    if d == 64:
        return 64
    if d == 128:
        return 128
    raise ValueError(f"unsupported head dim {d}")


def geometry(N: int, d: int, tile: Optional[int] = None) -> Tuple[int, int, int]:
    """(tile, T, W): tile edge, tiles per side, 32-bit mask words per query-tile row."""
    t = tile if tile is not None else tile_for_head_dim(d)
    T = (N + t - 1) // t
    W = (T + 31) // 32
    return t, T, W


def _as_u32(mask) -> np.ndarray:
    m = np.asarray(mask)
    if m.dtype == np.int32:
        m = m.view(np.uint32)
    return m.astype(np.uint32, copy=False)


def is_skipped(mask: np.ndarray, b: int, h: int, i: int, j: int) -> bool:
    """Skip-Mask bit of (b, h, query tile i, key tile j)."""
    return bool((int(mask[b, h, i, j >> 5]) >> (j & 31)) & 1)


def live_key_tiles(mask: Optional[np.ndarray], b: int, h: int, i: int, T: int) -> List[int]:
    """Skip-List of query tile i: the key tiles not marked in the mask, highest index first."""
    if mask is None:
        return list(range(T - 1, -1, -1))
    return [j for j in range(T - 1, -1, -1) if not is_skipped(mask, b, h, i, j)]


def visit_order(tiles) -> List[int]:
    """Order in which a query tile's live key tiles are visited: highest index first (README,
    must_do_list: the kernel walks key positions in reverse order)."""
    return sorted(tiles, reverse=True)


def mask_to_list(mask, T: int) -> Tuple[np.ndarray, np.ndarray]:
    """Compaction of a Skip-Mask into per-row live lists.

    Returns (lists int16 [B,H,T,T], counts int32 [B,H,T]); entries past counts[b,h,i] are -1.
    """
    m = _as_u32(mask)
    B, H, T_, _ = m.shape
    assert T_ == T
    lists = np.full((B, H, T, T), -1, dtype=np.int16)
    counts = np.zeros((B, H, T), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(T):
                live = live_key_tiles(m, b, h, i, T)
                counts[b, h, i] = len(live)
                lists[b, h, i, : len(live)] = live
    return lists, counts


def mask_to_ranges(mask, T: int) -> Tuple[np.ndarray, np.ndarray]:
    """Range-encoded Skip-List (skill page, Architecture Overview: "Skip-List for high sparsity";
    pairs in the README's must_do_list convention: start inclusive, end exclusive, descending).

    Every maximal run of live key tiles a..b of a query tile becomes the pair (b, a - 1), runs from
    the highest down. Returns (ranges int16 [B,H,T,T+1], nruns int32 [B,H,T]); unused entries are
    -2 (a value no range entry takes).
    """
    m = _as_u32(mask)
    B, H, T_, _ = m.shape
    assert T_ == T
    ranges = np.full((B, H, T, T + 1), -2, dtype=np.int16)
    nruns = np.zeros((B, H, T), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(T):
                live = set(live_key_tiles(m, b, h, i, T))
                pairs = []
                j = T - 1
                while j >= 0:
                    if j in live:
                        top = j
                        while j >= 0 and j in live:
                            j -= 1
                        pairs += [top, j]  # j is now one below the run (a - 1)
                    else:
                        j -= 1
                nruns[b, h, i] = len(pairs) // 2
                ranges[b, h, i, : len(pairs)] = pairs
    return ranges, nruns


def schedule_order(counts) -> np.ndarray:
    """Work order over query-tile rows (flattened (b*H + h)*T + i).

    Heads are taken in order of decreasing total live-tile count (ties: lower head index first);
    inside a head, rows go by decreasing live count (ties: lower query-tile index first). This is
    a longest-processing-time-first list schedule that keeps one head's rows together so that the
    rows running at the same time read the same key/value tiles.
    """
    c = np.asarray(counts, dtype=np.int64)
    B, H, T = c.shape
    heads = c.reshape(B * H, T)
    totals = heads.sum(axis=1)
    head_order = sorted(range(B * H), key=lambda g: (-int(totals[g]), g))
    order = []
    for g in head_order:
        rows = sorted(range(T), key=lambda i: (-int(heads[g, i]), i))
        order.extend(g * T + i for i in rows)
    return np.asarray(order, dtype=np.int32)


@dataclass
class QTileResult:
    b: int
    h: int
    i: int
    rows: range
    out: np.ndarray  # [len(rows), d] float64
    lse: np.ndarray  # [len(rows)] float64
    live: List[int]  # visited key tiles, descending
    flagged: List[int]  # key tiles flagged by QK-Skip at this step
    margins: Dict[int, float] = field(default_factory=dict)  # j -> max_r delta_r - tau (float64 of fp32)


def range_tiles(ranges: Optional[Sequence[int]], Nk: int, tile: int, whole: bool) -> set:
    """Key tiles touched by a README-style range list (any token if whole=False, all tokens if True)."""
    out = set()
    if not ranges:
        return out
    r = list(ranges)
    assert len(r) % 2 == 0, "ranges come in (start, end) pairs"
    tokens = set()
    for a, e in zip(r[0::2], r[1::2]):
        assert a > e, "start_i > end_i (descending convention)"
        tokens.update(x for x in range(e + 1, a + 1) if 0 <= x < Nk)
    Tk = (Nk + tile - 1) // tile
    for j in range(Tk):
        cols = set(range(j * tile, min(Nk, (j + 1) * tile)))
        if (cols <= tokens) if whole else (cols & tokens):
            out.add(j)
    return out


def attend_query_tile(q, k, v, mask_in, b: int, h: int, i: int, tile: int, scale: float,
                      tau: float, skip_test: bool = True, force_live=frozenset(),
                      force_skip=frozenset()) -> QTileResult:
    """One query tile of one head: output, LSE and QK-Skip flags.

    q: float64 [B, Nq, H, d]; k, v: float64 [B, Nk, H, d]. mask_in: uint32 [B,H,Tq,Wk] or None.
    force_live / force_skip: key tiles the must-do / must-skip ranges pin.
    """
    N = q.shape[1]
    Nk = k.shape[1]
    T = (Nk + tile - 1) // tile
    rows = range(i * tile, min(N, (i + 1) * tile))
    d = q.shape[3]
    candidates = {j for j in live_key_tiles(mask_in, b, h, i, T) if j not in force_skip} | set(force_live)
    live = visit_order(candidates)
    if not live:
        # every key tile skipped: nothing to normalise over
        return QTileResult(b, h, i, rows, np.zeros((len(rows), d)), np.full(len(rows), NEG_INF), [], [], {})

    qi = q[b, rows.start:rows.stop, h, :]
    # step 2: scores of the live tiles, scale * q . k, float64
    scores = {}
    for j in live:
        c0, c1 = j * tile, min(Nk, (j + 1) * tile)
        scores[j] = scale * (qi @ k[b, c0:c1, h, :].T)

    # step 3: output by its plain definition -- softmax over the union of live columns
    cols = np.concatenate([np.arange(j * tile, min(Nk, (j + 1) * tile)) for j in live])
    s_all = np.concatenate([scores[j] for j in live], axis=1)
    row_max = s_all.max(axis=1)
    lse = row_max + np.log(np.exp(s_all - row_max[:, None]).sum(axis=1))
    p = np.exp(s_all - lse[:, None])
    out = p @ v[b, cols, h, :]

    # step 4: QK-Skip flags, ordered scan over live tiles from the highest index down (fp32)
    flagged: List[int] = []
    margins: Dict[int, float] = {}
    if skip_test:
        tau32 = np.float32(tau)
        m = np.full(len(rows), -np.inf, dtype=np.float32)
        for j in live:
            loc = scores[j].astype(np.float32).max(axis=1)
            with np.errstate(invalid="ignore"):
                delta = loc - m  # +inf where m = -inf
            if bool(np.all(delta < tau32)) and j not in force_live:
                flagged.append(j)
            margins[j] = float(delta.max()) - float(tau)
            m = np.maximum(m, loc)
    return QTileResult(b, h, i, rows, out, lse, live, flagged, margins)


@dataclass
class ForwardResult:
    out: np.ndarray  # [B, N, H, d] float64 (NaN for rows not computed in sampled mode)
    lse: np.ndarray  # [B, H, N] float64
    mask_out: np.ndarray  # uint32 [B, H, T, W]
    tiles: Dict[Tuple[int, int, int], QTileResult]


def lite_attention_forward(q, k, v, mask_in=None, scale: Optional[float] = None, tau: float = -10.0,
                           tile: Optional[int] = None,
                           query_tiles: Optional[Iterable[Tuple[int, int, int]]] = None,
                           skip_test: bool = True, must_do=None, must_skip=None) -> ForwardResult:
    """LiteAttention forward for one layer at one denoising step.

    q: [B, Nq, H, d]; k, v: [B, Nk, H, d] (Nq = Nk for self attention), bf16-representable values
    (any float dtype; widened to float64).
    mask_in: uint32/int32 [B, H, Tq, Wk] Skip-Mask read at this step, or None for all-live.
    must_do / must_skip: README-style key-token range lists, or None.
    scale: softmax scale; None, NaN or <= 0 gives 1/sqrt(d) (the README's Wan2.1 call passes none).
    tau: QK-Skip threshold (natural-log units of scale*QK^T); -inf disables flagging.
    query_tiles: optional list of (b, h, i) to compute (sampled mode); default all.
    skip_test: False gives the dense path (no flags; mask_out = mask_in).
    Returns output, lse, mask_out = mask_in | flags, and the per-query-tile details.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, H, d = q.shape
    Nk = k.shape[1]
    t, Tq, _ = geometry(N, d, tile)
    _, T, W = geometry(Nk, d, tile)
    force_live = range_tiles(must_do, Nk, t, whole=False)
    force_skip = range_tiles(must_skip, Nk, t, whole=True)
    if scale is None or not (scale > 0):
        scale = 1.0 / math.sqrt(d)
    if mask_in is None:
        m_in = None
        mask_out = np.zeros((B, H, Tq, W), dtype=np.uint32)
    else:
        m_in = _as_u32(mask_in).copy()
        # bits at or above T in the last word carry no tile; they read as live and are written 0
        if T % 32:
            m_in[..., W - 1] &= np.uint32((1 << (T % 32)) - 1)
        mask_out = m_in.copy()
    if query_tiles is None:
        query_tiles = [(b, h, i) for b in range(B) for h in range(H) for i in range(Tq)]
    out = np.full((B, N, H, d), np.nan)
    lse = np.full((B, H, N), np.nan)
    tiles = {}
    for (b, h, i) in query_tiles:
        r = attend_query_tile(q, k, v, m_in, b, h, i, t, scale, tau, skip_test=skip_test,
                              force_live=force_live, force_skip=force_skip)
        out[b, r.rows.start:r.rows.stop, h, :] = r.out
        lse[b, h, r.rows.start:r.rows.stop] = r.lse
        for j in r.flagged:
            mask_out[b, h, i, j >> 5] |= np.uint32(1 << (j & 31))
        tiles[(b, h, i)] = r
    return ForwardResult(out, lse, mask_out, tiles)


def dense_attention(q, k, v, scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Plain softmax attention, no tiles and no mask (the no-skip path). Returns (out, lse)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, H, d = q.shape
    if scale is None or not (scale > 0):
        scale = 1.0 / math.sqrt(d)
    out = np.empty((B, N, H, v.shape[3]))
    lse = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            s = scale * (q[b, :, h, :] @ k[b, :, h, :].T)
            mx = s.max(axis=1)
            l = mx + np.log(np.exp(s - mx[:, None]).sum(axis=1))
            out[b, :, h, :] = np.exp(s - l[:, None]) @ v[b, :, h, :]
            lse[b, h, :] = l
    return out, lse


def live_flop(mask, N: int, d: int, tile: Optional[int] = None) -> float:
    """Executed FLOP of one step: sum over live (i, j) of 4 * rows_i * cols_j * d."""
    t, T, W = geometry(N, d, tile)
    m = _as_u32(mask)
    bits = np.unpackbits(m.view(np.uint8), axis=-1, bitorder="little")[..., :T]  # [B,H,T,T] 1 = skip
    size = np.full(T, t, dtype=np.float64)
    size[T - 1] = N - (T - 1) * t
    live = 1.0 - bits.astype(np.float64)
    return float(4.0 * d * np.einsum("bhij,i,j->", live, size, size))


def lse_merge(parts: Sequence[Tuple[np.ndarray, np.ndarray]]) -> Tuple[np.ndarray, np.ndarray]:
    """Combine partial attentions over disjoint key sets by their LSE.

    parts: [(out [B, N, H, d], lse [B, H, N]), ...]. A part whose lse is -inf for a row (no key
    there) contributes nothing to that row; if every part is -inf the row is 0 with lse -inf.
    """
    lses = np.stack([np.asarray(l, dtype=np.float64) for _, l in parts])  # [P, B, H, N]
    outs = np.stack([np.asarray(o, dtype=np.float64) for o, _ in parts])  # [P, B, N, H, d]
    mx = lses.max(axis=0)
    finite = np.isfinite(mx)
    safe = np.where(finite, mx, 0.0)
    w = np.where(np.isneginf(lses), 0.0, np.exp(lses - safe[None]))  # [P, B, H, N]
    tot = w.sum(axis=0)
    lse = np.where(finite, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    wn = np.where(tot > 0, w / np.where(tot > 0, tot, 1.0)[None], 0.0)  # [P, B, H, N]
    out = np.einsum("pbhn,pbnhd->bnhd", wn, outs)
    return out, lse
