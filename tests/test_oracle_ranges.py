"""Pins for the oracle's range-encoded Skip-List (CPU).

Skill page "Lite Attention Temporal Sparse", Architecture Overview: the Skip-Mask may be held as a
Skip-List for high sparsity; README must_do_list: ranges are (start inclusive, end exclusive) pairs
in strictly descending order. Pinned by: expansion of the ranges gives exactly the per-tile live
list of mask_to_list, the pairs are well formed and maximal, and hand-written special cases.
"""

import numpy as np
import pytest

import oracle


def _mask_from_live(B, H, T, live_sets):
    W = (T + 31) // 32
    m = np.zeros((B, H, T, W), dtype=np.uint32)
    for (b, h, i), live in live_sets.items():
        for j in range(T):
            if j not in live:
                m[b, h, i, j >> 5] |= np.uint32(1 << (j & 31))
    return m


def _expand(row, n):
    out = []
    for k in range(n):
        start, end = int(row[2 * k]), int(row[2 * k + 1])
        out += list(range(start, end, -1))
    return out


@pytest.mark.parametrize("T,density,seed", [(1, 0.5, 0), (16, 0.5, 1), (33, 0.2, 2), (64, 0.9, 3), (100, 0.05, 4)])
def test_ranges_expand_to_the_live_list(T, density, seed):
    rng = np.random.default_rng(seed)
    B, H = 2, 2
    W = (T + 31) // 32
    mask = rng.integers(0, 2**32, size=(B, H, T, W), dtype=np.uint64).astype(np.uint32)
    keep = rng.random((B, H, T, W * 32)) < density  # extra live tiles to vary run lengths
    for b in range(B):
        for h in range(H):
            for i in range(T):
                for j in range(T):
                    if keep[b, h, i, j]:
                        mask[b, h, i, j >> 5] &= ~np.uint32(1 << (j & 31))
    lists, counts = oracle.mask_to_list(mask, T)
    ranges, nruns = oracle.mask_to_ranges(mask, T)
    for b in range(B):
        for h in range(H):
            for i in range(T):
                row, n = ranges[b, h, i], int(nruns[b, h, i])
                assert _expand(row, n) == list(lists[b, h, i, : counts[b, h, i]])
                vals = [int(x) for x in row[: 2 * n]]
                assert all(vals[2 * k] > vals[2 * k + 1] for k in range(n))              # start > end
                assert all(vals[2 * k + 1] > vals[2 * k + 2] for k in range(n - 1))      # runs are maximal
                assert all(-1 <= x < T for x in vals)


def test_ranges_special_cases():
    T = 40
    full_live = _mask_from_live(1, 1, T, {(0, 0, i): set(range(T)) for i in range(T)})
    r, n = oracle.mask_to_ranges(full_live, T)
    assert (n == 1).all() and (r[..., 0] == T - 1).all() and (r[..., 1] == -1).all()
    none_live = _mask_from_live(1, 1, T, {(0, 0, i): set() for i in range(T)})
    _, n = oracle.mask_to_ranges(none_live, T)
    assert (n == 0).all()
    alt = _mask_from_live(1, 1, T, {(0, 0, i): set(range(0, T, 2)) for i in range(T)})
    r, n = oracle.mask_to_ranges(alt, T)
    assert (n == T // 2).all()
    assert list(r[0, 0, 0, :4]) == [38, 37, 36, 35]
    # a README-style example in tiles: live 31..20 and 5..2 -> [31, 19, 5, 1]
    one = _mask_from_live(1, 1, T, {(0, 0, 0): set(range(20, 32)) | set(range(2, 6))})
    r, n = oracle.mask_to_ranges(one, T)
    assert n[0, 0, 0] == 2 and list(r[0, 0, 0, :4]) == [31, 19, 5, 1]
