"""Pins of the oracle's cross-attention, partial-attention (LSE) composition and key-range features.

Sources: LiteAttention README -- LSE returned "for combining results from multiple partial attention
computations" (the t2t / t2v / v2t / v2v example), must_do_list / must_skip_list (range convention
and the worked example on a length-100 sequence).
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from temporal_block_sparse_b200 import workload as wlmod

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "must_do_skip_ranges.json")


def _f64(t):
    return t.float().numpy().astype(np.float64)


def _inputs(B, H, F, gh, gw, d, seed_offset=200, locality=2.0):
    wl = wlmod.small_workload(B, H, F, gh, gw, d, locality=locality, seed_offset=seed_offset)
    q, k, v = wlmod.Trajectory(wl, device="cpu").current()
    return _f64(q), _f64(k), _f64(v)


def _sdpa(q, k, v):
    qt, kt, vt = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).permute(0, 2, 1, 3).numpy()
    s = torch.einsum("bhnd,bhmd->bhnm", qt, kt) / math.sqrt(q.shape[3])
    return out, torch.logsumexp(s, dim=-1).numpy()


def test_cross_attention_dense_matches_sdpa():
    q, _, _ = _inputs(1, 2, 1, 6, 10, 64)          # Nq = 60
    _, k, v = _inputs(1, 2, 3, 6, 11, 64, 201)     # Nk = 198
    res = oracle.lite_attention_forward(q, k, v, None, tau=-math.inf)
    o_ref, l_ref = _sdpa(q, k, v)
    np.testing.assert_allclose(res.out, o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res.lse, l_ref, rtol=1e-12)
    assert res.mask_out.shape == (1, 2, 1, 1)  # Tq = 1 query tile, Tk = 4 key tiles -> 1 word


def test_lse_merge_of_key_splits_equals_attention_over_the_union():
    q, k, v = _inputs(2, 3, 2, 9, 11, 64, 202)      # N = 198
    full = oracle.lite_attention_forward(q, k, v, None, tau=-math.inf)
    for cuts in ([70], [50, 130], [128]):
        edges = [0, *cuts, k.shape[1]]
        parts = []
        for a, e in zip(edges[:-1], edges[1:]):
            r = oracle.lite_attention_forward(q, k[:, a:e], v[:, a:e], None, tau=-math.inf)
            parts.append((r.out, r.lse))
        o, l = oracle.lse_merge(parts)
        np.testing.assert_allclose(o, full.out, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(l, full.lse, rtol=1e-12)


def test_readme_text_video_composition():
    """t2t + t2v for text rows and v2t + v2v for video rows, merged by LSE, equal full self-attention."""
    q, k, v = _inputs(1, 2, 2, 8, 12, 64, 203)      # N = 192
    text = 40
    full = oracle.lite_attention_forward(q, k, v, None, tau=-math.inf)
    sl = lambda x, a, b: x[:, a:b]
    N = q.shape[1]
    for (qa, qb) in ((0, text), (text, N)):
        parts = []
        for (ka, kb) in ((0, text), (text, N)):
            r = oracle.lite_attention_forward(sl(q, qa, qb), sl(k, ka, kb), sl(v, ka, kb), None, tau=-math.inf)
            parts.append((r.out, r.lse))
        o, l = oracle.lse_merge(parts)
        np.testing.assert_allclose(o, full.out[:, qa:qb], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(l, full.lse[:, :, qa:qb], rtol=1e-12)


def test_lse_merge_ignores_parts_without_keys():
    q, k, v = _inputs(1, 1, 1, 8, 16, 64, 204)      # N = 128 -> tiles 0, 1
    a = oracle.lite_attention_forward(q, k, v, None, tau=-math.inf)
    empty = (np.zeros_like(a.out), np.full_like(a.lse, -np.inf))
    o, l = oracle.lse_merge([(a.out, a.lse), empty])
    np.testing.assert_allclose(o, a.out, rtol=1e-13)
    np.testing.assert_allclose(l, a.lse, rtol=1e-13)
    o2, l2 = oracle.lse_merge([empty, empty])
    assert (o2 == 0).all() and np.isneginf(l2).all()


def test_readme_range_example():
    g = json.load(open(GOLDEN))
    assert sorted(oracle.range_tiles(g["must_do"], g["N"], g["tile"], whole=False)) == g["must_do_tiles"]
    assert sorted(oracle.range_tiles(g["must_skip"], g["N"], g["tile"], whole=True)) == g["must_skip_tiles"]


def _range_case():
    g = json.load(open(GOLDEN))
    wl = wlmod.small_workload(1, 2, 1, 10, 10, 16, locality=4.0, seed_offset=205)  # N = 100, d = 16
    q, k, v = (_f64(x) for x in wlmod.Trajectory(wl, device="cpu").current())
    return g, q, k, v


def test_must_skip_tiles_are_masked_and_must_do_wins():
    g, q, k, v = _range_case()
    T = 10
    res = oracle.lite_attention_forward(q, k, v, None, tau=-math.inf, tile=10, must_do=g["must_do"],
                                        must_skip=g["must_skip"])
    skipped = set(g["effective_skipped_tiles_with_both"])
    # reference: dense softmax with -inf on the skipped key tiles (every query tile)
    s = 0.25 * np.einsum("bnhd,bmhd->bhnm", q, k)
    cols = np.arange(100) // 10
    s[..., np.isin(cols, list(skipped))] = -np.inf
    lse = torch.logsumexp(torch.from_numpy(s), -1).numpy()
    out = np.einsum("bhnm,bmhd->bnhd", np.exp(s - lse[..., None]), v)
    np.testing.assert_allclose(res.out, out, rtol=1e-10, atol=1e-12)
    for t in res.tiles.values():
        assert skipped.isdisjoint(t.live) and set(g["must_do_tiles"]) <= set(t.live)


def test_must_do_tiles_are_never_flagged():
    g, q, k, v = _range_case()
    plain = oracle.lite_attention_forward(q, k, v, None, tau=-1.0, tile=10)
    forced = oracle.lite_attention_forward(q, k, v, None, tau=-1.0, tile=10, must_do=g["must_do"])
    flagged_plain = {(key, j) for key, t in plain.tiles.items() for j in t.flagged}
    flagged_forced = {(key, j) for key, t in forced.tiles.items() for j in t.flagged}
    must = set(g["must_do_tiles"])
    assert any(j in must for _, j in flagged_plain)  # the case exercises the rule
    assert flagged_forced == {(key, j) for key, j in flagged_plain if j not in must}
