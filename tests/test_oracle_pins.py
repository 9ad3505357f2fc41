"""Pins of the CPU oracle against things other than itself (CPU only).

Each test ties the oracle to a statement that the LiteAttention pages or plain mathematics fix:
a hand-worked example, brute-force attention, a textbook library routine for the no-skip case, the
additive -inf masking definition of the skill page's Step 2 listing, a non-iterative restatement of
the flag rule, and the invariants the README states (monotone mask, skipped mass bounded by the
threshold). A few tests plant a mistake in the oracle and check that a pin catches it.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import lite_attention as ola
from temporal_block_sparse_b200 import workload as wlmod

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "qk_skip_hand_example.json")


def _f64(t):
    return t.float().numpy().astype(np.float64)


def _traj_inputs(B, H, frames, gh, gw, d, locality=2.0, seed_offset=100, steps=1):
    wl = wlmod.small_workload(B, H, frames, gh, gw, d, steps=steps, locality=locality, seed_offset=seed_offset)
    tr = wlmod.Trajectory(wl, device="cpu")
    return wl, tr


def _words_from_bits(bits):
    """bits: bool [..., T] -> uint32 words [..., ceil(T/32)]."""
    T = bits.shape[-1]
    W = (T + 31) // 32
    pad = np.zeros(bits.shape[:-1] + (W * 32,), dtype=bool)
    pad[..., :T] = bits
    w = np.zeros(bits.shape[:-1] + (W,), dtype=np.uint64)
    for b in range(32):
        w |= pad[..., b::32].astype(np.uint64) << np.uint64(b)
    return w.astype(np.uint32)


def _bits_from_words(words, T):
    u = np.asarray(words).view(np.uint32) if np.asarray(words).dtype == np.int32 else np.asarray(words, np.uint32)
    return np.unpackbits(u.view(np.uint8), axis=-1, bitorder="little")[..., :T].astype(bool)


# --------------------------------------------------------------------------------------------- golden


def _load_golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _golden_inputs(g):
    s = np.array(g["scores"], dtype=np.float64)
    N = s.shape[0]
    q = s[None, :, None, :]  # [1, N, 1, d=N]
    k = np.eye(N)[None, :, None, :]
    v = np.eye(N)[None, :, None, :]
    return q, k, v


@pytest.mark.parametrize("case_idx", range(4))
def test_hand_worked_example(case_idx):
    g = _load_golden()
    case = g["cases"][case_idx]
    q, k, v = _golden_inputs(g)
    tau = float(case["tau"])
    mask_in = np.array(case["mask_in"], dtype=np.uint32).reshape(1, 1, 3, 1)
    res = oracle.lite_attention_forward(q, k, v, mask_in, scale=g["scale"], tau=tau, tile=g["tile"])
    assert res.mask_out.reshape(-1).tolist() == case["mask_out"]
    for i, flags in case["flags"].items():
        assert res.tiles[(0, 0, int(i))].flagged == flags, (case["name"], i)


def test_hand_example_output_is_masked_softmax():
    # rows of q-tile 0 with tile 2 skipped: softmax over columns 0..3 only, columns 4,5 get zero weight
    g = _load_golden()
    q, k, v = _golden_inputs(g)
    mask_in = np.array([4, 0, 0], dtype=np.uint32).reshape(1, 1, 3, 1)
    res = oracle.lite_attention_forward(q, k, v, mask_in, scale=1.0, tau=-3.0, tile=2)
    s = np.array(g["scores"])
    for r in (0, 1):
        w = np.exp(s[r, :4] - s[r, :4].max())
        w /= w.sum()
        np.testing.assert_allclose(res.out[0, r, 0, :4], w, rtol=1e-13)
        assert res.out[0, r, 0, 4] == 0 and res.out[0, r, 0, 5] == 0
        assert res.lse[0, 0, r] == pytest.approx(math.log(sum(math.exp(x) for x in s[r, :4])), rel=1e-13)


def test_planted_ascending_order_is_caught(monkeypatch):
    """Plant a mistake in the oracle (ascending key-tile order); the hand example must reject it."""
    g = _load_golden()
    q, k, v = _golden_inputs(g)
    monkeypatch.setattr(ola, "visit_order", lambda tiles: sorted(tiles))
    case = g["cases"][0]
    res = oracle.lite_attention_forward(q, k, v, np.zeros((1, 1, 3, 1), np.uint32), scale=1.0,
                                        tau=case["tau"], tile=2)
    assert res.mask_out.reshape(-1).tolist() != case["mask_out"]


def test_planted_dropped_scale_is_caught(monkeypatch):
    """Plant a mistake (scale ignored): brute-force attention must reject it."""
    wl, tr = _traj_inputs(1, 1, 1, 4, 8, 64)
    q, k, v = (_f64(x) for x in tr.current())
    ref_o, ref_l = _brute_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], 1 / 8.0)
    orig = ola.attend_query_tile

    def bad(q_, k_, v_, m_, b, h, i, tile, scale, tau, skip_test=True, **kw):
        return orig(q_, k_, v_, m_, b, h, i, tile, 1.0, tau, skip_test, **kw)

    monkeypatch.setattr(ola, "attend_query_tile", bad)
    res = oracle.lite_attention_forward(q, k, v, None, tau=-math.inf)
    assert not np.allclose(res.lse[0, 0], ref_l, rtol=1e-6)


# ---------------------------------------------------------------------------- P1: dense = brute force


def _brute_head(q, k, v, scale):
    """Naive softmax attention, one head, scalar Python loops with exact summation."""
    N, d = q.shape
    out = np.zeros((N, v.shape[1]))
    lse = np.zeros(N)
    for r in range(N):
        s = [scale * math.fsum(float(q[r, x]) * float(k[c, x]) for x in range(d)) for c in range(N)]
        mx = max(s)
        lse[r] = mx + math.log(math.fsum(math.exp(x - mx) for x in s))
        for c in range(N):
            out[r] += math.exp(s[c] - lse[r]) * v[c]
    return out, lse


@pytest.mark.parametrize("shape", [(1, 1, 2, 5, 15, 64), (1, 1, 1, 10, 13, 128)])
def test_dense_equals_brute_force(shape):
    """tau=-inf and an all-zero mask give plain softmax attention (N=150/130: ragged tail tile)."""
    B, H, F, gh, gw, d = shape
    wl, tr = _traj_inputs(B, H, F, gh, gw, d)
    q, k, v = (_f64(x) for x in tr.current())
    res = oracle.lite_attention_forward(q, k, v, np.zeros((B, H, *oracle.geometry(wl.N, d)[1:]), np.uint32),
                                        tau=-math.inf)
    scale = 1.0 / math.sqrt(d)
    o_ref, l_ref = _brute_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], scale)
    np.testing.assert_allclose(res.out[0, :, 0], o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(res.lse[0, 0], l_ref, rtol=1e-12)
    assert (res.mask_out == 0).all()


def test_dense_matches_library_sdpa():
    """The no-skip case reduces to the textbook routine (torch SDPA in float64 on CPU)."""
    wl, tr = _traj_inputs(2, 3, 2, 9, 11, 64)
    q, k, v = tr.current()
    res = oracle.lite_attention_forward(_f64(q), _f64(k), _f64(v), None, tau=-math.inf)
    qt, kt, vt = (x.double().permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(res.out, ref, rtol=1e-10, atol=1e-12)
    o2, l2 = oracle.dense_attention(_f64(q), _f64(k), _f64(v))
    np.testing.assert_allclose(o2, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res.lse, l2, rtol=1e-12)
    s = torch.einsum("bnhd,bmhd->bhnm", qt.permute(0, 2, 1, 3), kt.permute(0, 2, 1, 3)) / 8.0
    np.testing.assert_allclose(res.lse, torch.logsumexp(s, dim=-1).numpy(), rtol=1e-12)


# --------------------------------------------------------------- P2: masked = additive -inf bias


def _bias_reference(q, k, v, mask, tile, scale):
    """Dense softmax over all keys with -inf added on skipped blocks (the skill page's Step 2 masking)."""
    B, N, H, d = q.shape
    T = (N + tile - 1) // tile
    bits = _bits_from_words(mask, T)  # [B,H,T,T]
    tok = np.arange(N) // tile
    out = np.zeros_like(q)
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            s = torch.from_numpy(scale * (q[b, :, h] @ k[b, :, h].T))
            blocked = torch.from_numpy(bits[b, h][tok[:, None], tok[None, :]])
            s = s.masked_fill(blocked, -math.inf)
            l = torch.logsumexp(s, dim=-1)
            p = torch.exp(s - l[:, None])
            p = torch.nan_to_num(p, nan=0.0)
            out[b, :, h] = (p @ torch.from_numpy(v[b, :, h])).numpy()
            lse[b, h] = l.numpy()
    return out, lse


@pytest.mark.parametrize("tile,density", [(8, 0.3), (8, 0.7), (64, 0.5)])
def test_masked_output_equals_additive_bias(tile, density):
    wl, tr = _traj_inputs(1, 2, 2, 7, 9, 64)  # N=126
    q, k, v = (_f64(x) for x in tr.current())
    T = (wl.N + tile - 1) // tile
    mask = wlmod.random_mask(1, 2, T, density, seed=7).numpy().view(np.uint32)
    res = oracle.lite_attention_forward(q, k, v, mask, tau=-math.inf, tile=tile)
    o_ref, l_ref = _bias_reference(q, k, v, mask, tile, 1 / 8.0)
    np.testing.assert_allclose(res.out, o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res.lse, l_ref, rtol=1e-12)


def test_empty_live_set_gives_zero_and_minus_inf():
    wl, tr = _traj_inputs(1, 1, 1, 8, 16, 64)  # N=128, tile 64, T=2
    q, k, v = (_f64(x) for x in tr.current())
    mask = np.array([[[[3], [0]]]], dtype=np.uint32)
    res = oracle.lite_attention_forward(q, k, v, mask, tau=-3.0)
    assert (res.out[0, :64] == 0).all() and np.isneginf(res.lse[0, 0, :64]).all()
    assert np.isfinite(res.lse[0, 0, 64:]).all()
    assert res.mask_out[0, 0, 0, 0] == 3


def test_bits_beyond_T_are_ignored_and_cleared():
    wl, tr = _traj_inputs(1, 1, 1, 8, 16, 64)  # T=2
    q, k, v = (_f64(x) for x in tr.current())
    clean = np.zeros((1, 1, 2, 1), np.uint32)
    dirty = clean | np.uint32(0xFFFFFFFC)
    a = oracle.lite_attention_forward(q, k, v, clean, tau=-math.inf)
    b = oracle.lite_attention_forward(q, k, v, dirty, tau=-math.inf)
    np.testing.assert_array_equal(a.out, b.out)
    assert (b.mask_out == 0).all()


@pytest.mark.parametrize("scale", [None, 0.0, -1.0, float("nan")])
def test_default_scale_is_inverse_sqrt_d(scale):
    wl, tr = _traj_inputs(1, 1, 1, 4, 16, 64)
    q, k, v = (_f64(x) for x in tr.current())
    a = oracle.lite_attention_forward(q, k, v, None, scale=scale, tau=-math.inf)
    b = oracle.lite_attention_forward(q, k, v, None, scale=0.125, tau=-math.inf)
    np.testing.assert_array_equal(a.out, b.out)


# ------------------------------------------------------------ P3: flags, non-iterative closed form


def _closed_form_flags(q, k, mask, tile, scale, tau):
    """flag(i,j) <=> j live, some live j' > j, and for every valid row r:
    max_{c in j} s_rc - max_{c in live tiles above j} s_rc < tau  (scores rounded to float32)."""
    B, N, H, d = q.shape
    T = (N + tile - 1) // tile
    bits = _bits_from_words(mask, T) if mask is not None else np.zeros((B, H, T, T), bool)
    tau32 = np.float32(tau)
    flags = np.zeros((B, H, T, T), dtype=bool)
    for b in range(B):
        for h in range(H):
            s = (scale * (torch.from_numpy(q[b, :, h]) @ torch.from_numpy(k[b, :, h]).T)).float().numpy()
            # per-tile row maxima [N, T]
            tmax = np.stack([s[:, j * tile:min(N, (j + 1) * tile)].max(axis=1) for j in range(T)], axis=1)
            for i in range(T):
                rows = slice(i * tile, min(N, (i + 1) * tile))
                live = ~bits[b, h, i]
                for j in range(T):
                    above = [jj for jj in range(j + 1, T) if live[jj]]
                    if not live[j] or not above:
                        continue
                    m = tmax[rows][:, above].max(axis=1)
                    flags[b, h, i, j] = bool(np.all(tmax[rows, j] - m < tau32))
    return flags


@pytest.mark.parametrize("tau,density,locality", [(-3.0, 0.0, 4.0), (-1.0, 0.2, 2.0), (-6.0, 0.3, 5.0),
                                                  (0.0, 0.0, 1.0)])
def test_flags_match_closed_form(tau, density, locality):
    wl, tr = _traj_inputs(2, 2, 2, 6, 9, 16, locality=locality, seed_offset=11)  # N=108, tile 8 -> T=14
    q, k, v = (_f64(x) for x in tr.current())
    tile = 8
    T = (wl.N + tile - 1) // tile
    mask = wlmod.random_mask(2, 2, T, density, seed=3).numpy().view(np.uint32)
    res = oracle.lite_attention_forward(q, k, v, mask, scale=0.25, tau=tau, tile=tile)
    cf = _closed_form_flags(q, k, mask, tile, 0.25, tau)
    got = _bits_from_words(res.mask_out, T) & ~_bits_from_words(mask, T)
    np.testing.assert_array_equal(got, cf)
    # the inputs must exercise both outcomes
    assert cf.sum() > 10 and (~cf & ~_bits_from_words(mask, T)).sum() > 10


# --------------------------------------------------------------------------- P4: invariants over steps


def test_mask_monotone_and_rows_never_empty_over_steps():
    wl, tr = _traj_inputs(1, 2, 3, 6, 8, 16, locality=3.0, seed_offset=12, steps=6)  # N=144
    tile = 8
    T = (wl.N + tile - 1) // tile
    mask = np.zeros((1, 2, T, (T + 31) // 32), np.uint32)
    grew = 0
    for t, (q, k, v) in enumerate(tr):
        res = oracle.lite_attention_forward(_f64(q), _f64(k), _f64(v), mask, tau=-2.0, tile=tile)
        before, after = _bits_from_words(mask, T), _bits_from_words(res.mask_out, T)
        assert (after | before == after).all()  # monotone
        for key, r in res.tiles.items():
            if r.live:
                assert r.live[0] not in r.flagged  # first visited tile is never flagged
        assert (~after).any(axis=-1).all()  # no query tile loses every key tile
        grew += int(after.sum() - before.sum())
        mask = res.mask_out
    assert grew > 0


def test_minus_inf_tau_never_flags():
    wl, tr = _traj_inputs(1, 2, 2, 6, 8, 16, locality=4.0, seed_offset=13)
    q, k, v = (_f64(x) for x in tr.current())
    res = oracle.lite_attention_forward(q, k, v, None, tau=-math.inf, tile=8)
    assert (res.mask_out == 0).all()


# ------------------------------------------------------------------------ P5: skipped-mass bound


@pytest.mark.parametrize("tau", [-3.0, -6.0, -1.0])
def test_flagged_tiles_have_bounded_probability(tau):
    wl, tr = _traj_inputs(1, 2, 3, 6, 8, 16, locality=3.0, seed_offset=14)
    q, k, v = (_f64(x) for x in tr.current())
    tile = 8
    N = wl.N
    res = oracle.lite_attention_forward(q, k, v, None, scale=0.25, tau=tau, tile=tile)
    nflag = 0
    for (b, h, i), r in res.tiles.items():
        s = 0.25 * (q[b, :, h] @ k[b, :, h].T)
        p_dense = np.exp(s - torch.logsumexp(torch.from_numpy(s), -1).numpy()[:, None])
        for j in r.flagged:
            nflag += 1
            blk = p_dense[r.rows.start:r.rows.stop, j * tile:min(N, (j + 1) * tile)]
            assert (blk < math.exp(tau) * (1 + 1e-6)).all()
            assert (blk.sum(axis=1) < blk.shape[1] * math.exp(tau) * (1 + 1e-6)).all()
    assert nflag > 0


# ----------------------------------------------------------------------- P6: tile-order invariance


def test_output_invariant_to_key_tile_order_when_nothing_skipped():
    wl, tr = _traj_inputs(1, 2, 2, 8, 8, 64)  # N=128, tile 64 -> 2 tiles; use tile 16 -> 8 tiles
    q, k, v = (_f64(x) for x in tr.current())
    tile = 16
    T = wl.N // tile
    perm = np.random.default_rng(5).permutation(T)
    idx = np.concatenate([np.arange(p * tile, (p + 1) * tile) for p in perm])
    a = oracle.lite_attention_forward(q, k, v, None, tau=-math.inf, tile=tile)
    b = oracle.lite_attention_forward(q, k[:, idx], v[:, idx], None, tau=-math.inf, tile=tile)
    np.testing.assert_allclose(a.out, b.out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(a.lse, b.lse, rtol=1e-13)


# --------------------------------------------------------------------- compaction and scheduling


def test_mask_to_list_invariants():
    T = 45
    mask = wlmod.random_mask(2, 3, T, 0.6, seed=9).numpy().view(np.uint32)
    lists, counts = oracle.mask_to_list(mask, T)
    bits = _bits_from_words(mask, T)
    np.testing.assert_array_equal(counts, T - bits.sum(-1))
    for b in range(2):
        for h in range(3):
            for i in range(T):
                n = counts[b, h, i]
                row = lists[b, h, i, :n]
                assert (np.diff(row) < 0).all()
                assert not bits[b, h, i, row].any()
                assert (lists[b, h, i, n:] == -1).all()


def test_schedule_order_is_grouped_lpt_permutation():
    rng = np.random.default_rng(3)
    counts = rng.integers(0, 20, size=(2, 3, 17))
    order = oracle.schedule_order(counts)
    T = 17
    assert sorted(order.tolist()) == list(range(2 * 3 * T))
    heads = order // T
    totals = counts.reshape(6, T).sum(1)
    # each head's rows are contiguous and heads come by decreasing total
    for g in range(6):
        pos = np.nonzero(heads == g)[0]
        assert pos.max() - pos.min() == T - 1
    head_seq = heads[::T]
    assert all(totals[head_seq[x]] >= totals[head_seq[x + 1]] for x in range(5))
    flat = counts.reshape(-1)
    for g in range(6):
        c = flat[order[g * T:(g + 1) * T]]
        assert (np.diff(c) <= 0).all()


def test_live_flop_counts_tail_sizes():
    N, d, tile = 150, 64, 64  # tiles of 64, 64, 22
    m = np.zeros((1, 1, 3, 1), np.uint32)
    m[0, 0, 0, 0] = 0b100  # skip (0, 2)
    full = 4 * d * (150 * 150)
    assert oracle.live_flop(m, N, d) == full - 4 * d * 64 * 22
