"""GPU path vs the CPU oracle, through the C ABI (needs a B200).

Small cases are compared element by element over every row; the full-size workloads (480p, 720p,
stress) run in the same launch configuration the benchmark uses and are compared on sampled query
tiles (always including the first and the ragged last one). Across denoising steps the oracle is
teacher-forced: at step t it reads the GPU's own mask_in, so one near-threshold flip cannot cascade.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from temporal_block_sparse_b200 import lite_attn as la
from temporal_block_sparse_b200 import workload as wl

from gpu_parity import assert_within, compare, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(autouse=True)
def _clean_state():
    la.load()
    yield
    la.lite_set_option(la.LITE_OPT_MAX_CTAS, 0)
    la.lite_set_option(la.LITE_OPT_DEBUG_STALL, 0)
    la.lite_set_option(la.LITE_OPT_WAIT_LIMIT_NS, 4_000_000_000)
    assert la.lite_get_device_status() == 0


def _np(t):
    return to_np(t)


def oracle_step(q, k, v, mask_in, tau, query_tiles=None, skip_test=True):
    """Run the oracle on (q, k, v) GPU tensors; in sampled mode only the needed heads go to the host."""
    mi = None if mask_in is None else mask_in.cpu().numpy().view(np.uint32)
    if query_tiles is None:
        return oracle.lite_attention_forward(_np(q), _np(k), _np(v), mi, tau=tau, skip_test=skip_test)
    B, N, H, d = q.shape
    _, T, W = oracle.geometry(N, d)
    out = np.full((B, N, H, d), np.nan)
    lse = np.full((B, H, N), np.nan)
    mask_out = mi.copy() if mi is not None else np.zeros((B, H, T, W), np.uint32)
    tiles = {}
    heads = sorted({(b, h) for b, h, _ in query_tiles})
    for b, h in heads:
        qs = [(0, 0, i) for bb, hh, i in query_tiles if (bb, hh) == (b, h)]
        sub = lambda x: _np(x[b:b + 1, :, h:h + 1, :])
        m = None if mi is None else mi[b:b + 1, h:h + 1]
        r = oracle.lite_attention_forward(sub(q), sub(k), sub(v), m, tau=tau, query_tiles=qs, skip_test=skip_test)
        out[b, :, h] = r.out[0, :, 0]
        lse[b, h] = r.lse[0, 0]
        for (_, _, i), t in r.tiles.items():
            mask_out[b, h, i] = r.mask_out[0, 0, i]
            t.b, t.h = b, h
            tiles[(b, h, i)] = t
    return oracle.ForwardResult(out, lse, mask_out, tiles)


# --------------------------------------------------------------------------- compaction, schedule


@pytest.mark.parametrize("B,H,N,d,density,dirty", [
    (1, 1, 1024, 64, 0.0, False), (2, 3, 1000, 64, 0.4, True), (1, 2, 75600, 128, 0.7, True),
    (2, 1, 4100, 128, 0.95, False), (1, 1, 100, 128, 1.0, True), (1, 1, 8192 * 2 + 5, 64, 0.5, True)])
def test_compaction_matches_oracle(B, H, N, d, density, dirty):
    _, T, W = la.lite_mask_geometry(N, d)
    mask = wl.random_mask(B, H, T, density, seed=N + B).cuda()
    if dirty and T % 32:
        mask[..., W - 1] |= torch.tensor(-(1 << (T % 32)), dtype=torch.int32)  # junk above bit T
    lst, counts = la.lite_mask_to_list(mask, B, H, N, d)
    rl, rc = oracle.mask_to_list(mask.cpu().numpy(), T)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(lst.cpu().numpy(), rl)


def test_compaction_without_mask_lists_every_tile():
    lst, counts = la.lite_mask_to_list(None, 1, 2, 700, 128)
    T = 6
    assert (counts.cpu().numpy() == T).all()
    assert (lst.cpu().numpy()[..., :] == np.arange(T - 1, -1, -1)).all()


@pytest.mark.parametrize("B,H,T,hi", [(1, 1, 16, 16), (1, 40, 256, 256), (2, 40, 591, 591), (3, 5, 77, 3)])
def test_schedule_matches_oracle(B, H, T, hi):
    g = torch.Generator().manual_seed(T)
    counts = torch.randint(0, hi + 1, (B, H, T), generator=g, dtype=torch.int32)
    order = la.lite_schedule(counts.cuda())
    np.testing.assert_array_equal(order.cpu().numpy(), oracle.schedule_order(counts.numpy()))


# ------------------------------------------------------------------------------ small, all rows


def _trajectory_parity(w, steps, tau, mask_density=0.0, seed=1, in_place=False):
    tr = wl.Trajectory(w, device="cuda")
    B, N, H, d = w.B, w.N, w.H, w.d
    _, T, W = la.lite_mask_geometry(N, d)
    m_in = wl.random_mask(B, H, T, mask_density, seed=seed).cuda() if mask_density else la.new_mask(B, H, N, d)
    reports = []
    for t in range(steps):
        q, k, v = tr.current()
        m_out = m_in if in_place else torch.full_like(m_in, 0x5A5A5A5A)
        m_before = m_in.clone()
        o, lse = la.lite_attn_fwd(q, k, v, m_in, m_out, tau=tau)
        assert la.lite_get_device_status() == 0
        ref = oracle_step(q, k, v, m_before, tau)
        rep = compare(o, lse, m_out, ref)
        assert_within(rep)
        got = m_out.cpu().numpy().view(np.uint32)
        assert ((got & m_before.cpu().numpy().view(np.uint32)) == m_before.cpu().numpy().view(np.uint32)).all()
        reports.append(rep)
        m_in = m_out
        tr.advance()
    return reports


def test_tiny_workload_all_steps():
    """The tiny workload: 4 frames x 16x16, d=64, tile 64, 5 steps, tau=-3."""
    w = wl.WORKLOADS["tiny"]
    _trajectory_parity(w, w.steps, w.tau(0))


@pytest.mark.parametrize("B,H,F,gh,gw,d,tau,density", [
    (1, 2, 3, 10, 10, 128, -3.0, 0.0),     # N=300: tail tile of 44
    (2, 3, 2, 9, 11, 64, -2.0, 0.3),       # N=198, tile 64, random skips
    (1, 1, 1, 5, 10, 128, -3.0, 0.0),      # N=50 < one tile
    (1, 4, 5, 8, 16, 128, -10.0, 0.2),     # N=640 exact multiple
    (2, 2, 4, 8, 9, 128, -1.0, 0.5),       # N=288, dense-ish flags
])
def test_small_shapes(B, H, F, gh, gw, d, tau, density):
    w = wl.small_workload(B, H, F, gh, gw, d, steps=3, locality=3.0, tau=tau, seed_offset=F * gh + gw)
    reps = _trajectory_parity(w, 3, tau, mask_density=density, seed=gh)
    print(f"flagged={sum(r.flagged for r in reps)} near-tau mismatches={sum(r.mask_mismatches for r in reps)}")


def test_in_place_mask_update():
    w = wl.small_workload(1, 2, 3, 8, 10, 128, steps=3, locality=3.0, tau=-3.0, seed_offset=9)
    _trajectory_parity(w, 3, -3.0, in_place=True)


def test_optional_outputs_and_no_mask():
    w = wl.small_workload(1, 2, 2, 8, 10, 128, locality=3.0, seed_offset=3)
    q, k, v = wl.Trajectory(w, device="cuda").current()
    ref = oracle_step(q, k, v, None, -3.0)
    o, _ = la.lite_attn_fwd(q, k, v, None, None, tau=-3.0, return_lse=False)
    assert_within(compare(o, None, None, ref, check_mask=False))
    m = la.new_mask(1, 2, w.N, 128)
    o2, lse2 = la.lite_attn_fwd(q, k, v, None, m, tau=-3.0)
    assert_within(compare(o2, lse2, m, ref))


@pytest.mark.parametrize("d,gw", [(64, 15), (128, 14)])
def test_paired_query_tiles_with_disjoint_lists(d, gw):
    """The kernel pairs query tiles and walks the union of their Skip-Lists; with d = 64 each
    128-row kernel tile stacks two 64-row mask rows. Here neighbouring query tiles have disjoint
    live sets: even key tiles for one, odd for the other, so most union tiles (and, at d = 64,
    every key tile of a stacked pair of rows) are live for one query tile only. One pair has a fully skipped tile, and an
    odd tile count leaves the last query tile without a partner. All rows against the oracle,
    three steps with QK-Skip on."""
    tile = 64 if d == 64 else 128
    w = wl.small_workload(1, 2, 5, 9, gw, d, steps=3, locality=3.0, tau=-2.0, seed_offset=77 + d)
    B, N, H = w.B, w.N, w.H
    _, T, W = la.lite_mask_geometry(N, d)
    assert T % 2 == 1 and N % tile != 0
    bits = torch.zeros((B, H, T, W * 32), dtype=torch.bool)
    for i in range(T):
        bits[:, :, i, (i + 1) % 2:T:2] = True  # tile i skips the key tiles of the other parity
    bits[:, 1, 2, :T] = True                   # head 1: query tile 2 fully skipped
    weights = 2 ** torch.arange(32, dtype=torch.int64)
    words = (bits.view(B, H, T, W, 32).to(torch.int64) * weights).sum(-1)
    mask = torch.where(words >= 2 ** 31, words - 2 ** 32, words).to(torch.int32).cuda()
    tr = wl.Trajectory(w, device="cuda")
    for t in range(w.steps):
        q, k, v = tr.current()
        m_out = torch.empty_like(mask)
        o, lse = la.lite_attn_fwd(q, k, v, mask, m_out, tau=-2.0)
        assert la.lite_get_device_status() == 0
        ref = oracle_step(q, k, v, mask, -2.0)
        assert_within(compare(o, lse, m_out, ref))
        mask = m_out
        tr.advance()


def test_fully_skipped_row_gives_zero_and_minus_inf():
    w = wl.small_workload(1, 1, 2, 8, 16, 128, seed_offset=4)  # N=256, T=2
    q, k, v = wl.Trajectory(w, device="cuda").current()
    mask = torch.tensor([[[[3], [1]]]], dtype=torch.int32, device="cuda")
    o, lse = la.lite_attn_fwd(q, k, v, mask, mask, tau=-3.0)
    ref = oracle_step(q, k, v, mask, -3.0)
    assert (o[0, :128].float() == 0).all() and torch.isneginf(lse[0, 0, :128]).all()
    assert_within(compare(o, lse, None, ref, check_mask=False))


def test_minus_inf_tau_records_no_flags():
    w = wl.small_workload(1, 2, 3, 8, 10, 128, locality=6.0, seed_offset=5)
    q, k, v = wl.Trajectory(w, device="cuda").current()
    m_in = la.new_mask(1, 2, w.N, 128)
    m_out = torch.full_like(m_in, -1)
    la.lite_attn_fwd(q, k, v, m_in, m_out, tau=-math.inf)
    assert (m_out == 0).all()


@pytest.mark.parametrize("d", [64, 128])
def test_dense_path_matches_oracle_and_sdpa(d):
    w = wl.small_workload(2, 3, 3, 7, 9, d, locality=2.0, seed_offset=d)  # N=189
    q, k, v = wl.Trajectory(w, device="cuda").current()
    o, lse = la.lite_attn_dense(q, k, v)
    ref = oracle_step(q, k, v, None, -math.inf, skip_test=False)
    assert_within(compare(o, lse, None, ref, check_mask=False))
    sd = torch.nn.functional.scaled_dot_product_attention(*(x.transpose(1, 2).float() for x in (q, k, v)))
    assert (o.float() - sd.transpose(1, 2)).abs().max().item() <= 2e-2


def test_persistent_loop_with_few_ctas():
    """Many items per CTA: barrier phases and TMEM reuse across items."""
    la.lite_set_option(la.LITE_OPT_MAX_CTAS, 3)
    w = wl.small_workload(2, 3, 4, 8, 12, 128, steps=2, locality=3.0, seed_offset=21)  # N=384, 36 items
    _trajectory_parity(w, 2, -3.0, mask_density=0.2, seed=5)
    la.lite_set_option(la.LITE_OPT_MAX_CTAS, 1)
    w64 = wl.small_workload(1, 2, 4, 8, 12, 64, steps=2, locality=3.0, seed_offset=22)
    _trajectory_parity(w64, 2, -3.0)


def test_timeout_is_reported_and_context_survives():
    """A wait that nothing completes (test hook) gives up after its limit and sets the status word."""
    w = wl.small_workload(1, 1, 2, 8, 16, 128, seed_offset=6)
    q, k, v = wl.Trajectory(w, device="cuda").current()
    la.lite_set_option(la.LITE_OPT_WAIT_LIMIT_NS, 20_000_000)  # 20 ms
    la.lite_set_option(la.LITE_OPT_DEBUG_STALL, 1)
    la.lite_attn_fwd(q, k, v, None, None, tau=-3.0)
    assert la.lite_get_device_status() == la.LITE_ERR_TIMEOUT
    la.lite_set_option(la.LITE_OPT_DEBUG_STALL, 0)
    la.lite_set_option(la.LITE_OPT_WAIT_LIMIT_NS, 4_000_000_000)
    o, lse = la.lite_attn_fwd(q, k, v, None, None, tau=-3.0)
    assert la.lite_get_device_status() == 0
    assert_within(compare(o, lse, None, oracle_step(q, k, v, None, -3.0), check_mask=False))


# ------------------------------------------------------------------- full-size workloads, sampled


def _sample_tiles(B, H, T, n, seed):
    rng = np.random.default_rng(seed)
    picks = {(0, 0, 0), (B - 1, H - 1, T - 1), (0, H // 2, T // 2)}
    while len(picks) < n:
        picks.add((int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(T))))
    return sorted(picks)


def _full_size(name, steps, n_tiles, tau=None, first_step=0):
    """Run `steps` denoising steps of a workload from step `first_step` (fresh mask there)."""
    w = wl.WORKLOADS[name]
    tr = wl.Trajectory(w, device="cuda")
    for _ in range(first_step):
        tr.advance()
    B, N, H, d = w.B, w.N, w.H, w.d
    _, T, _ = la.lite_mask_geometry(N, d)
    m_in = la.new_mask(B, H, N, d)
    m_out = torch.empty_like(m_in)
    sparsity = []
    for t in range(first_step, first_step + steps):
        q, k, v = tr.current()
        ta = w.tau(t) if tau is None else tau
        o, lse = la.lite_attn_fwd(q, k, v, m_in, m_out, tau=ta)
        assert la.lite_get_device_status() == 0
        tiles = _sample_tiles(B, H, T, n_tiles, seed=t)
        ref = oracle_step(q, k, v, m_in, ta, query_tiles=tiles)
        rep = compare(o, lse, m_out, ref)
        assert_within(rep)
        bits = np.unpackbits(m_out.cpu().numpy().view(np.uint8), axis=-1, bitorder="little")[..., :T]
        sparsity.append(float(bits.mean()))
        print(f"{name} step {t} tau={ta:.2f} skip-mask density={sparsity[-1]:.4f} "
              f"flagged(sampled)={rep.flagged} near-tau mismatches={rep.mask_mismatches} "
              f"o_max={rep.o_max_abs:.2e} rel_rms={rep.o_rel_rms:.2e} lse={rep.lse_max_abs:.2e}")
        m_in, m_out = m_out, m_in
        tr.advance()
    assert all(b >= a for a, b in zip(sparsity, sparsity[1:]))  # monotone mask
    return sparsity


def test_480p_layer_sampled_early_steps():
    _full_size("480p", 2, 10)


def test_480p_layer_sampled_late_steps():
    """The last steps of the 480p schedule (tau near 0), where QK-Skip flags appear."""
    sp = _full_size("480p", 3, 12, first_step=7)
    assert sp[-1] > 0


def test_480p_d64_layer_sampled():
    """The 480p latent at d = 64: 512 mask rows stacked two to a kernel query tile, run by two
    CTAs per SM; sampled mask rows over three steps of its trajectory."""
    sp = _full_size("480p_d64", 3, 12)
    assert sp[-1] > 0


@pytest.mark.parametrize("d,F,gh,gw", [(64, 27, 133, 73), (128, 5, 47, 2231)])
def test_maximum_tile_count(d, F, gh, gw):
    """The largest layer the library accepts: 4096 query and key tiles (N = 262,143 at d=64 and
    524,285 at d=128, each with a ragged last tile, so list entries reach 4095), a random Skip-Mask
    and QK-Skip on; sampled query tiles, the last one included, against the oracle."""
    w = wl.small_workload(1, 1, F, gh, gw, d, steps=1, locality=3.0, tau=-3.0, seed_offset=4096 + d)
    q, k, v = wl.Trajectory(w, device="cuda").current()
    tile, T, _ = la.lite_mask_geometry(w.N, d)
    assert T == 4096 and w.N % tile != 0
    m_in = wl.random_mask(1, 1, T, 0.8, seed=d).cuda()
    m_out = torch.empty_like(m_in)
    o, lse = la.lite_attn_fwd(q, k, v, m_in, m_out, tau=-3.0)
    assert la.lite_get_device_status() == 0
    ref = oracle_step(q, k, v, m_in, -3.0, query_tiles=[(0, 0, 0), (0, 0, 2047), (0, 0, T - 1)])
    rep = compare(o, lse, m_out, ref)
    assert_within(rep)
    print(f"d={d} N={w.N} flagged(sampled)={rep.flagged} o_max={rep.o_max_abs:.2e} lse={rep.lse_max_abs:.2e}")


def test_720p_layer_sampled():
    _full_size("720p", 2, 8)


def test_stress_layer_sampled():
    _full_size("stress", 2, 8)


# ------------------------------------------------- full-size workloads at their operating point


def _mask_bits(mask, T):
    """[B, H, Tq, W] int32 Skip-Mask -> bool [B, H, Tq, T] (True = skipped)."""
    return np.unpackbits(mask.cpu().numpy().view(np.uint8), axis=-1, bitorder="little")[..., :T].astype(bool)


def _pairing_partner(live):
    """The partner of every query tile under the pairing the kernel picks for this mask: the stride
    s in [1, min(64, T/2)] whose pairs (tile r with r + s inside each block of 2s tiles, the tiles
    after the last full block as (t, t+1)) share the most live key tiles, the smaller on ties
    (include/lite_attn.h, LITE_OPT_PAIR_STRIDE). Returns partner[T] (-1: no partner)."""
    B, H, T, _ = live.shape
    X = live.astype(np.int64)

    def pairs(s):
        full = (T // (2 * s)) * (2 * s)
        idx = np.arange(full)
        a = idx[(idx % (2 * s)) < s]
        rest = np.arange(full, T - 1, 2)
        return np.concatenate([a, rest]), np.concatenate([a + s, rest + 1])

    best, best_s = -1, 1
    for s in range(1, max(1, min(64, T // 2)) + 1):
        a, b = pairs(s)
        sc = int((X[:, :, a] & X[:, :, b]).sum())
        if sc > best:
            best, best_s = sc, s
    a, b = pairs(best_s)
    partner = np.full(T, -1)
    partner[a], partner[b] = b, a
    return partner


def _lone_heavy_tiles(skipped, n, seed):
    """Query tiles whose pair partner (under the pairing the kernel picks) has a disjoint or empty
    live list, so that the kernel's union walk gives them many key tiles computed for one query
    tile only; the first and the ragged last tile of a head are always included."""
    B, H, T, _ = skipped.shape
    live = ~skipped
    partner = _pairing_partner(live)
    has_partner = partner >= 0
    pidx = np.where(has_partner, partner, 0)
    own = live.sum(-1)
    shared = np.where(has_partner, (live & live[:, :, pidx]).sum(-1), 0)
    lone = own - shared  # live tiles of this query tile that its partner skips
    rng = np.random.default_rng(seed)
    picks = {(0, 0, 0), (B - 1, H - 1, T - 1)}
    if (~has_partner).any():
        picks.add((0, int(rng.integers(H)), int(np.argmin(has_partner))))  # an unpaired tile
    order = np.argsort(-(lone + rng.random(lone.shape)), axis=None)  # most lone tiles first, ties random
    for flat in order[: 4 * n]:
        b, h, i = np.unravel_index(flat, lone.shape)
        picks.add((int(b), int(h), int(i)))
        if len(picks) >= n - 2:
            break
    empty_partner = np.argwhere((own > 0) & has_partner & (own[:, :, pidx] == 0))
    for b, h, i in empty_partner[:2]:
        picks.add((int(b), int(h), int(i)))
    while len(picks) < n:
        picks.add((int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(T))))
    frac_lone = float(lone.sum() / max(own.sum(), 1))
    return sorted(picks), frac_lone


def _operating_point(name, advance, n_compare, n_tiles, min_skipped):
    """Advance a workload's trajectory on the GPU alone for `advance` steps (its own tau schedule,
    the Skip-Mask growing step to step in the benchmark's launch configuration), then compare the
    next `n_compare` steps with the oracle, teacher-forced on the GPU's mask_in, on sampled query
    tiles biased to lone union tiles."""
    w = wl.WORKLOADS[name]
    tr = wl.Trajectory(w, device="cuda")
    B, N, H, d = w.B, w.N, w.H, w.d
    _, T, _ = la.lite_mask_geometry(N, d)
    m_in = la.new_mask(B, H, N, d)
    m_out = torch.empty_like(m_in)
    o = torch.empty((B, N, H, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    for t in range(advance):
        q, k, v = tr.current()
        la.lite_attn_fwd(q, k, v, m_in, m_out, tau=w.tau(t), o=o, lse=lse)
        m_in, m_out = m_out, m_in
        tr.advance()
    assert la.lite_get_device_status() == 0
    for t in range(advance, advance + n_compare):
        q, k, v = tr.current()
        skipped = _mask_bits(m_in, T)
        frac = float(skipped.mean())
        assert frac >= min_skipped, (name, t, frac)
        tiles, lone = _lone_heavy_tiles(skipped, n_tiles, seed=t)
        la.lite_attn_fwd(q, k, v, m_in, m_out, tau=w.tau(t), o=o, lse=lse)
        assert la.lite_get_device_status() == 0
        ref = oracle_step(q, k, v, m_in, w.tau(t), query_tiles=tiles)
        rep = compare(o, lse, m_out, ref)
        assert_within(rep)
        grown = _mask_bits(m_out, T)
        assert (grown | ~skipped).all()  # monotone: every skipped tile stays skipped
        print(f"{name} step {t}: skipped {frac:.3f}, lone share of live tiles {lone:.3f}, "
              f"flagged(sampled) {rep.flagged}, near-tau mismatches {rep.mask_mismatches}, "
              f"o_max {rep.o_max_abs:.2e} rel_rms {rep.o_rel_rms:.2e} lse {rep.lse_max_abs:.2e}")
        m_in, m_out = m_out, m_in
        tr.advance()


def test_720p_layer_after_ten_steps():
    """The 720p layer (tau -3) once half of its tiles are skipped."""
    _operating_point("720p", 10, 2, 16, 0.5)


def test_stress_layer_after_twelve_steps():
    """The stress layer (B=2, per-head locality U[2,8]) at >= 75% skipped, with its per-head spread."""
    _operating_point("stress", 12, 2, 20, 0.75)


def test_480p_layer_last_step_of_its_schedule():
    """Step 9, the last of the 480p schedule (tau 0)."""
    _operating_point("480p", 9, 1, 16, 0.3)


def test_two_empty_items_after_a_full_one():
    """One CTA, work items in their natural order: a pair of query tiles with live key tiles, then
    two pairs whose query tiles are fully skipped, then live pairs again. The producer must release
    the first pair's last PV before it hands out more items (a bundle with V only); without that
    the CTA stalls until the wait limit, which is lowered here so that a stall shows as
    LITE_ERR_TIMEOUT within half a second."""
    w = wl.small_workload(1, 2, 2, 8, 64, 128, steps=1, locality=3.0, tau=-2.0, seed_offset=71)  # N=1024, T=8
    q, k, v = wl.Trajectory(w, device="cuda").current()
    B, N, H, d = q.shape
    _, T, W = la.lite_mask_geometry(N, d)
    assert T == 8 and W == 1
    mask = la.new_mask(B, H, N, d)
    mask[:, :, 2:6, 0] = (1 << T) - 1  # query tiles 2..5 (pairs 1 and 2) skip every key tile
    m_out = torch.empty_like(mask)
    la.lite_set_option(la.LITE_OPT_MAX_CTAS, 1)
    la.lite_set_option(la.LITE_OPT_SCHEDULE, 0)
    la.lite_set_option(la.LITE_OPT_WAIT_LIMIT_NS, 500_000_000)
    try:
        o, lse = la.lite_attn_fwd(q, k, v, mask, m_out, tau=-2.0)
        assert la.lite_get_device_status() == 0
    finally:
        la.lite_set_option(la.LITE_OPT_SCHEDULE, 1)
    rep = compare(o, lse, m_out, oracle_step(q, k, v, mask, -2.0))
    assert_within(rep)
    assert torch.isneginf(lse[:, :, 2 * 128:6 * 128]).all()
