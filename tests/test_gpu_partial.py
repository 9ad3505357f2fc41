"""Partial attention on the GPU vs the CPU oracle, through the C ABI (needs a B200).

Covers cross attention (Nq != Nk, ragged tails on both sides), must-do / must-skip key ranges
(README, must_do_list / must_skip_list), the LSE merge kernel, and the README's text/video
composition (t2t, t2v, v2t without skipping, v2v with skipping, merged by LSE).
"""

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
    assert la.lite_get_device_status() == 0


def _tokens(B, H, N, d, seed, locality=2.0):
    """q, k, v [B, N, H, d] bf16 on the GPU from the seeded video-token generator (N = F * gh * gw)."""
    gw = 16 if d == 128 else 8
    F = -(-N // (8 * gw))
    w = wl.small_workload(B, H, F, 8, gw, d, locality=locality, seed_offset=seed)
    q, k, v = wl.Trajectory(w, device="cuda").current()
    return q[:, :N].contiguous(), k[:, :N].contiguous(), v[:, :N].contiguous()


def _cross(B, H, Nq, Nk, d, seed):
    """Queries from the first Nq tokens, keys / values from the last Nk tokens of one clip."""
    q, k, v = _tokens(B, H, Nq + Nk, d, seed)
    return q[:, :Nq].contiguous(), k[:, Nq:].contiguous(), v[:, Nq:].contiguous()


def _oracle(q, k, v, mask_in=None, tau=-np.inf, must_do=None, must_skip=None, skip_test=True):
    mi = None if mask_in is None else mask_in.cpu().numpy().view(np.uint32)
    return oracle.lite_attention_forward(to_np(q), to_np(k), to_np(v), mi, tau=tau, must_do=must_do,
                                         must_skip=must_skip, skip_test=skip_test)


def _mask(B, H, Nq, Nk, d, density, seed):
    _, Tq, _ = la.lite_mask_geometry(Nq, d)
    _, Tk, _ = la.lite_mask_geometry(Nk, d)
    return wl.random_mask(B, H, Tq, density, seed=seed, Tk=Tk).cuda()


# ------------------------------------------------------------------------------ cross attention


@pytest.mark.parametrize("B,H,Nq,Nk,d", [
    (1, 2, 200, 1000, 64), (2, 1, 300, 77, 128), (1, 3, 1000, 4100, 128), (1, 1, 193, 64, 64),
    (1, 2, 128, 1, 128)])
def test_cross_dense_matches_oracle(B, H, Nq, Nk, d):
    q, k, v = _cross(B, H, Nq, Nk, d, seed=Nq + Nk)
    o, lse = la.lite_attn_dense_ex(q, k, v)
    assert la.lite_get_device_status() == 0
    assert_within(compare(o, lse, None, _oracle(q, k, v), check_mask=False))


@pytest.mark.parametrize("B,H,Nq,Nk,d,density,tau", [
    (1, 2, 500, 1300, 64, 0.3, -3.0), (2, 2, 700, 260, 128, 0.2, -1.0), (1, 4, 2000, 3000, 128, 0.5, 0.0)])
def test_cross_masked_matches_oracle(B, H, Nq, Nk, d, density, tau):
    q, k, v = _cross(B, H, Nq, Nk, d, seed=3 * Nq + Nk)
    m_in = _mask(B, H, Nq, Nk, d, density, seed=Nq)
    m_out = torch.full_like(m_in, 0x5A5A5A5A)
    o, lse = la.lite_attn_fwd_ex(q, k, v, m_in, m_out, tau=tau)
    assert la.lite_get_device_status() == 0
    rep = compare(o, lse, m_out, _oracle(q, k, v, m_in, tau))
    assert_within(rep)
    assert rep.mask_mismatches <= max(2, rep.flagged // 100)


# ------------------------------------------------------------------------------ key-token ranges


RANGE_CASES = [
    # (Nq, Nk, d, must_do, must_skip): README convention, start inclusive, end exclusive, descending
    (1000, 1000, 64, [900, 700, 450, 440, 12, 2], [999, 620, 300, 100]),
    (640, 1000, 64, [], [999, 640, 511, 255]),
    (700, 1500, 128, [1499, 1400, 3, -1], [1300, -1]),
    (300, 2000, 128, [2500, 1900, 1024, 1000], [1999, 1023]),
]


@pytest.mark.parametrize("Nq,Nk,d,must_do,must_skip", RANGE_CASES)
@pytest.mark.parametrize("tau", [-np.inf, -2.0])
def test_ranges_match_oracle(Nq, Nk, d, must_do, must_skip, tau):
    B, H = 1, 3
    q, k, v = _cross(B, H, Nq, Nk, d, seed=Nk + len(must_do))
    m_in = _mask(B, H, Nq, Nk, d, 0.25, seed=Nk)
    m_out = torch.full_like(m_in, 0x5A5A5A5A)
    o, lse = la.lite_attn_fwd_ex(q, k, v, m_in, m_out, must_do=must_do, must_skip=must_skip, tau=tau)
    assert la.lite_get_device_status() == 0
    ref = _oracle(q, k, v, m_in, tau, must_do=must_do, must_skip=must_skip)
    rep = compare(o, lse, m_out, ref)
    assert_within(rep)
    # must-do tiles are never flagged: their mask_out bits are mask_in's
    t = la.lite_mask_geometry(Nk, d)[0]
    forced = oracle.range_tiles(must_do, Nk, t, whole=False)
    got, before = m_out.cpu().numpy().view(np.uint32), m_in.cpu().numpy().view(np.uint32)
    for j in forced:
        bit = np.uint32(1 << (j & 31))
        np.testing.assert_array_equal(got[..., j >> 5] & bit, before[..., j >> 5] & bit)


def test_ranges_on_the_readme_example():
    """The README's length-100 example; tile 64 here (d = 64): tokens 41..80 span tiles 0 and 1,
    neither wholly, so must-skip removes nothing; must-do keeps both live."""
    q, k, v = _cross(1, 1, 100, 100, 64, seed=7)
    m_in = _mask(1, 1, 100, 100, 64, 1.0, seed=1)  # everything masked
    o, lse = la.lite_attn_fwd_ex(q, k, v, m_in, None, must_do=[80, 60, 45, 40, 12, 2], must_skip=[80, 40],
                                 tau=-np.inf)
    ref = _oracle(q, k, v, m_in, must_do=[80, 60, 45, 40, 12, 2], must_skip=[80, 40])
    assert_within(compare(o, lse, None, ref, check_mask=False))


def test_must_skip_everything_gives_empty_rows():
    q, k, v = _cross(1, 2, 300, 500, 128, seed=11)
    o, lse = la.lite_attn_fwd_ex(q, k, v, None, None, must_skip=[499, -1], tau=-np.inf)
    assert la.lite_get_device_status() == 0
    assert (o == 0).all() and torch.isneginf(lse).all()


# ------------------------------------------------------------------------------------ LSE merge


def _parts(P, B, H, N, d, seed, neg_inf_rows=True):
    g = torch.Generator().manual_seed(seed)
    parts = []
    for p in range(P):
        o = torch.randn((B, N, H, d), generator=g).to(torch.bfloat16)
        lse = torch.randn((B, H, N), generator=g) * 3.0 + 5.0
        if neg_inf_rows:
            lse[torch.rand((B, H, N), generator=g) < 0.15] = -np.inf  # rows without keys in this part
            lse[:, :, :3] = -np.inf  # rows with no key in any part
        parts.append((o.cuda(), lse.cuda()))
    return parts


def _merge_ref(parts):
    return oracle.lse_merge([(to_np(o), lse.cpu().numpy().astype(np.float64)) for o, lse in parts])


def _merge_check(o, lse, ref):
    ro, rl = ref
    got = to_np(o)
    err = np.abs(got - ro)
    # fp32 arithmetic, then one bf16 rounding of the result (relative 2^-9)
    assert (err <= 2.0 ** -8 * np.abs(ro) + 1e-3).all(), float(err.max())
    gl = lse.cpu().numpy()
    inf = np.isneginf(rl)
    assert (np.isneginf(gl) == inf).all()
    np.testing.assert_allclose(gl[~inf], rl[~inf], rtol=1e-6, atol=1e-5)
    assert (got[np.broadcast_to(np.isneginf(rl).transpose(0, 2, 1)[..., None], got.shape)] == 0).all()


@pytest.mark.parametrize("P,B,H,N,d", [(1, 1, 2, 100, 64), (2, 2, 3, 777, 128), (3, 1, 4, 1000, 64),
                                       (5, 1, 2, 513, 128), (8, 2, 2, 300, 128)])
def test_lse_merge_matches_oracle(P, B, H, N, d):
    parts = _parts(P, B, H, N, d, seed=P * N)
    o, lse = la.lite_lse_merge(parts)
    assert la.lite_get_device_status() == 0
    _merge_check(o, lse, _merge_ref(parts))


def test_lse_merge_in_place():
    parts = _parts(2, 1, 3, 1000, 128, seed=5)
    ref = _merge_ref(parts)
    o, lse = la.lite_lse_merge(parts, o=parts[0][0], lse=parts[0][1])
    assert o.data_ptr() == parts[0][0].data_ptr()
    _merge_check(o, lse, ref)


def test_lse_merge_of_key_splits_equals_full_attention():
    """Split the keys at non-tile boundaries, attend to each split, merge: the full attention."""
    B, H, N, d = 1, 2, 1500, 128
    q, k, v = _tokens(B, H, N, d, seed=21)
    cuts = [0, 333, 900, N]
    parts = [la.lite_attn_dense_ex(q, k[:, a:e].contiguous(), v[:, a:e].contiguous()) for a, e in zip(cuts, cuts[1:])]
    o, lse = la.lite_lse_merge(parts)
    assert_within(compare(o, lse, None, _oracle(q, k, v), check_mask=False))


# ------------------------------------------------------------------ README text / video composition


@pytest.mark.parametrize("tau", [-np.inf, -3.0])
def test_text_video_composition(tau):
    B, H, d, text, video = 1, 2, 128, 300, 2000
    q, k, v = _tokens(B, H, text + video, d, seed=31)
    sl = lambda x, a, b: x[:, a:b].contiguous()
    qt, qv, kt, kv, vt, vv = sl(q, 0, text), sl(q, text, None), sl(k, 0, text), sl(k, text, None), \
        sl(v, 0, text), sl(v, text, None)
    m_in = _mask(B, H, video, video, d, 0.3, seed=2)
    m_out = torch.zeros_like(m_in)
    t2t = la.lite_attn_dense_ex(qt, kt, vt)
    t2v = la.lite_attn_dense_ex(qt, kv, vv)
    v2t = la.lite_attn_dense_ex(qv, kt, vt)
    v2v = la.lite_attn_fwd_ex(qv, kv, vv, m_in, m_out, tau=tau)
    o_text, l_text = la.lite_lse_merge([t2t, t2v])
    o_video, l_video = la.lite_lse_merge([v2t, v2v])
    assert la.lite_get_device_status() == 0

    r_v2v = _oracle(qv, kv, vv, m_in, tau)
    rep = compare(v2v[0], v2v[1], m_out, r_v2v)
    assert_within(rep)
    r_t = oracle.lse_merge([(r.out, r.lse) for r in (_oracle(qt, kt, vt), _oracle(qt, kv, vv))])
    r_v = oracle.lse_merge([(r.out, r.lse) for r in (_oracle(qv, kt, vt), r_v2v)])
    for (o, l), (ro, rl) in (((o_text, l_text), r_t), ((o_video, l_video), r_v)):
        ref = oracle.ForwardResult(ro, rl, None, {})
        assert_within(compare(o, l, None, ref, check_mask=False))
