"""The C ABI library loads and exports what include/lite_attn.h declares; host-side argument checks.

CPU only. Every call here is rejected by argument validation before the library touches CUDA, so
none of them launches anything (the fake pointers are never dereferenced).
"""

import ctypes
import math
import os
import re

import pytest

from temporal_block_sparse_b200 import lite_attn as la

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "lite_attn.h")
FAKE = 1 << 20  # 16-byte aligned, never dereferenced


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(lite_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_abi():
    names = declared_functions()
    for expected in ("lite_attn_fwd", "lite_attn_dense", "lite_mask_to_list", "lite_mask_geometry",
                     "lite_get_device_status", "lite_status_string", "lite_schedule", "lite_attn_fwd_ex",
                     "lite_attn_dense_ex", "lite_lse_merge", "lite_dropped_mass", "lite_mask_to_ranges"):
        assert expected in names


def test_library_exports_every_declared_symbol():
    lib = la.load()
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
        assert n in la.SIGNATURES, f"binding lacks {n}"


def test_geometry():
    assert la.lite_mask_geometry(1024, 64) == (64, 16, 1)
    assert la.lite_mask_geometry(32760, 128) == (128, 256, 8)
    assert la.lite_mask_geometry(75600, 128) == (128, 591, 19)
    assert la.lite_mask_geometry(1, 128) == (128, 1, 1)
    lib = la.load()
    t = ctypes.c_int()
    assert lib.lite_mask_geometry(100, 96, ctypes.byref(t), None, None) == la.LITE_ERR_UNSUPPORTED
    assert lib.lite_mask_geometry(0, 64, None, None, None) == la.LITE_ERR_INVALID_ARG


def test_list_entry_checks_its_arguments():
    lib = la.load()
    args = lambda lst, cnt: (FAKE, FAKE, FAKE, FAKE, None, lst, cnt, None, 1, 1, 256, 128, 0.0, -3.0, None)
    assert lib.lite_attn_fwd_list(*args(None, FAKE)) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_fwd_list(*args(FAKE, None)) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_fwd_list(*args(FAKE + 1, FAKE)) == la.LITE_ERR_UNSUPPORTED
    assert lib.lite_attn_fwd_list(*args(FAKE, FAKE + 2)) == la.LITE_ERR_UNSUPPORTED


def test_scratch_pool_hook_refuses_null():
    assert la.load().lite_scratch_pool_bytes(None) == la.LITE_ERR_INVALID_ARG


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, 7):
        s = la.status_string(code)
        assert isinstance(s, str) and s


def _fwd(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, mi=None, mo=None, B=1, H=1, N=256, d=128, scale=0.0,
         tau=-3.0):
    return la.load().lite_attn_fwd(q, k, v, o, lse, mi, mo, B, H, N, d, scale, tau, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), la.LITE_ERR_INVALID_ARG),
    (dict(k=None), la.LITE_ERR_INVALID_ARG),
    (dict(v=None), la.LITE_ERR_INVALID_ARG),
    (dict(o=None), la.LITE_ERR_INVALID_ARG),
    (dict(B=0), la.LITE_ERR_INVALID_ARG),
    (dict(H=-1), la.LITE_ERR_INVALID_ARG),
    (dict(N=0), la.LITE_ERR_INVALID_ARG),
    (dict(d=96), la.LITE_ERR_UNSUPPORTED),
    (dict(d=256), la.LITE_ERR_UNSUPPORTED),
    (dict(q=FAKE + 8), la.LITE_ERR_UNSUPPORTED),
    (dict(o=FAKE + 2), la.LITE_ERR_UNSUPPORTED),
    (dict(lse=FAKE + 1), la.LITE_ERR_UNSUPPORTED),
    (dict(mi=FAKE + 2), la.LITE_ERR_UNSUPPORTED),
    (dict(N=4097 * 128), la.LITE_ERR_UNSUPPORTED),
    (dict(B=200, H=41), la.LITE_ERR_UNSUPPORTED),
    (dict(tau=float("nan")), la.LITE_ERR_INVALID_ARG),
])
def test_fwd_argument_errors(kw, code):
    assert _fwd(**kw) == code


def test_positive_tau_needs_debug_env(monkeypatch):
    monkeypatch.delenv("LITE_ATTN_DEBUG", raising=False)
    assert _fwd(tau=0.5) == la.LITE_ERR_INVALID_ARG
    assert _fwd(tau=0.5, q=None) == la.LITE_ERR_INVALID_ARG


def test_dense_argument_errors():
    lib = la.load()
    assert lib.lite_attn_dense(None, FAKE, FAKE, FAKE, None, 1, 1, 128, 128, 0.0, None) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_dense(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 128, 80, 0.0, None) == la.LITE_ERR_UNSUPPORTED
    assert lib.lite_attn_dense(FAKE, FAKE, FAKE, FAKE + 4, None, 1, 1, 128, 64, 0.0, None) == la.LITE_ERR_UNSUPPORTED


def test_list_and_schedule_argument_errors():
    lib = la.load()
    assert lib.lite_mask_to_list(None, None, FAKE, 1, 1, 128, 128, None) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_mask_to_list(None, FAKE, FAKE, 1, 1, 128, 32, None) == la.LITE_ERR_UNSUPPORTED
    assert lib.lite_schedule(None, FAKE, 1, 1, 4, None) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_schedule(FAKE, FAKE, 100, 100, 4, None) == la.LITE_ERR_UNSUPPORTED
    assert lib.lite_schedule(FAKE, FAKE, 1, 1, 5000, None) == la.LITE_ERR_UNSUPPORTED


def test_options():
    lib = la.load()
    assert lib.lite_set_option(99, 1) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_set_option(la.LITE_OPT_WAIT_LIMIT_NS, 10) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_set_option(la.LITE_OPT_DEBUG_STALL, 2) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_set_option(la.LITE_OPT_MAX_CTAS, -1) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_set_option(la.LITE_OPT_MAX_CTAS, 0) == la.LITE_OK
    assert lib.lite_set_kernel_events(FAKE, None) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_set_kernel_events(None, None) == la.LITE_OK


def test_binding_refuses_without_library(tmp_path):
    saved = la._lib
    try:
        la._lib = None
        with pytest.raises(RuntimeError):
            la.load(str(tmp_path / "missing.so"))
    finally:
        la._lib = saved


def _arr(vals):
    return (ctypes.c_int32 * max(1, len(vals)))(*vals) if vals else None


def _fwd_ex(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, mi=None, mo=None, do=None, skip=None, B=1, H=1, Nq=256,
            Nk=384, d=128, scale=0.0, tau=-3.0, n_do=None, n_skip=None):
    da, sa = _arr(do), _arr(skip)
    nd = len(do or []) if n_do is None else n_do
    ns = len(skip or []) if n_skip is None else n_skip
    return la.load().lite_attn_fwd_ex(q, k, v, o, lse, mi, mo, ctypes.cast(da, ctypes.c_void_p) if da else None, nd,
                                      ctypes.cast(sa, ctypes.c_void_p) if sa else None, ns, B, H, Nq, Nk, d, scale,
                                      tau, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), la.LITE_ERR_INVALID_ARG),
    (dict(Nq=0), la.LITE_ERR_INVALID_ARG),
    (dict(Nk=0), la.LITE_ERR_INVALID_ARG),
    (dict(Nk=4097 * 128), la.LITE_ERR_UNSUPPORTED),
    (dict(Nq=4097 * 128), la.LITE_ERR_UNSUPPORTED),
    (dict(d=32), la.LITE_ERR_UNSUPPORTED),
    (dict(tau=float("nan")), la.LITE_ERR_INVALID_ARG),
    # README range convention: strictly descending pairs, start inclusive, end exclusive
    (dict(do=[80, 60, 45]), la.LITE_ERR_INVALID_ARG),              # odd length
    (dict(do=[60, 80]), la.LITE_ERR_INVALID_ARG),                  # start below end
    (dict(do=[80, 60, 60, 40]), la.LITE_ERR_INVALID_ARG),          # end_0 == start_1
    (dict(do=[80, 60, 70, 40]), la.LITE_ERR_INVALID_ARG),          # overlapping, not descending
    (dict(skip=[80, 40, 10, -2]), la.LITE_ERR_INVALID_ARG),        # end below -1
    (dict(skip=[40, 40]), la.LITE_ERR_INVALID_ARG),                # empty pair
    (dict(do=None, n_do=2), la.LITE_ERR_INVALID_ARG),              # count without a list
    (dict(do=[80, 60], n_do=-2), la.LITE_ERR_INVALID_ARG),
])
def test_fwd_ex_argument_errors(kw, code):
    assert _fwd_ex(**kw) == code


def test_dense_ex_argument_errors():
    lib = la.load()
    assert lib.lite_attn_dense_ex(None, FAKE, FAKE, FAKE, None, 1, 1, 128, 64, 128, 0.0, None) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_dense_ex(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 128, 0, 128, 0.0, None) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_attn_dense_ex(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 128, 64, 48, 0.0, None) == la.LITE_ERR_UNSUPPORTED


def test_lse_merge_argument_errors():
    lib = la.load()
    P = ctypes.c_void_p

    def ptrs(*xs):
        return ctypes.cast((P * len(xs))(*xs), P)

    two = ptrs(FAKE, FAKE)
    assert lib.lite_lse_merge(None, two, 2, FAKE, None, 1, 1, 64, 128, None) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_lse_merge(two, two, 0, FAKE, None, 1, 1, 64, 128, None) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_lse_merge(ptrs(*[FAKE] * 9), ptrs(*[FAKE] * 9), 9, FAKE, None, 1, 1, 64, 128, None) == \
        la.LITE_ERR_UNSUPPORTED
    assert lib.lite_lse_merge(two, two, 2, None, None, 1, 1, 64, 128, None) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_lse_merge(two, ptrs(FAKE, None), 2, FAKE, None, 1, 1, 64, 128, None) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_lse_merge(ptrs(FAKE, FAKE + 8), two, 2, FAKE, None, 1, 1, 64, 128, None) == la.LITE_ERR_UNSUPPORTED
    assert lib.lite_lse_merge(two, ptrs(FAKE, FAKE + 2), 2, FAKE, None, 1, 1, 64, 128, None) == la.LITE_ERR_UNSUPPORTED
    assert lib.lite_lse_merge(two, two, 2, FAKE, None, 1, 1, 64, 96, None) == la.LITE_ERR_UNSUPPORTED
    assert lib.lite_lse_merge(two, two, 2, FAKE, None, 0, 1, 64, 128, None) == la.LITE_ERR_INVALID_ARG


def test_dropped_mass_argument_checks():
    lib = la.load()
    f = lib.lite_dropped_mass
    assert f(None, FAKE, None, FAKE, 1, 1, 8, None) == la.LITE_ERR_INVALID_ARG
    assert f(FAKE, FAKE, None, None, 1, 1, 8, None) == la.LITE_ERR_INVALID_ARG
    assert f(FAKE, FAKE, None, FAKE, 0, 1, 8, None) == la.LITE_ERR_INVALID_ARG
    assert f(FAKE, FAKE, None, FAKE, 1, 1, -3, None) == la.LITE_ERR_INVALID_ARG
    assert f(FAKE + 2, FAKE, None, FAKE, 1, 1, 8, None) == la.LITE_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE + 1, FAKE, 1, 1, 8, None) == la.LITE_ERR_UNSUPPORTED


def test_mask_to_ranges_argument_checks():
    f = la.load().lite_mask_to_ranges
    assert f(None, None, FAKE, 1, 1, 256, 128, None) == la.LITE_ERR_INVALID_ARG
    assert f(None, FAKE, None, 1, 1, 256, 128, None) == la.LITE_ERR_INVALID_ARG
    assert f(None, FAKE, FAKE, 0, 1, 256, 128, None) == la.LITE_ERR_INVALID_ARG
    assert f(None, FAKE, FAKE, 1, 1, 256, 96, None) == la.LITE_ERR_UNSUPPORTED
    assert f(None, FAKE + 1, FAKE, 1, 1, 256, 128, None) == la.LITE_ERR_UNSUPPORTED
    assert f(FAKE + 2, FAKE, FAKE, 1, 1, 256, 128, None) == la.LITE_ERR_UNSUPPORTED
    assert f(None, FAKE, FAKE, 1, 1, 4096 * 128 + 1, 128, None) == la.LITE_ERR_UNSUPPORTED


def test_cta_timing_and_schedule_option_checks():
    lib = la.load()
    assert lib.lite_set_cta_timing(None, 0) == la.LITE_OK
    assert lib.lite_set_cta_timing(None, 4) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_set_cta_timing(FAKE, 0) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_set_cta_timing(FAKE, -1) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_set_cta_timing(FAKE + 4, 8) == la.LITE_ERR_UNSUPPORTED
    assert lib.lite_set_option(la.LITE_OPT_SCHEDULE, 2) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_set_option(la.LITE_OPT_SCHEDULE, 0) == la.LITE_OK
    assert lib.lite_set_option(la.LITE_OPT_SCHEDULE, 1) == la.LITE_OK
    assert lib.lite_set_option(la.LITE_OPT_PAIR_STRIDE, -1) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_set_option(la.LITE_OPT_PAIR_STRIDE, 4097) == la.LITE_ERR_INVALID_ARG
    assert lib.lite_set_option(la.LITE_OPT_PAIR_STRIDE, 28) == la.LITE_OK
    assert lib.lite_set_option(la.LITE_OPT_PAIR_STRIDE, 0) == la.LITE_OK
