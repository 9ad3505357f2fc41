"""Python binding of the LiteAttention C ABI (include/lite_attn.h).

Argument marshalling only: every step of the forward pass runs in the CUDA library
`liblite_attn.so` built next to this file. There is no fallback -- if the library is missing or
cannot be loaded, every call raises.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblite_attn.so")

LITE_OK = 0
LITE_ERR_INVALID_ARG = -1
LITE_ERR_UNSUPPORTED = -2
LITE_ERR_CUDA = -3
LITE_ERR_TIMEOUT = -4
LITE_ERR_CHECK = -5
LITE_ERR_SCRATCH_LIMIT = -6
NOALLOC_SCRATCH_BYTES = 8 << 20

LITE_OPT_WAIT_LIMIT_NS = 1
LITE_OPT_DEBUG_STALL = 2
LITE_OPT_MAX_CTAS = 3

# every exported symbol and its (argtypes, restype)
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
SIGNATURES = {
    "lite_attn_fwd": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _F, _P], _I),
    "lite_attn_dense": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P], _I),
    "lite_mask_to_list": ([_P, _P, _P, _I, _I, _I, _I, _P], _I),
    "lite_schedule": ([_P, _P, _I, _I, _I, _P], _I),
    "lite_mask_geometry": ([_I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I)], _I),
    "lite_get_device_status": ([_P], _I),
    "lite_status_string": ([_I], ctypes.c_char_p),
    "lite_set_option": ([_I, ctypes.c_longlong], _I),
    "lite_set_kernel_events": ([_P, _P], _I),
    "lite_attn_fwd_noalloc": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _F, _P], _I),
    "lite_attn_fwd_ex": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _F, _F, _P], _I),
    "lite_attn_dense_ex": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P], _I),
    "lite_lse_merge": ([_P, _P, _I, _P, _P, _I, _I, _I, _I, _P], _I),
    "lite_dropped_mass": ([_P, _P, _P, _P, _I, _I, _I, _P], _I),
    "lite_mask_to_ranges": ([_P, _P, _P, _I, _I, _I, _I, _P], _I),
    "lite_set_cta_timing": ([_P, _I], _I),
    "lite_scratch_pool_bytes": ([ctypes.POINTER(ctypes.c_longlong)], _I),
    "lite_attn_fwd_list": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _F, _P], _I),
}
MAX_MERGE_PARTS = 8

_lib = None


class LiteAttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {status} ({status_string(status)})")


def load(path: str = LIB_PATH):
    """Load the CUDA library (once). Raises if it is absent: there is no CPU path."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library {path} is missing; build it with __graft_entry__.build()")
        lib = ctypes.CDLL(path)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().lite_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != LITE_OK:
        raise LiteAttnError(fn, status)


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def lite_mask_geometry(N: int, d: int) -> Tuple[int, int, int]:
    """(tile, T, W) for sequence length N and head dim d."""
    tile, T, W = _I(), _I(), _I()
    _check("lite_mask_geometry", load().lite_mask_geometry(int(N), int(d), ctypes.byref(tile), ctypes.byref(T),
                                                           ctypes.byref(W)))
    return tile.value, T.value, W.value


def _check_bf16(name, t):
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
        raise ValueError(f"{name} must be a contiguous 4-D bf16 CUDA tensor [B, N, H, d]")


def _check_qkv(q, k, v):
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_bf16(name, t)
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must have the same shape [B, N, H, d]")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k, v must be on one device")


def _check_qkv_cross(q, k, v):
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_bf16(name, t)
    if k.shape != v.shape or q.shape[0] != k.shape[0] or q.shape[2:] != k.shape[2:]:
        raise ValueError("q [B, Nq, H, d] and k, v [B, Nk, H, d] must agree in B, H and d")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k, v must be on one device")


def _ranges(r, name):
    """README-style range list -> (ctypes int32 array or None, length)."""
    if r is None or len(r) == 0:
        return None, 0
    vals = [int(x) for x in r]
    return (ctypes.c_int32 * len(vals))(*vals), len(vals)


def new_mask(B: int, H: int, N: int, d: int, device=None, Nk: Optional[int] = None) -> torch.Tensor:
    """A fresh (all-live) Skip-Mask, int32 [B, H, Tq, Wk] holding uint32 bit patterns (Nk defaults to N)."""
    _, T, _ = lite_mask_geometry(N, d)
    _, _, W = lite_mask_geometry(N if Nk is None else Nk, d)
    return torch.zeros((B, H, T, W), dtype=torch.int32, device=device or "cuda")


def lite_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, mask_in: Optional[torch.Tensor] = None,
                  mask_out: Optional[torch.Tensor] = None, scale: Optional[float] = None, tau: float = -10.0,
                  o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, return_lse: bool = True,
                  stream=None):
    """One LiteAttention forward (see include/lite_attn.h). Returns (o, lse or None)."""
    _check_qkv(q, k, v)
    B, N, H, d = q.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check_fwd_buffers(q, k, o, lse, mask_in, mask_out)
    st = load().lite_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), _ptr(lse), _ptr(mask_in),
                              _ptr(mask_out), B, H, N, d, float(scale or 0.0), float(tau), _stream_handle(stream))
    _check("lite_attn_fwd", st)
    return o, lse


def lite_attn_dense(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: Optional[float] = None,
                    o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, return_lse: bool = True,
                    stream=None):
    """No-skip forward through the same kernel. Returns (o, lse or None)."""
    _check_qkv(q, k, v)
    B, N, H, d = q.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check_outputs(q, o, lse)
    st = load().lite_attn_dense(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), _ptr(lse), B, H, N, d,
                                float(scale or 0.0), _stream_handle(stream))
    _check("lite_attn_dense", st)
    return o, lse


def lite_mask_to_list(mask: Optional[torch.Tensor], B: int, H: int, N: int, d: int, stream=None):
    """Skip-Mask -> (list int16 [B,H,T,T], counts int32 [B,H,T]); list entries past counts are -1."""
    _, T, W = lite_mask_geometry(N, d)
    dev = mask.device if mask is not None else torch.device("cuda")
    lst = torch.full((B, H, T, T), -1, dtype=torch.int16, device=dev)
    counts = torch.empty((B, H, T), dtype=torch.int32, device=dev)
    st = load().lite_mask_to_list(_ptr(mask), lst.data_ptr(), counts.data_ptr(), B, H, N, d, _stream_handle(stream))
    _check("lite_mask_to_list", st)
    return lst, counts


def lite_schedule(counts: torch.Tensor, stream=None) -> torch.Tensor:
    """Work order int32 [B*H*T] from live counts [B, H, T]."""
    if counts.dtype != torch.int32 or not counts.is_contiguous() or counts.dim() != 3:
        raise ValueError("counts must be contiguous int32 [B, H, T]")
    B, H, T = counts.shape
    order = torch.empty(B * H * T, dtype=torch.int32, device=counts.device)
    _check("lite_schedule", load().lite_schedule(counts.data_ptr(), order.data_ptr(), B, H, T, _stream_handle(stream)))
    return order


def lite_get_device_status(stream=None) -> int:
    """Synchronise and read/clear the device status word (0 = ok)."""
    return load().lite_get_device_status(_stream_handle(stream))


def lite_set_option(option: int, value: int):
    _check("lite_set_option", load().lite_set_option(int(option), int(value)))


def lite_set_kernel_events(before: Optional[torch.cuda.Event], after: Optional[torch.cuda.Event]):
    """Record `before`/`after` around the attention kernel of later calls (None, None to stop)."""
    b = before.cuda_event if before is not None else None
    a = after.cuda_event if after is not None else None
    _check("lite_set_kernel_events", load().lite_set_kernel_events(b, a))


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def lite_attn_fwd_list(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, lst: torch.Tensor, counts: torch.Tensor,
                       mask_out: Optional[torch.Tensor] = None, scale: Optional[float] = None, tau: float = -10.0,
                       o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, return_lse: bool = True,
                       stream=None):
    """Forward pass over caller-supplied Skip-Lists (int16 [B, H, T, T] live key tiles, descending,
    with int32 [B, H, T] counts, as lite_mask_to_list returns them); flags are OR-ed into mask_out
    (see include/lite_attn.h). The list buffer may be larger than [B, H, T, T]: only its first
    B*H*T*T entries are addressed. Returns (o, lse or None)."""
    _check_qkv(q, k, v)
    B, N, H, d = q.shape
    _, T, _ = lite_mask_geometry(N, d)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _check_fwd_buffers(q, k, o, lse, None, mask_out)
    if (lst.dtype != torch.int16 or not lst.is_contiguous() or not lst.is_cuda or lst.device != q.device
            or lst.numel() < B * H * T * T):
        raise ValueError("lst must be a contiguous int16 CUDA tensor of at least B*H*T*T entries on q's device")
    if (counts.dtype != torch.int32 or not counts.is_contiguous() or not counts.is_cuda or counts.device != q.device
            or tuple(counts.shape) != (B, H, T)):
        raise ValueError("counts must be a contiguous int32 CUDA tensor [B, H, T] on q's device")
    st = load().lite_attn_fwd_list(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), _ptr(lse), lst.data_ptr(),
                                   counts.data_ptr(), _ptr(mask_out), B, H, N, d, float(scale or 0.0), float(tau),
                                   _stream_handle(stream))
    _check("lite_attn_fwd_list", st)
    return o, lse


def lite_attn_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                          lse: Optional[torch.Tensor] = None, mask_in: Optional[torch.Tensor] = None,
                          mask_out: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                          tau: float = -10.0, stream=None):
    """lite_attn_fwd for callers that must not allocate device memory (see include/lite_attn.h).

    The library allocates nothing here: the caller passes every output buffer, and the per-call
    scratch sits in the library's fixed 8 MiB device array (layers needing more are refused with
    LITE_ERR_SCRATCH_LIMIT). Calls that overlap on the GPU race on that array.
    """
    _check_qkv(q, k, v)
    B, N, H, d = q.shape
    _check_fwd_buffers(q, k, o, lse, mask_in, mask_out)
    st = load().lite_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), _ptr(lse),
                                      _ptr(mask_in), _ptr(mask_out), B, H, N, d, float(scale or 0.0), float(tau),
                                      _stream_handle(stream))
    _check("lite_attn_fwd_noalloc", st)
    return o, lse


def _check_masks(*masks, shape=None, device=None):
    """Skip-Masks: contiguous int32 CUDA tensors, of `shape` [B, H, Tq, Wk] and on `device` when given."""
    for m in masks:
        if m is None:
            continue
        if m.dtype != torch.int32 or not m.is_contiguous() or not m.is_cuda:
            raise ValueError("masks must be contiguous int32 CUDA tensors [B, H, Tq, Wk]")
        if shape is not None and tuple(m.shape) != tuple(shape):
            raise ValueError(f"mask shape {tuple(m.shape)} != [B, H, Tq, Wk] = {tuple(shape)}")
        if device is not None and m.device != device:
            raise ValueError("masks must be on the device of q")


def _check_outputs(q: torch.Tensor, o: torch.Tensor, lse: Optional[torch.Tensor]):
    """o: contiguous bf16 shaped like q [B, Nq, H, d]; lse: contiguous fp32 [B, H, Nq]; both on q's device."""
    _check_bf16("o", o)
    if o.shape != q.shape or o.device != q.device:
        raise ValueError("o must have q's shape [B, Nq, H, d] and device")
    if lse is not None:
        B, Nq, H, _ = q.shape
        if (lse.dtype != torch.float32 or not lse.is_contiguous() or not lse.is_cuda or lse.device != q.device
                or tuple(lse.shape) != (B, H, Nq)):
            raise ValueError("lse must be a contiguous fp32 CUDA tensor [B, H, Nq] on q's device")


def _check_fwd_buffers(q, k, o, lse, mask_in, mask_out):
    """Every device buffer of a masked forward call, checked before the C call (the library cannot
    tell a host pointer or a short buffer from a good one)."""
    B, Nq, H, d = q.shape
    _, Tq, _ = lite_mask_geometry(Nq, d)
    _, _, Wk = lite_mask_geometry(k.shape[1], d)
    _check_outputs(q, o, lse)
    _check_masks(mask_in, mask_out, shape=(B, H, Tq, Wk), device=q.device)


def scratch_pool_bytes() -> int:
    """Device memory held by the library's scratch pool on the current device (0 before any pooled call)."""
    v = ctypes.c_longlong(0)
    _check("lite_scratch_pool_bytes", load().lite_scratch_pool_bytes(ctypes.byref(v)))
    return int(v.value)


def lite_attn_fwd_ex(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, mask_in: Optional[torch.Tensor] = None,
                     mask_out: Optional[torch.Tensor] = None, must_do=None, must_skip=None,
                     scale: Optional[float] = None, tau: float = -10.0, o: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, return_lse: bool = True, stream=None):
    """Partial attention: q [B, Nq, H, d] against k, v [B, Nk, H, d], with README-style must-do /
    must-skip key-token range lists (see include/lite_attn.h). Returns (o, lse or None)."""
    _check_qkv_cross(q, k, v)
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    if o is None:
        o = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check_fwd_buffers(q, k, o, lse, mask_in, mask_out)
    do_arr, n_do = _ranges(must_do, "must_do")
    skip_arr, n_skip = _ranges(must_skip, "must_skip")
    st = load().lite_attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), _ptr(lse), _ptr(mask_in),
                                 _ptr(mask_out), ctypes.cast(do_arr, _P) if do_arr is not None else None, n_do,
                                 ctypes.cast(skip_arr, _P) if skip_arr is not None else None, n_skip, B, H, Nq, Nk, d,
                                 float(scale or 0.0), float(tau), _stream_handle(stream))
    _check("lite_attn_fwd_ex", st)
    return o, lse


def lite_attn_dense_ex(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: Optional[float] = None,
                       o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, return_lse: bool = True,
                       stream=None):
    """No-skip partial attention, q [B, Nq, H, d] against k, v [B, Nk, H, d]. Returns (o, lse or None)."""
    _check_qkv_cross(q, k, v)
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    if o is None:
        o = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    _check_outputs(q, o, lse)
    st = load().lite_attn_dense_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), _ptr(lse), B, H, Nq, Nk,
                                   d, float(scale or 0.0), _stream_handle(stream))
    _check("lite_attn_dense_ex", st)
    return o, lse


def lite_lse_merge(parts, o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   return_lse: bool = True, stream=None):
    """Combine partial attentions [(o_p [B, N, H, d] bf16, lse_p [B, H, N] fp32), ...] over disjoint
    key sets into (o, lse). o / lse may be one of the parts' tensors (in place)."""
    parts = list(parts)
    if not 1 <= len(parts) <= MAX_MERGE_PARTS:
        raise ValueError(f"1 to {MAX_MERGE_PARTS} parts")
    o0 = parts[0][0]
    B, N, H, d = o0.shape
    for op, lp in parts:
        _check_bf16("o_p", op)
        if op.shape != o0.shape:
            raise ValueError("all partial outputs must have one shape [B, N, H, d]")
        if lp.dtype != torch.float32 or not lp.is_contiguous() or tuple(lp.shape) != (B, H, N):
            raise ValueError("lse_p must be contiguous fp32 [B, H, N]")
    if o is None:
        o = torch.empty_like(o0)
    if lse is None and return_lse:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=o0.device)
    outs = (_P * len(parts))(*[op.data_ptr() for op, _ in parts])
    lses = (_P * len(parts))(*[lp.data_ptr() for _, lp in parts])
    st = load().lite_lse_merge(ctypes.cast(outs, _P), ctypes.cast(lses, _P), len(parts), o.data_ptr(), _ptr(lse),
                               B, H, N, d, _stream_handle(stream))
    _check("lite_lse_merge", st)
    return o, lse


def lite_dropped_mass(lse_live: torch.Tensor, lse_full: torch.Tensor, row_mass: Optional[torch.Tensor] = None,
                      stats: Optional[torch.Tensor] = None, stream=None):
    """Per-row softmax mass a Skip-Mask drops, 1 - exp(lse_live - lse_full), for lse tensors
    [B, H, N] fp32 on the GPU. Returns (row_mass or None, stats) with stats a device fp32 [2] tensor
    {largest per-row value, sum over rows}; reading it synchronises."""
    for name, t in (("lse_live", lse_live), ("lse_full", lse_full)):
        if t.dtype != torch.float32 or not t.is_contiguous() or t.dim() != 3:
            raise ValueError(f"{name} must be a contiguous fp32 [B, H, N] tensor")
    if lse_live.shape != lse_full.shape:
        raise ValueError("lse_live and lse_full differ in shape")
    B, H, N = lse_live.shape
    if row_mass is not None and (row_mass.shape != lse_live.shape or row_mass.dtype != torch.float32):
        raise ValueError("row_mass must match the lse tensors")
    if stats is None:
        stats = torch.empty(2, dtype=torch.float32, device=lse_live.device)
    st = load().lite_dropped_mass(lse_live.data_ptr(), lse_full.data_ptr(), _ptr(row_mass), stats.data_ptr(), B, H,
                                  N, _stream_handle(stream))
    _check("lite_dropped_mass", st)
    return row_mass, stats


def lite_mask_to_ranges(mask: Optional[torch.Tensor], B: int, H: int, N: int, d: int, device=None, stream=None):
    """Range-encoded Skip-List of a mask: (ranges int16 [B, H, T, T+1], nruns int32 [B, H, T]); row r
    holds nruns[r] (start, end) pairs of live key-tile runs, highest first (end exclusive)."""
    _, T, _ = lite_mask_geometry(N, d)
    dev = mask.device if mask is not None else (device or "cuda")
    if mask is not None:
        _check_masks(mask)
    ranges = torch.empty((B, H, T, T + 1), dtype=torch.int16, device=dev)
    nruns = torch.empty((B, H, T), dtype=torch.int32, device=dev)
    st = load().lite_mask_to_ranges(_ptr(mask), ranges.data_ptr(), nruns.data_ptr(), B, H, N, d, _stream_handle(stream))
    _check("lite_mask_to_ranges", st)
    return ranges, nruns


LITE_OPT_SCHEDULE = 4
LITE_OPT_PAIR_STRIDE = 5


def lite_set_cta_timing(buf: Optional[torch.Tensor]):
    """Per-CTA {start ns, end ns, tiles} records of every following attention launch go to buf
    (int64 [capacity, 3] on the GPU); None stops recording."""
    if buf is None:
        _check("lite_set_cta_timing", load().lite_set_cta_timing(None, 0))
        return
    if buf.dtype != torch.int64 or buf.dim() != 2 or buf.shape[1] != 3 or not buf.is_contiguous():
        raise ValueError("buf must be a contiguous int64 [capacity, 3] tensor")
    _check("lite_set_cta_timing", load().lite_set_cta_timing(buf.data_ptr(), buf.shape[0]))
