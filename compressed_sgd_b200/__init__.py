"""compressed_sgd_b200 — residual gradient sparsification on NVIDIA B200.

Thin ctypes binding of ``libgsparse.so`` (C ABI declared in ``include/gsparse.h``). Each function
below marshals torch tensors into device pointers, sizes and the current CUDA stream, and calls the
entry point of the same name; every step of the computation runs in the library's CUDA kernels.
There is no CPU path: if the library is missing, ``lib()`` raises.

Tensors must be CUDA tensors, contiguous, of the dtype stated. Outputs that are not supplied are
allocated here with torch; scratch memory ("workspace") likewise.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libgsparse.so")

GSPARSE_SELECT_EXHAUSTIVE = 1
GSPARSE_BINARIZE_BY_MAGNITUDE = 2
GSPARSE_SELECT_TEST_EXPIRE_WAIT = 4
DERR_CAPACITY, DERR_CORRUPT_STREAM, DERR_INDEX_RANGE, DERR_SEGMENTS, DERR_TIMEOUT = 1, 2, 4, 8, 16
MAX_WORKERS = 64

_i64, _i32, _u32, _vp, _f32, _f64, _sz = (ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_void_p,
                                          ctypes.c_float, ctypes.c_double, ctypes.c_size_t)


class GsparseError(RuntimeError):
    pass


class GsparsePending(ctypes.Structure):
    _fields_ = [("idx", _vp), ("val", _vp), ("d_count", _vp), ("capacity", _i64)]


class GsparseList(ctypes.Structure):
    _fields_ = [("idx", _vp), ("val", _vp), ("uniform_val", _vp), ("d_count", _vp), ("capacity", _i64)]


class GsparsePassEvents(ctypes.Structure):
    _fields_ = [("before", _vp), ("after", _vp)]


# name -> (restype, argtypes)
_SIGNATURES = {
    "gsparse_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "gsparse_version": (ctypes.c_char_p, []),
    "gsparse_k_for": (_i64, [_i64, _i64, _i64]),
    "gsparse_golomb_b_star": (_i32, [_f64]),
    "gsparse_golomb_chunk_hint": (_i32, [_i64]),
    "gsparse_warmup_keep_num": (_i64, [_i64, _i64, _f64, _f64, _i64]),
    "gsparse_residual_topk_workspace_size": (_sz, [_i64, _i32, _i64, _i64]),
    "gsparse_residual_topk_workspace_min": (_sz, [_i64, _i32]),
    "gsparse_residual_topk": (ctypes.c_int, [_vp, _vp, _i64, _vp, _i32, _i64, _i64, _vp, _vp, _vp, _i64,
                                             ctypes.POINTER(GsparsePending), _u32, _vp, _sz, _vp, _vp,
                                             ctypes.POINTER(GsparsePassEvents)]),
    "gsparse_residual_topk_momentum": (ctypes.c_int, [_vp, _vp, ctypes.c_float, _vp, _i64, _vp, _i32, _i64, _i64,
                                                      _vp, _vp, _vp, _i64, ctypes.POINTER(GsparsePending), _u32,
                                                      _vp, _sz, _vp, _vp, ctypes.POINTER(GsparsePassEvents)]),
    "gsparse_residual_topk_noalloc": (ctypes.c_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _vp]),
    "gsparse_quantize_workspace_size": (_sz, [_i64]),
    "gsparse_quantize": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _vp, _i64, _vp, _vp, _vp, _i32, _vp, _sz, _vp,
                                        _vp]),
    "gsparse_quantize_segments_workspace_size": (_sz, [_i64, _i32]),
    "gsparse_quantize_segments": (ctypes.c_int, [_vp, _vp, _vp, _i32, _i64, _vp, _i64, _vp, _vp, _vp, _i32, _vp, _sz,
                                                 _vp, _vp]),
    "gsparse_binarize_workspace_size": (_sz, [_i64, _i32, _i64, _i64]),
    "gsparse_binarize_workspace_min": (_sz, [_i64, _i32, _i64, _i64]),
    "gsparse_binarize": (ctypes.c_int, [_vp, _vp, _i64, _vp, _i32, _i64, _i64, _vp, _vp, _vp, _vp, _i64, _u32,
                                        _vp, _sz, _vp, _vp, ctypes.POINTER(GsparsePassEvents)]),
    "gsparse_golomb_encode_workspace_size": (_sz, [_i64]),
    "gsparse_golomb_encode": (ctypes.c_int, [_vp, _vp, _vp, _i64, _i64, _i32, _vp, _i64, _vp, _vp, _i32, _vp,
                                             _sz, _vp, _vp]),
    "gsparse_golomb_decode": (ctypes.c_int, [_vp, _i64, _vp, _vp, _i64, _i64, _i32, _vp, _i32, _i64, _vp, _vp,
                                             _vp]),
    "gsparse_scatter_accumulate_workspace_size": (_sz, [_i32, _i64]),
    "gsparse_scatter_accumulate": (ctypes.c_int, [ctypes.POINTER(GsparseList), _i32, _i64, _vp, _vp, _vp, _vp,
                                                  _i64, _vp, _sz, _vp, _vp]),
    "gsparse_accumulate_combine_workspace_size": (_sz, [_i32, _i64]),
    "gsparse_accumulate_combine": (ctypes.c_int, [ctypes.POINTER(GsparseList), _i32, _i64, _vp, _vp, _f32, _f32,
                                                  _i32, _i32, _vp, _vp, _sz, _vp, _vp]),
    "gsparse_combine_local": (ctypes.c_int, [_vp, _vp, _vp, _i64, _f32, _f32, _i32, _vp, _vp, _vp, _i64, _vp,
                                             _vp]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libgsparse.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise GsparseError(f"{LIB_PATH} not found: build it with `python -m compressed_sgd_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def exported_symbols() -> List[str]:
    return list(_SIGNATURES)


def _check(status: int, what: str):
    if status != 0:
        raise GsparseError(f"{what}: {lib().gsparse_status_string(status).decode()} ({status})")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, dtype, name):
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise GsparseError(f"{name} must be a contiguous CUDA {dtype} tensor")
    return t


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def k_for(n_s: int, keep: Tuple[int, int]) -> int:
    return int(lib().gsparse_k_for(n_s, keep[0], keep[1]))


def golomb_b_star(p: float) -> int:
    return int(lib().gsparse_golomb_b_star(p))


def golomb_chunk_hint(capacity: int) -> int:
    """Side-table chunk recommended for lists of up to `capacity` codewords."""
    return int(lib().gsparse_golomb_chunk_hint(capacity))


def warmup_keep(t: int, T: int, start: float = 0.25, end: float = 0.001, den: int = 1_000_000) -> Tuple[int, int]:
    """Keep fraction (num, den) at step t of a warm-up of T steps (exponential from start to end)."""
    return int(lib().gsparse_warmup_keep_num(t, T, start, end, den)), den


def _pass_events(events):
    """(before, after) torch.cuda.Event pair -> a by-reference gsparse_pass_events, or None."""
    if events is None:
        return None
    before, after = events
    for e in (before, after):
        if not e.cuda_event:   # torch creates the CUDA event on its first record
            e.record()
    return ctypes.byref(GsparsePassEvents(before.cuda_event, after.cuda_event))


def status_tensor(device="cuda") -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


# ---------------------------------------------------------------------------------------------
# residual top-k

def residual_topk_workspace_size(n: int, num_segments: int = 1, keep=(1, 100)) -> int:
    return int(lib().gsparse_residual_topk_workspace_size(n, num_segments, keep[0], keep[1]))


def residual_topk_capacity(n: int, seg_sizes: Optional[Sequence[int]], keep) -> int:
    if seg_sizes is None:
        return k_for(n, keep)
    return sum(k_for(int(s), keep) for s in seg_sizes)


def residual_topk(g: torch.Tensor, residual: torch.Tensor, keep=(1, 100), seg_offsets: Optional[torch.Tensor] = None,
                  out_idx: Optional[torch.Tensor] = None, out_val: Optional[torch.Tensor] = None,
                  out_offsets: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  flags: int = 0, d_status: Optional[torch.Tensor] = None, capacity: Optional[int] = None,
                  pending: Optional[GsparsePending] = None, momentum: Optional[Tuple[torch.Tensor, float]] = None,
                  pass_events: Optional[Tuple[torch.cuda.Event, torch.cuda.Event]] = None):
    """residual <- acc with the sent entries zeroed. Returns (idx, val, offsets) device tensors;
    idx/val hold `capacity` slots of which offsets[-1] are used. `pending` (make_pending) are
    residual writes applied first. `momentum` = (u, m): momentum correction and masking
    (v = m u + g replaces g, u <- v, sent entries of u zeroed). `pass_events` = (before, after):
    CUDA events this call records around its streaming pass."""
    _dev(g, torch.float32, "g")
    _dev(residual, torch.float32, "residual")
    n = g.numel()
    T = 1 if seg_offsets is None else seg_offsets.numel() - 1
    if seg_offsets is not None:
        _dev(seg_offsets, torch.int64, "seg_offsets")
    if capacity is None:
        capacity = k_for(n, keep) + (0 if T == 1 else T)
    dev = g.device
    if out_idx is None:
        out_idx = torch.empty(max(capacity, 1), dtype=torch.int32, device=dev)
    if out_val is None:
        out_val = torch.empty(max(capacity, 1), dtype=torch.float32, device=dev)
    if out_offsets is None:
        out_offsets = torch.empty(T + 1, dtype=torch.int64, device=dev)
    if workspace is None:
        workspace = _workspace(residual_topk_workspace_size(n, T, keep), dev)
    pend = ctypes.byref(pending) if pending is not None else None
    if momentum is not None:
        u, m = momentum
        _dev(u, torch.float32, "momentum buffer")
        st = lib().gsparse_residual_topk_momentum(_ptr(g), _ptr(u), float(m), _ptr(residual), n, _ptr(seg_offsets), T,
                                                  keep[0], keep[1], _ptr(out_idx), _ptr(out_val), _ptr(out_offsets),
                                                  capacity, pend, flags, _ptr(workspace), workspace.numel(),
                                                  _ptr(d_status), _stream(dev), _pass_events(pass_events))
        _check(st, "gsparse_residual_topk_momentum")
        return out_idx, out_val, out_offsets
    st = lib().gsparse_residual_topk(_ptr(g), _ptr(residual), n, _ptr(seg_offsets), T, keep[0], keep[1],
                                     _ptr(out_idx), _ptr(out_val), _ptr(out_offsets), capacity, pend, flags,
                                     _ptr(workspace), workspace.numel(), _ptr(d_status), _stream(dev),
                                     _pass_events(pass_events))
    _check(st, "gsparse_residual_topk")
    return out_idx, out_val, out_offsets


NOALLOC_MAX_N = 1 << 24


def residual_topk_noalloc(g: torch.Tensor, residual: torch.Tensor, keep=(1, 100),
                          out_idx: Optional[torch.Tensor] = None, out_val: Optional[torch.Tensor] = None,
                          out_offsets: Optional[torch.Tensor] = None, d_status: Optional[torch.Tensor] = None,
                          capacity: Optional[int] = None):
    """Global residual top-k whose scratch is the library's own fixed device array (for callers that
    must not allocate; n <= NOALLOC_MAX_N). Outputs as for residual_topk; pass them in to allocate
    nothing here either."""
    _dev(g, torch.float32, "g")
    _dev(residual, torch.float32, "residual")
    n = g.numel()
    dev = g.device
    if capacity is None:
        capacity = k_for(n, keep)
    if out_idx is None:
        out_idx = torch.empty(max(capacity, 1), dtype=torch.int32, device=dev)
    if out_val is None:
        out_val = torch.empty(max(capacity, 1), dtype=torch.float32, device=dev)
    if out_offsets is None:
        out_offsets = torch.empty(2, dtype=torch.int64, device=dev)
    st = lib().gsparse_residual_topk_noalloc(_ptr(g), _ptr(residual), n, keep[0], keep[1], _ptr(out_idx),
                                             _ptr(out_val), _ptr(out_offsets), capacity, _ptr(d_status),
                                             _stream(dev))
    _check(st, "gsparse_residual_topk_noalloc")
    return out_idx, out_val, out_offsets


# ---------------------------------------------------------------------------------------------
# quantise

def make_pending(idx: torch.Tensor, val: torch.Tensor, d_count: torch.Tensor,
                 capacity: Optional[int] = None) -> GsparsePending:
    """Residual writes residual[idx_j] <- val_j for the next residual_topk (e.g. quantize's feedback)."""
    cap = idx.numel() if capacity is None else capacity
    return GsparsePending(_ptr(idx), _ptr(val), _ptr(d_count), cap)


def quantize(idx: torch.Tensor, val: torch.Tensor, d_end: torch.Tensor, d_begin: Optional[torch.Tensor] = None,
             residual: Optional[torch.Tensor] = None, write_dequantized: bool = False,
             feedback_out: Optional[torch.Tensor] = None,
             sign_bits: Optional[torch.Tensor] = None, means: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None, d_status: Optional[torch.Tensor] = None,
             capacity: Optional[int] = None):
    """Returns (sign_bits uint32-as-int32 tensor, means float32[2])."""
    dev = val.device
    capacity = val.numel() if capacity is None else capacity
    if sign_bits is None:
        sign_bits = torch.zeros(max((capacity + 31) // 32, 1), dtype=torch.int32, device=dev)
    if means is None:
        means = torch.empty(2, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = _workspace(lib().gsparse_quantize_workspace_size(capacity), dev)
    n = 0 if residual is None else residual.numel()
    st = lib().gsparse_quantize(_ptr(idx), _ptr(val), _ptr(d_begin), _ptr(d_end), capacity, _ptr(residual), n,
                                _ptr(feedback_out), _ptr(sign_bits), _ptr(means), int(write_dequantized),
                                _ptr(workspace), workspace.numel(), _ptr(d_status), _stream(dev))
    _check(st, "gsparse_quantize")
    return sign_bits, means


def quantize_segments(idx: torch.Tensor, val: torch.Tensor, offsets: torch.Tensor,
                      residual: Optional[torch.Tensor] = None, write_dequantized: bool = False,
                      feedback_out: Optional[torch.Tensor] = None, sign_bits: Optional[torch.Tensor] = None,
                      means: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                      d_status: Optional[torch.Tensor] = None, capacity: Optional[int] = None):
    """2-bit quantisation of the T sub-lists [offsets[s], offsets[s+1]) in one call (per-segment
    means). Returns (sign_bits, means float32[2T])."""
    dev = val.device
    _dev(offsets, torch.int64, "offsets")
    T = offsets.numel() - 1
    capacity = val.numel() if capacity is None else capacity
    if sign_bits is None:
        sign_bits = torch.zeros(max((capacity + 31) // 32, 1), dtype=torch.int32, device=dev)
    if means is None:
        means = torch.empty(2 * T, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = _workspace(lib().gsparse_quantize_segments_workspace_size(capacity, T), dev)
    n = 0 if residual is None else residual.numel()
    st = lib().gsparse_quantize_segments(_ptr(idx), _ptr(val), _ptr(offsets), T, capacity, _ptr(residual), n,
                                         _ptr(feedback_out), _ptr(sign_bits), _ptr(means), int(write_dequantized),
                                         _ptr(workspace), workspace.numel(), _ptr(d_status), _stream(dev))
    _check(st, "gsparse_quantize_segments")
    return sign_bits, means


# ---------------------------------------------------------------------------------------------
# binarise

def binarize_workspace_size(n: int, num_segments: int = 1, keep=(1, 1000)) -> int:
    return int(lib().gsparse_binarize_workspace_size(n, num_segments, keep[0], keep[1]))


def binarize(g: torch.Tensor, residual: torch.Tensor, keep=(1, 1000), seg_offsets: Optional[torch.Tensor] = None,
             out_idx=None, out_val=None, mean=None, out_offsets=None, workspace=None, flags: int = 0,
             d_status=None, capacity: Optional[int] = None, want_values: bool = True, by_magnitude: bool = False,
             pass_events=None):
    """Returns (idx, val or None, mean[T], offsets[T+1]). by_magnitude: the magnitude-first reading
    (top fraction by |acc|, then the sign with the larger mean)."""
    if by_magnitude:
        flags |= GSPARSE_BINARIZE_BY_MAGNITUDE
    _dev(g, torch.float32, "g")
    _dev(residual, torch.float32, "residual")
    n = g.numel()
    T = 1 if seg_offsets is None else seg_offsets.numel() - 1
    dev = g.device
    if capacity is None:
        capacity = k_for(n, keep) + (0 if T == 1 else T)
    if out_idx is None:
        out_idx = torch.empty(max(capacity, 1), dtype=torch.int32, device=dev)
    if out_val is None and want_values:
        out_val = torch.empty(max(capacity, 1), dtype=torch.float32, device=dev)
    if mean is None:
        mean = torch.empty(T, dtype=torch.float32, device=dev)
    if out_offsets is None:
        out_offsets = torch.empty(T + 1, dtype=torch.int64, device=dev)
    if workspace is None:
        workspace = _workspace(binarize_workspace_size(n, T, keep), dev)
    st = lib().gsparse_binarize(_ptr(g), _ptr(residual), n, _ptr(seg_offsets), T, keep[0], keep[1], _ptr(out_idx),
                                _ptr(out_val), _ptr(mean), _ptr(out_offsets), capacity, flags, _ptr(workspace),
                                workspace.numel(), _ptr(d_status), _stream(dev), _pass_events(pass_events))
    _check(st, "gsparse_binarize")
    return out_idx, out_val, mean, out_offsets


# ---------------------------------------------------------------------------------------------
# Golomb

def golomb_word_capacity(capacity: int, b: int, n: int) -> int:
    """Words enough for any ascending list of <= capacity indices below n."""
    bits = capacity * (b + 1) + ((n + 1) >> b) + 64
    return (bits + 31) // 32


def golomb_encode(idx: torch.Tensor, d_end: torch.Tensor, b: int, n: int, d_begin: Optional[torch.Tensor] = None,
                  base: int = 0, chunk: int = 64, words=None, nbits=None, table=None, workspace=None,
                  d_status=None, capacity: Optional[int] = None):
    """Returns (words int32 tensor, nbits int64[1] tensor, chunk table int64[C, 2] or None)."""
    dev = idx.device
    capacity = idx.numel() if capacity is None else capacity
    if words is None:
        words = torch.empty(golomb_word_capacity(capacity, b, n), dtype=torch.int32, device=dev)
    if nbits is None:
        nbits = torch.zeros(1, dtype=torch.int64, device=dev)
    if table is None and chunk > 0:
        table = torch.empty((max((capacity + chunk - 1) // chunk, 1), 2), dtype=torch.int64, device=dev)
    if workspace is None:
        workspace = _workspace(lib().gsparse_golomb_encode_workspace_size(capacity), dev)
    st = lib().gsparse_golomb_encode(_ptr(idx), _ptr(d_begin), _ptr(d_end), capacity, base, b, _ptr(words),
                                     words.numel(), _ptr(nbits), _ptr(table), chunk, _ptr(workspace),
                                     workspace.numel(), _ptr(d_status), _stream(dev))
    _check(st, "gsparse_golomb_encode")
    return words, nbits, table


def golomb_decode(words: torch.Tensor, nbits: torch.Tensor, d_count: torch.Tensor, capacity: int, b: int,
                  base: int = 0, table: Optional[torch.Tensor] = None, chunk: int = 64, n_limit: int = 2**31 - 1,
                  out_idx=None, d_status=None):
    dev = words.device
    if out_idx is None:
        out_idx = torch.empty(max(capacity, 1), dtype=torch.int32, device=dev)
    st = lib().gsparse_golomb_decode(_ptr(words), words.numel(), _ptr(nbits), _ptr(d_count), capacity, base, b,
                                     _ptr(table),
                                     chunk if table is not None else 0, n_limit, _ptr(out_idx), _ptr(d_status),
                                     _stream(dev))
    _check(st, "gsparse_golomb_decode")
    return out_idx


# ---------------------------------------------------------------------------------------------
# scatter-accumulate and combine

def make_list(idx: torch.Tensor, d_count: torch.Tensor, val: Optional[torch.Tensor] = None,
              uniform_val: Optional[torch.Tensor] = None, capacity: Optional[int] = None) -> GsparseList:
    cap = idx.numel() if capacity is None else capacity
    return GsparseList(_ptr(idx), _ptr(val), _ptr(uniform_val), _ptr(d_count), cap)


def scatter_accumulate(lists: Sequence[GsparseList], n: int, dense_out: Optional[torch.Tensor] = None,
                       merged: bool = False, merged_capacity: Optional[int] = None, device="cuda",
                       workspace=None, d_status=None, want_dense: bool = True):
    """Returns (dense or None, merged_idx, merged_val, merged_count) (merged_* None unless merged)."""
    W = len(lists)
    arr = (GsparseList * W)(*lists)
    dev = torch.device(device)
    if dense_out is None and want_dense:
        dense_out = torch.empty(max(n, 1), dtype=torch.float32, device=dev)
    mi = mv = mc = None
    if merged:
        cap = merged_capacity if merged_capacity is not None else sum(int(x.capacity) for x in lists)
        mi = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
        mv = torch.empty(max(cap, 1), dtype=torch.float32, device=dev)
        mc = torch.zeros(1, dtype=torch.int64, device=dev)
    else:
        cap = 0
    if workspace is None:
        workspace = _workspace(lib().gsparse_scatter_accumulate_workspace_size(W, n), dev)
    st = lib().gsparse_scatter_accumulate(arr, W, n, _ptr(dense_out), _ptr(mi), _ptr(mv), _ptr(mc), cap,
                                          _ptr(workspace), workspace.numel(), _ptr(d_status), _stream(dev))
    _check(st, "gsparse_scatter_accumulate")
    return dense_out, mi, mv, mc


def accumulate_combine(lists: Sequence[GsparseList], n: int, L: torch.Tensor, out: Optional[torch.Tensor] = None,
                       alpha: float = 1.0, beta: float = 1.0, mode: int = 0, own: int = -1,
                       dense_out: Optional[torch.Tensor] = None, workspace=None, d_status=None):
    """Fused receive side: out = combine(scatter_accumulate(lists), L) without materialising G."""
    W = len(lists)
    arr = (GsparseList * W)(*lists)
    dev = L.device
    if out is None:
        out = torch.empty_like(L)
    if workspace is None:
        workspace = _workspace(lib().gsparse_accumulate_combine_workspace_size(W, n), dev)
    st = lib().gsparse_accumulate_combine(arr, W, n, _ptr(L), _ptr(out), alpha, beta, mode, own, _ptr(dense_out),
                                          _ptr(workspace), workspace.numel(), _ptr(d_status), _stream(dev))
    _check(st, "gsparse_accumulate_combine")
    return out


def combine_local(G: torch.Tensor, L: torch.Tensor, out: Optional[torch.Tensor] = None, alpha: float = 1.0,
                  beta: float = 1.0, mode: int = 0, own_idx=None, own_val=None, own_count=None,
                  own_capacity: int = 0, d_status=None):
    dev = G.device
    if out is None:
        out = torch.empty_like(G)
    st = lib().gsparse_combine_local(_ptr(G), _ptr(L), _ptr(out), G.numel(), alpha, beta, mode, _ptr(own_idx),
                                     _ptr(own_val), _ptr(own_count), own_capacity, _ptr(d_status), _stream(dev))
    _check(st, "gsparse_combine_local")
    return out
