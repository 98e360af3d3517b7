"""CPU oracle for the gradient-compression hot path -- TEST INFRASTRUCTURE ONLY.

Python view (ctypes + numpy) of the plain C++17 oracle in ``oracle/oracle.cpp``. Only the tests,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import this module; the
product path (``compressed_sgd_b200``) never does, and the two share no code.

Every function takes and returns host numpy arrays and raises ``OracleError`` on a non-zero
status. The rules each function follows are stated, with the page and section they come from,
beside the C++ code.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

_STATUS = {1: "invalid argument", 2: "capacity", 3: "corrupt stream", 4: "index out of range"}


class OracleError(RuntimeError):
    def __init__(self, status: int):
        super().__init__(f"oracle status {status}: {_STATUS.get(status, '?')}")
        self.status = status


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so with g++ (plain IEEE fp32, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, _SRC])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        i64, i32, vp, f32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_float, ctypes.c_double
        _lib.orc_k_for.argtypes = [i64, i64, i64]
        _lib.orc_k_for.restype = i64
        _lib.orc_golomb_b_star.argtypes = [f64]
        _lib.orc_golomb_b_star.restype = i32
        _lib.orc_warmup_keep_num.argtypes = [i64, i64, f64, f64, i64]
        _lib.orc_warmup_keep_num.restype = i64
        _lib.orc_residual_topk.argtypes = [vp, vp, i64, vp, i32, i64, i64, vp, vp, vp, i64]
        _lib.orc_residual_topk_momentum.argtypes = [vp, vp, f32, vp, i64, vp, i32, i64, i64, vp, vp, vp, i64]
        _lib.orc_quantize.argtypes = [vp, vp, i64, vp, i64, vp, vp, i32]
        _lib.orc_binarize.argtypes = [vp, vp, i64, vp, i32, i64, i64, vp, vp, vp, vp, i64]
        _lib.orc_binarize_magnitude.argtypes = [vp, vp, i64, vp, i32, i64, i64, vp, vp, vp, vp, i64]
        _lib.orc_golomb_encode.argtypes = [vp, i64, i64, i32, vp, i64, vp, i64, vp]
        _lib.orc_golomb_decode.argtypes = [vp, ctypes.c_uint64, i64, i64, i32, i64, vp]
        _lib.orc_scatter_accumulate.argtypes = [i32, vp, vp, vp, vp, i64, vp, vp, vp, vp, i64]
        _lib.orc_combine_local.argtypes = [vp, vp, vp, i64, f32, f32, i32, vp, vp, i64]
        for name in ("orc_residual_topk", "orc_residual_topk_momentum", "orc_quantize", "orc_binarize",
                     "orc_binarize_magnitude", "orc_golomb_encode",
                     "orc_golomb_decode", "orc_scatter_accumulate", "orc_combine_local"):
            getattr(_lib, name).restype = ctypes.c_int
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _check(st: int):
    if st != 0:
        raise OracleError(st)


def _segments(n: int, seg: Optional[Sequence[int]]) -> np.ndarray:
    return np.array([0, n] if seg is None else list(seg), dtype=np.int64)


def k_for(n_s: int, num: int, den: int) -> int:
    return int(_L().orc_k_for(n_s, num, den))


def golomb_b_star(p: float) -> int:
    return int(_L().orc_golomb_b_star(p))


def warmup_keep(t: int, T: int, start: float = 0.25, end: float = 0.001, den: int = 1_000_000):
    """Keep fraction (num, den) at step t of a warm-up of T steps."""
    return int(_L().orc_warmup_keep_num(t, T, start, end, den)), den


def residual_topk(g: np.ndarray, r: np.ndarray, keep=(1, 100), seg=None):
    """Returns (idx int32[K], val float32[K], offsets int64[T+1], new residual float32[n])."""
    g = np.ascontiguousarray(g, dtype=np.float32)
    r = np.array(r, dtype=np.float32, copy=True)
    n = g.size
    s = _segments(n, seg)
    T = s.size - 1
    cap = sum(k_for(int(s[t + 1] - s[t]), *keep) for t in range(T))
    idx = np.empty(max(cap, 1), np.int32)
    val = np.empty(max(cap, 1), np.float32)
    off = np.empty(T + 1, np.int64)
    _check(_L().orc_residual_topk(_p(g), _p(r), n, _p(s), T, keep[0], keep[1], _p(idx), _p(val), _p(off), cap))
    return idx[:cap], val[:cap], off, r


def residual_topk_momentum(g: np.ndarray, u: np.ndarray, m: float, r: np.ndarray, keep=(1, 100), seg=None):
    """Momentum-corrected residual top-k with momentum masking.
    Returns (idx, val, offsets, new residual, new momentum)."""
    g = np.ascontiguousarray(g, dtype=np.float32)
    u = np.array(u, dtype=np.float32, copy=True)
    r = np.array(r, dtype=np.float32, copy=True)
    n = g.size
    s = _segments(n, seg)
    T = s.size - 1
    cap = sum(k_for(int(s[t + 1] - s[t]), *keep) for t in range(T))
    idx = np.empty(max(cap, 1), np.int32)
    val = np.empty(max(cap, 1), np.float32)
    off = np.empty(T + 1, np.int64)
    _check(_L().orc_residual_topk_momentum(_p(g), _p(u), float(m), _p(r), n, _p(s), T, keep[0], keep[1], _p(idx),
                                           _p(val), _p(off), cap))
    return idx[:cap], val[:cap], off, r, u


def quantize(idx: np.ndarray, val: np.ndarray, residual: Optional[np.ndarray] = None,
             write_dequantized: bool = False):
    """Returns (sign_bits uint32[ceil(K/32)], means float32[2], val', residual')."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    val = np.array(val, dtype=np.float32, copy=True)
    res = None if residual is None else np.array(residual, dtype=np.float32, copy=True)
    K = val.size
    bits = np.zeros(max((K + 31) // 32, 1), np.uint32)
    means = np.zeros(2, np.float32)
    n = 0 if res is None else res.size
    _check(_L().orc_quantize(_p(idx), _p(val), K, _p(res), n, _p(bits), _p(means), int(write_dequantized)))
    return bits[:(K + 31) // 32], means, val, res


def binarize(g: np.ndarray, r: np.ndarray, keep=(1, 1000), seg=None, by_magnitude: bool = False):
    """Returns (idx int32[K'], val float32[K'], mean float32[T], offsets int64[T+1], new residual).
    by_magnitude: the magnitude-first reading (top-k by |acc|, then the sign with the larger mean)."""
    g = np.ascontiguousarray(g, dtype=np.float32)
    r = np.array(r, dtype=np.float32, copy=True)
    n = g.size
    s = _segments(n, seg)
    T = s.size - 1
    cap = sum(k_for(int(s[t + 1] - s[t]), *keep) for t in range(T))
    idx = np.empty(max(cap, 1), np.int32)
    val = np.empty(max(cap, 1), np.float32)
    mean = np.empty(T, np.float32)
    off = np.empty(T + 1, np.int64)
    fn = _L().orc_binarize_magnitude if by_magnitude else _L().orc_binarize
    _check(fn(_p(g), _p(r), n, _p(s), T, keep[0], keep[1], _p(idx), _p(val), _p(mean), _p(off), cap))
    K = int(off[-1])
    return idx[:K], val[:K], mean, off, r


def golomb_encode(idx: np.ndarray, b: int, base: int = 0, chunk: int = 0):
    """Returns (words uint32[ceil(nbits/32)], nbits, chunk_table int64[C, 2] or None)."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    K = idx.size
    # capacity: every codeword is at most (gap >> b) + 1 + b bits, gaps summing to < 2^31 + K
    gaps_hi = int(idx[-1]) - base + 1 if K else 0
    cap_bits = K * (b + 1) + (gaps_hi >> b) + 64
    words = np.zeros((cap_bits + 31) // 32 + 1, np.uint32)
    table = np.zeros(((K + chunk - 1) // chunk if chunk > 0 else 0, 2), np.int64) if chunk > 0 else None
    nbits = ctypes.c_uint64(0)
    _check(_L().orc_golomb_encode(_p(idx), K, base, b, _p(words), words.size, _p(table),
                                  chunk if chunk > 0 else 0, ctypes.addressof(nbits)))
    nb = int(nbits.value)
    return words[:(nb + 31) // 32], nb, table


def golomb_decode(words: np.ndarray, nbits: int, K: int, b: int, base: int = 0, n_limit: int = 2**31 - 1):
    words = np.ascontiguousarray(words, dtype=np.uint32)
    if words.size == 0:
        words = np.zeros(1, np.uint32)
    out = np.empty(max(K, 1), np.int32)
    _check(_L().orc_golomb_decode(_p(words), nbits, K, base, b, n_limit, _p(out)))
    return out[:K]


def scatter_accumulate(lists, n: int, dense: bool = True, merged: bool = True):
    """lists: sequence of (idx, val) or (idx, None, uniform_value). Returns (dense, merged_idx, merged_val)."""
    W = len(lists)
    keep_alive = []
    idx_ptrs = (ctypes.c_void_p * W)()
    val_ptrs = (ctypes.c_void_p * W)()
    uniform = np.zeros(W, np.float32)
    counts = np.zeros(W, np.int64)
    total = 0
    for w, item in enumerate(lists):
        idx = np.ascontiguousarray(item[0], dtype=np.int32)
        keep_alive.append(idx)
        idx_ptrs[w] = idx.ctypes.data if idx.size else None
        counts[w] = idx.size
        total += idx.size
        if item[1] is not None:
            val = np.ascontiguousarray(item[1], dtype=np.float32)
            keep_alive.append(val)
            val_ptrs[w] = val.ctypes.data if val.size else None
            if val.size == 0:
                val_ptrs[w] = None
        else:
            val_ptrs[w] = None
            uniform[w] = item[2]
    d = np.empty(max(n, 1), np.float32) if dense else None
    mi = np.empty(max(total, 1), np.int32) if merged else None
    mv = np.empty(max(total, 1), np.float32) if merged else None
    mc = ctypes.c_int64(0)
    _check(_L().orc_scatter_accumulate(W, ctypes.cast(idx_ptrs, ctypes.c_void_p), ctypes.cast(val_ptrs, ctypes.c_void_p),
                                       _p(uniform), _p(counts), n, _p(d), _p(mi), _p(mv),
                                       ctypes.addressof(mc) if merged else None, total))
    u = int(mc.value)
    return (d[:n] if dense else None), (mi[:u] if merged else None), (mv[:u] if merged else None)


def combine_local(G: np.ndarray, L: np.ndarray, alpha: float = 1.0, beta: float = 1.0, mode: int = 0,
                  own_idx: Optional[np.ndarray] = None, own_val: Optional[np.ndarray] = None):
    G = np.ascontiguousarray(G, dtype=np.float32)
    L = np.ascontiguousarray(L, dtype=np.float32)
    n = G.size
    out = np.empty(max(n, 1), np.float32)
    oi = None if own_idx is None else np.ascontiguousarray(own_idx, dtype=np.int32)
    ov = None if own_val is None else np.ascontiguousarray(own_val, dtype=np.float32)
    cnt = 0 if oi is None else oi.size
    _check(_L().orc_combine_local(_p(G), _p(L), _p(out), n, alpha, beta, mode, _p(oi), _p(ov), cnt))
    return out[:n]
