"""CPU oracle of the group-32 symmetric INT4 quantizer path.

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's CPU
baseline use it.  The product package never imports it.  The arithmetic lives
in ``qat4_oracle.c`` (plain C, fp64 sums); this module only marshals NumPy
arrays into it.  ``twin.py`` is a second, independent NumPy implementation for
tiny inputs.
"""
from __future__ import annotations

import ctypes as ct

import numpy as np

from .build import build as _build

_LIB = None
_P = ct.c_void_p
_I64 = ct.c_int64


def lib():
    global _LIB
    if _LIB is None:
        _LIB = ct.CDLL(_build())
        L = _LIB
        L.oracle_set_threads.argtypes = [ct.c_int]
        L.oracle_set_threads.restype = ct.c_int
        L.oracle_hessian.argtypes = [_P, _I64, _I64, _P]
        L.oracle_hessian_entries.argtypes = [_P, _I64, _I64, _P, _P, _I64, _P]
        L.oracle_hessian_block.argtypes = [_P, _I64, _I64, _I64, _I64, _I64, _I64, _P]
        L.oracle_hessian_blocks.argtypes = [_P, _I64, _I64, _P, _P, _I64, _I64, _P]
        L.oracle_scale_search.argtypes = [_P, _I64, _I64, _P, _I64, _P, ct.c_int32, _P, _P, _P, _P]
        L.oracle_lsq_fwd.argtypes = [_P, _P, _I64, _I64, _P]
        L.oracle_lsq_bwd.argtypes = [_P, _P, _P, ct.c_int, _I64, _I64, ct.c_float, _P, _P]
        L.oracle_pack_w4a16.argtypes = [_P, _P, _I64, _I64, _P, _P]
        L.oracle_codes.argtypes = [_P, _P, _I64, _I64, _P]
        L.oracle_lsq_fwd_rowwise.argtypes = [_P, _P, _I64, _I64, _P]
        L.oracle_lsq_bwd_rowwise.argtypes = [_P, _P, _P, ct.c_int, _I64, _I64, ct.c_float, _P, _P]
        L.oracle_pack_w4a16_rowwise.argtypes = [_P, _P, _I64, _I64, _P, _P]
        L.oracle_scale_search_rowwise.argtypes = [_P, _I64, _I64, _P, _I64, _P, ct.c_int32, _P, _P, _P, _P]
        L.oracle_w4a16_gemv.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _P]
        for f in ("oracle_hessian", "oracle_hessian_entries", "oracle_hessian_block", "oracle_hessian_blocks",
                  "oracle_scale_search", "oracle_lsq_fwd", "oracle_lsq_bwd",
                  "oracle_pack_w4a16", "oracle_codes", "oracle_lsq_fwd_rowwise",
                  "oracle_lsq_bwd_rowwise", "oracle_pack_w4a16_rowwise", "oracle_scale_search_rowwise",
                  "oracle_w4a16_gemv"):
            getattr(L, f).restype = None
    return _LIB


def _p(a: np.ndarray):
    return a.ctypes.data_as(_P)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int = 0) -> int:
    """Set the OpenMP thread count (n <= 0 keeps it); returns the count in use."""
    return lib().oracle_set_threads(int(n))


def hessian(X_bits: np.ndarray) -> np.ndarray:
    """H = X^T X / n in float64 for X given as bf16 bits [n, C]."""
    X = _c(X_bits, np.uint16)
    n, C = X.shape
    H = np.empty((C, C), np.float64)
    lib().oracle_hessian(_p(X), n, C, _p(H))
    return H


def hessian_entries(X_bits: np.ndarray, ii, jj) -> np.ndarray:
    X = _c(X_bits, np.uint16)
    n, C = X.shape
    ii = _c(ii, np.int64)
    jj = _c(jj, np.int64)
    out = np.empty(ii.size, np.float64)
    lib().oracle_hessian_entries(_p(X), n, C, _p(ii), _p(jj), ii.size, _p(out))
    return out


def hessian_block(X_bits: np.ndarray, r0: int, nr: int, c0: int, nc: int) -> np.ndarray:
    X = _c(X_bits, np.uint16)
    n, C = X.shape
    out = np.empty((nr, nc), np.float64)
    lib().oracle_hessian_block(_p(X), n, C, r0, nr, c0, nc, _p(out))
    return out


def hessian_blocks(X_bits: np.ndarray, r0, c0, b: int) -> np.ndarray:
    """Blocks H[r0[m]:r0[m]+b, c0[m]:c0[m]+b] in float64, shape [count, b, b] (one block per thread)."""
    X = _c(X_bits, np.uint16)
    n, C = X.shape
    r0 = _c(r0, np.int64)
    c0 = _c(c0, np.int64)
    assert r0.shape == c0.shape and r0.ndim == 1 and 0 < b <= 256
    assert np.all((r0 >= 0) & (r0 + b <= C) & (c0 >= 0) & (c0 + b <= C))
    out = np.empty((r0.size, b, b), np.float64)
    lib().oracle_hessian_blocks(_p(X), n, C, _p(r0), _p(c0), r0.size, b, _p(out))
    return out


def scale_search(W: np.ndarray, H: np.ndarray, alpha: np.ndarray, *, all_err: bool = False):
    """Returns (delta f32 [R,G], idx i32 [R,G], best_err f64 [R,G][, all f64 [R,G,K]])."""
    W = _c(W, np.float32)
    H = _c(H, np.float32)
    alpha = _c(alpha, np.float32)
    R, C = W.shape
    G = C // 32
    K = alpha.size
    delta = np.empty((R, G), np.float32)
    idx = np.empty((R, G), np.int32)
    best = np.empty((R, G), np.float64)
    allv = np.empty((R, G, K), np.float64) if all_err else None
    lib().oracle_scale_search(_p(W), R, C, _p(H), H.shape[1], _p(alpha), K, _p(delta), _p(idx),
                              _p(best), _p(allv) if all_err else None)
    return (delta, idx, best, allv) if all_err else (delta, idx, best)


def lsq_fwd(W: np.ndarray, delta: np.ndarray) -> np.ndarray:
    W = _c(W, np.float32)
    delta = _c(delta, np.float32)
    R, C = W.shape
    Q = np.empty_like(W)
    lib().oracle_lsq_fwd(_p(W), _p(delta), R, C, _p(Q))
    return Q


def lsq_bwd(W: np.ndarray, delta: np.ndarray, G: np.ndarray, grad_scale: float):
    """G: float32 array, or uint16 bf16 bits.  Returns (grad_W f32, grad_delta f64)."""
    W = _c(W, np.float32)
    delta = _c(delta, np.float32)
    is_bf16 = np.asarray(G).dtype == np.uint16
    G = _c(G, np.uint16 if is_bf16 else np.float32)
    R, C = W.shape
    gW = np.empty_like(W)
    gD = np.empty((R, C // 32), np.float64)
    lib().oracle_lsq_bwd(_p(W), _p(delta), _p(G), int(is_bf16), R, C, ct.c_float(grad_scale),
                         _p(gW), _p(gD))
    return gW, gD


def pack_w4a16(W: np.ndarray, delta: np.ndarray):
    """Returns (packed uint8 [R, C/2], scale16 bits uint16 [R, C/32])."""
    W = _c(W, np.float32)
    delta = _c(delta, np.float32)
    R, C = W.shape
    packed = np.empty((R, C // 2), np.uint8)
    s16 = np.empty((R, C // 32), np.uint16)
    lib().oracle_pack_w4a16(_p(W), _p(delta), R, C, _p(packed), _p(s16))
    return packed, s16


def codes(W: np.ndarray, delta: np.ndarray) -> np.ndarray:
    W = _c(W, np.float32)
    delta = _c(delta, np.float32)
    R, C = W.shape
    out = np.empty((R, C), np.int8)
    lib().oracle_codes(_p(W), _p(delta), R, C, _p(out))
    return out


# ---------------------------------------------------------------- per-channel
def lsq_fwd_rowwise(W: np.ndarray, delta: np.ndarray) -> np.ndarray:
    """Q with one scale per row: delta float32 [R]."""
    W = _c(W, np.float32)
    delta = _c(delta, np.float32).reshape(-1)
    R, C = W.shape
    Q = np.empty_like(W)
    lib().oracle_lsq_fwd_rowwise(_p(W), _p(delta), R, C, _p(Q))
    return Q


def lsq_bwd_rowwise(W: np.ndarray, delta: np.ndarray, G: np.ndarray, grad_scale: float):
    """Returns (grad_W f32 [R, C], grad_delta f64 [R])."""
    W = _c(W, np.float32)
    delta = _c(delta, np.float32).reshape(-1)
    is_bf16 = np.asarray(G).dtype == np.uint16
    G = _c(G, np.uint16 if is_bf16 else np.float32)
    R, C = W.shape
    gW = np.empty_like(W)
    gD = np.empty(R, np.float64)
    lib().oracle_lsq_bwd_rowwise(_p(W), _p(delta), _p(G), int(is_bf16), R, C, ct.c_float(grad_scale),
                                 _p(gW), _p(gD))
    return gW, gD


def pack_w4a16_rowwise(W: np.ndarray, delta: np.ndarray):
    """Returns (packed uint8 [R, C/2], scale16 bits uint16 [R])."""
    W = _c(W, np.float32)
    delta = _c(delta, np.float32).reshape(-1)
    R, C = W.shape
    packed = np.empty((R, C // 2), np.uint8)
    s16 = np.empty(R, np.uint16)
    lib().oracle_pack_w4a16_rowwise(_p(W), _p(delta), R, C, _p(packed), _p(s16))
    return packed, s16


def scale_search_rowwise(W: np.ndarray, H: np.ndarray, alpha: np.ndarray, *, all_err: bool = False):
    """Per-channel search with the full H.  Returns (delta f32 [R], idx i32 [R], best f64 [R][, all [R, K]])."""
    W = _c(W, np.float32)
    H = _c(H, np.float32)
    alpha = _c(alpha, np.float32)
    R, C = W.shape
    K = alpha.size
    delta = np.empty(R, np.float32)
    idx = np.empty(R, np.int32)
    best = np.empty(R, np.float64)
    allv = np.empty((R, K), np.float64) if all_err else None
    lib().oracle_scale_search_rowwise(_p(W), R, C, _p(H), H.shape[1], _p(alpha), K, _p(delta), _p(idx),
                                      _p(best), _p(allv) if all_err else None)
    return (delta, idx, best, allv) if all_err else (delta, idx, best)


def w4a16_gemv(x_bits: np.ndarray, packed: np.ndarray, scales16: np.ndarray, group: int) -> np.ndarray:
    """y [M, R] (float64) = x @ (scale * code)^T from the packed export; x as bf16 bits [M, C]."""
    x = _c(np.atleast_2d(x_bits), np.uint16)
    packed = _c(packed, np.uint8)
    scales16 = _c(scales16, np.uint16)
    M, C = x.shape
    R = packed.shape[0]
    y = np.empty((M, R), np.float64)
    lib().oracle_w4a16_gemv(_p(x), _p(packed), _p(scales16), M, R, C, int(group), _p(y))
    return y


def fq_gemm(X_bits: np.ndarray, W: np.ndarray, delta: np.ndarray) -> np.ndarray:
    """Y [T, R] (float64) = X @ bf16(Q_delta(W))^T; X as bf16 bits [T, C], W float32 [R, C],
    delta float32 [R, C/32]."""
    X = _c(np.atleast_2d(X_bits), np.uint16)
    W = _c(W, np.float32)
    delta = _c(delta, np.float32)
    T, C = X.shape
    R = W.shape[0]
    Y = np.empty((T, R), np.float64)
    lib().oracle_fq_gemm(_p(X), _p(W), _p(delta), T, R, C, _p(Y))
    return Y


def fq_gemm_entries(X_bits: np.ndarray, W: np.ndarray, delta: np.ndarray, tt, rr) -> np.ndarray:
    """Y[tt[m], rr[m]] of fq_gemm (float64), for sampled checks of large outputs."""
    X = _c(np.atleast_2d(X_bits), np.uint16)
    W = _c(W, np.float32)
    delta = _c(delta, np.float32)
    tt = _c(tt, np.int64)
    rr = _c(rr, np.int64)
    out = np.empty(tt.size, np.float64)
    lib().oracle_fq_gemm_entries(_p(X), _p(W), _p(delta), X.shape[1], tt.size, _p(tt), _p(rr), _p(out))
    return out


def refine(W: np.ndarray, H: np.ndarray, alpha: np.ndarray, idx_start: np.ndarray, sweeps: int = 1):
    """Full-objective coordinate descent from idx_start: (delta float32 [R, G], idx int32 [R, G],
    obj float64 [R])."""
    W = _c(W, np.float32)
    H = _c(H, np.float32)
    alpha = _c(alpha, np.float32)
    R, C = W.shape
    idx = _c(idx_start, np.int32).copy()
    delta = np.empty((R, C // 32), np.float32)
    obj = np.empty(R, np.float64)
    lib().oracle_refine(_p(W), R, C, _p(H), H.shape[1], _p(alpha), alpha.size, int(sweeps), _p(idx),
                        _p(delta), _p(obj))
    return delta, idx, obj


def refine_replay(W: np.ndarray, H: np.ndarray, alpha: np.ndarray, idx_start: np.ndarray, idx_pick: np.ndarray):
    """For one sweep that moved idx_start to idx_pick: per (row, group) the minimum of the full
    objective over the group's candidates at that point of the sweep, and its value at the pick."""
    W = _c(W, np.float32)
    H = _c(H, np.float32)
    alpha = _c(alpha, np.float32)
    R, C = W.shape
    s = _c(idx_start, np.int32)
    k = _c(idx_pick, np.int32)
    emin = np.empty((R, C // 32), np.float64)
    epick = np.empty((R, C // 32), np.float64)
    lib().oracle_refine_replay(_p(W), R, C, _p(H), H.shape[1], _p(alpha), alpha.size, _p(s), _p(k), _p(emin),
                               _p(epick))
    return emin, epick
