"""Python binding of libqat4, the B200 group-32 symmetric INT4 quantizer.

Argument marshalling only: every call checks tensor placement, dtype and
shape, allocates missing outputs with torch (device memory), and passes raw
device pointers plus the current CUDA stream to the C ABI in
``include/qat4.h``.  All arithmetic runs in the CUDA kernels of
``libqat4.so``; if that library is missing, every call raises.

Functions (same names as the C entry points, without the ``qat4_`` prefix):
``hessian``, ``hessian_workspace_bytes``, ``hessian_noalloc``, ``scale_search``, ``lsq_fwd``,
``lsq_bwd``, ``lsq_fwd_bwd``, ``lsq_fwd_bwd_host``, ``pack_w4a16``, ``sync_check``,
``status_string``, ``selftest_bounded_wait``.
"""
from __future__ import annotations

import ctypes as ct
import math
import os
import struct

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqat4.so")

# LSQ step-gradient normalisation 1/sqrt(group size * positive levels) as float32
GRAD_SCALE = struct.unpack("<f", struct.pack("<f", 1.0 / math.sqrt(32.0 * 7.0)))[0]

STATUS = {0: "QAT4_OK", 1: "QAT4_ERR_NULL", 2: "QAT4_ERR_SHAPE", 3: "QAT4_ERR_ALIGN",
          4: "QAT4_ERR_DTYPE", 5: "QAT4_ERR_WORKSPACE", 6: "QAT4_ERR_CUDA", 7: "QAT4_ERR_TIMEOUT"}
QAT4_F32, QAT4_BF16 = 0, 1

# (name, restype, argtypes) of every exported entry point
_P, _I64, _I32, _F, _Z = ct.c_void_p, ct.c_int64, ct.c_int32, ct.c_float, ct.c_size_t
EXPORTS = {
    "qat4_status_string": (ct.c_char_p, [ct.c_int]),
    "qat4_abi_version": (ct.c_int, []),
    "qat4_hessian_workspace_bytes": (_Z, [_I64, _I64]),
    "qat4_hessian": (ct.c_int, [_P, _I64, _I64, _P, _P, _Z, _P]),
    "qat4_hessian_partial": (ct.c_int, [_P, _I64, _I64, _I64, _P, _P, _Z, _P]),
    "qat4_hessian_noalloc": (ct.c_int, [_P, _I64, _I64, _P, _P]),
    "qat4_scale_search": (ct.c_int, [_P, _I64, _I64, _P, _I64, _P, _I32, _P, _P, _P, _P]),
    "qat4_lsq_fwd": (ct.c_int, [_P, _P, _I64, _I64, _P, _P]),
    "qat4_lsq_bwd": (ct.c_int, [_P, _P, _P, ct.c_int, _I64, _I64, _F, _P, _P, _P]),
    "qat4_lsq_fwd_bwd": (ct.c_int, [_P, _P, _P, ct.c_int, _I64, _I64, _F, _P, _P, _P, _P]),
    "qat4_lsq_fwd_bwd_host_workspace_bytes": (_Z, [_I64, _I64, ct.c_int]),
    "qat4_lsq_fwd_bwd_host": (ct.c_int, [_P, _P, _P, ct.c_int, _I64, _I64, _F, _P, _P, _P, _P, _Z, _P, _P]),
    "qat4_pack_w4a16": (ct.c_int, [_P, _P, _I64, _I64, _P, _P, _P]),
    "qat4_lsq_fwd_rowwise": (ct.c_int, [_P, _P, _I64, _I64, _P, _P]),
    "qat4_lsq_bwd_rowwise": (ct.c_int, [_P, _P, _P, ct.c_int, _I64, _I64, _F, _P, _P, _P]),
    "qat4_lsq_fwd_bwd_rowwise": (ct.c_int, [_P, _P, _P, ct.c_int, _I64, _I64, _F, _P, _P, _P, _P]),
    "qat4_pack_w4a16_rowwise": (ct.c_int, [_P, _P, _I64, _I64, _P, _P, _P]),
    "qat4_scale_search_rowwise_workspace_bytes": (_Z, [_I64, _I64]),
    "qat4_scale_search_rowwise": (ct.c_int, [_P, _I64, _I64, _P, _I64, _P, _I32, _P, _P, _P, _P, _Z, _P]),
    "qat4_w4a16_gemv": (ct.c_int, [_P, _I64, _P, _P, _I64, _I64, _I64, _P, _P]),
    "qat4_fq_gemm": (ct.c_int, [_P, _I64, _P, _P, _I64, _I64, _P, _P]),
    "qat4_fq_gemm_staged_workspace_bytes": (ct.c_size_t, [_I64, _I64]),
    "qat4_fq_gemm_staged": (ct.c_int, [_P, _I64, _P, _P, _I64, _I64, _P, _P, ct.c_size_t, _P]),
    "qat4_refine_workspace_bytes": (ct.c_size_t, [_I64, _I64]),
    "qat4_refine": (ct.c_int, [_P, _I64, _I64, _P, _I64, _P, ct.c_int32, ct.c_int32, _P, _P, _P, _P, _Z, _P]),
    "qat4_sync_check": (ct.c_int, [_P]),
    "qat4_selftest_bounded_wait": (ct.c_int, [_I64, _P]),
}

_lib = None


class Qat4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def lib() -> ct.CDLL:
    """Load libqat4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libqat4.so not found at {LIB_PATH}; build it with "
                              "`python -m int4_group_wise_b200.build` (no CPU fallback exists)")
        import torch  # noqa: F401  (loads the CUDA runtime shared with torch first)
        L = ct.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise Qat4Error(status, where)


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ct.c_void_p(s.cuda_stream)


def _dev(t, name, dtype=None, shape=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ct.c_void_p(t.data_ptr())


def _out(t, name, shape, dtype, like):
    import torch
    if t is None:
        return torch.empty(shape, dtype=dtype, device=like.device)
    _dev(t, name, dtype, shape)
    return t


def status_string(code: int) -> str:
    return lib().qat4_status_string(int(code)).decode()


def hessian_workspace_bytes(n: int, C: int) -> int:
    return int(lib().qat4_hessian_workspace_bytes(int(n), int(C)))


def hessian(X, H=None, workspace=None, stream=None):
    """H = X^T X / n for X bf16 [n, C]; returns float32 [C, C]."""
    import torch
    L = lib()
    _dev(X, "X", torch.bfloat16)
    n, C = X.shape
    H = _out(H, "H", (C, C), torch.float32, X)
    need = hessian_workspace_bytes(n, C)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    wp = _dev(workspace, "workspace", torch.uint8) if workspace is not None else None
    wbytes = workspace.numel() if workspace is not None else 0
    _check(L.qat4_hessian(_dev(X, "X"), n, C, _dev(H, "H"), wp, wbytes, _stream(stream)), "qat4_hessian")
    return H


def hessian_partial(X, n_total, H=None, workspace=None, stream=None):
    """One shard's share of a split-n Hessian: H = X^T X / n_total for this shard's rows X bf16
    [n, C]; the sum of all shards' partials is the Hessian of all n_total rows."""
    import torch
    L = lib()
    _dev(X, "X", torch.bfloat16)
    n, C = X.shape
    H = _out(H, "H", (C, C), torch.float32, X)
    need = hessian_workspace_bytes(n, C)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    wp = _dev(workspace, "workspace", torch.uint8) if workspace is not None else None
    wbytes = workspace.numel() if workspace is not None else 0
    _check(L.qat4_hessian_partial(_dev(X, "X"), n, C, int(n_total), _dev(H, "H"), wp, wbytes, _stream(stream)),
           "qat4_hessian_partial")
    return H


def hessian_noalloc(X, H=None, stream=None):
    """H = X^T X / n using the library's built-in scratch instead of a caller workspace.

    For callers that must not allocate device memory on their own (H may be
    passed in preallocated).  Calls that overlap on the GPU share the scratch
    and race; see include/qat4.h."""
    import torch
    L = lib()
    _dev(X, "X", torch.bfloat16)
    n, C = X.shape
    H = _out(H, "H", (C, C), torch.float32, X)
    _check(L.qat4_hessian_noalloc(_dev(X, "X"), n, C, _dev(H, "H"), _stream(stream)), "qat4_hessian_noalloc")
    return H


def scale_search(W, H, alpha, delta=None, idx=None, best_err=None, stream=None, want_err=True):
    """Returns (delta f32 [R, C/32], idx i32 [R, C/32], best_err f32 [R, C/32] or None)."""
    import torch
    L = lib()
    _dev(W, "W", torch.float32)
    R, C = W.shape
    _dev(H, "H", torch.float32)
    if H.dim() != 2 or H.shape[0] < C or H.shape[1] < C:
        raise ValueError("H must be at least [C, C]")
    _dev(alpha, "alpha", torch.float32)
    G = C // 32
    delta = _out(delta, "delta", (R, G), torch.float32, W)
    idx = _out(idx, "idx", (R, G), torch.int32, W)
    if want_err:
        best_err = _out(best_err, "best_err", (R, G), torch.float32, W)
    _check(L.qat4_scale_search(_dev(W, "W"), R, C, _dev(H, "H"), H.shape[1], _dev(alpha, "alpha"),
                               alpha.numel(), _dev(delta, "delta"), _dev(idx, "idx"),
                               _dev(best_err, "best_err") if best_err is not None else None,
                               _stream(stream)), "qat4_scale_search")
    return delta, idx, best_err


def _gdtype(G):
    import torch
    if G.dtype == torch.float32:
        return QAT4_F32
    if G.dtype == torch.bfloat16:
        return QAT4_BF16
    raise TypeError("G must be float32 or bfloat16")


def lsq_fwd(W, delta, Q=None, stream=None):
    import torch
    L = lib()
    _dev(W, "W", torch.float32)
    R, C = W.shape
    _dev(delta, "delta", torch.float32, (R, C // 32))
    Q = _out(Q, "Q", (R, C), torch.float32, W)
    _check(L.qat4_lsq_fwd(_dev(W, "W"), _dev(delta, "delta"), R, C, _dev(Q, "Q"), _stream(stream)),
           "qat4_lsq_fwd")
    return Q


def lsq_bwd(W, delta, G, grad_scale=GRAD_SCALE, grad_W=None, grad_delta=None, stream=None):
    import torch
    L = lib()
    _dev(W, "W", torch.float32)
    R, C = W.shape
    _dev(delta, "delta", torch.float32, (R, C // 32))
    _dev(G, "G", None, (R, C))
    grad_W = _out(grad_W, "grad_W", (R, C), torch.float32, W)
    grad_delta = _out(grad_delta, "grad_delta", (R, C // 32), torch.float32, W)
    _check(L.qat4_lsq_bwd(_dev(W, "W"), _dev(delta, "delta"), _dev(G, "G"), _gdtype(G), R, C,
                          ct.c_float(grad_scale), _dev(grad_W, "grad_W"), _dev(grad_delta, "grad_delta"),
                          _stream(stream)), "qat4_lsq_bwd")
    return grad_W, grad_delta


def lsq_fwd_bwd(W, delta, G, grad_scale=GRAD_SCALE, Q=None, grad_W=None, grad_delta=None, stream=None):
    import torch
    L = lib()
    _dev(W, "W", torch.float32)
    R, C = W.shape
    _dev(delta, "delta", torch.float32, (R, C // 32))
    _dev(G, "G", None, (R, C))
    Q = _out(Q, "Q", (R, C), torch.float32, W)
    grad_W = _out(grad_W, "grad_W", (R, C), torch.float32, W)
    grad_delta = _out(grad_delta, "grad_delta", (R, C // 32), torch.float32, W)
    _check(L.qat4_lsq_fwd_bwd(_dev(W, "W"), _dev(delta, "delta"), _dev(G, "G"), _gdtype(G), R, C,
                              ct.c_float(grad_scale), _dev(Q, "Q"), _dev(grad_W, "grad_W"),
                              _dev(grad_delta, "grad_delta"), _stream(stream)), "qat4_lsq_fwd_bwd")
    return Q, grad_W, grad_delta


def _host(t, name, dtype=None, shape=None):
    import torch
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise TypeError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ct.c_void_p(t.data_ptr())


def lsq_fwd_bwd_host_workspace_bytes(R: int, C: int, g_dtype: int) -> int:
    return int(lib().qat4_lsq_fwd_bwd_host_workspace_bytes(int(R), int(C), int(g_dtype)))


def lsq_fwd_bwd_host(W, delta, G, grad_scale=GRAD_SCALE, Q=None, grad_W=None, grad_delta=None,
                     workspace=None, stream=None, copy_stream=None):
    """The fused LSQ step on host tensors (page-locked for overlap), streamed through the current
    GPU in row chunks; returns host (Q, grad_W, grad_delta).  Asynchronous: synchronize `stream`
    (default: the current stream) before reading the outputs."""
    import torch
    L = lib()
    _host(W, "W", torch.float32)
    R, C = W.shape
    _host(delta, "delta", torch.float32, (R, C // 32))
    _host(G, "G", None, (R, C))
    gd = _gdtype(G)
    pin = W.is_pinned()
    Q = torch.empty((R, C), dtype=torch.float32, pin_memory=pin) if Q is None else Q
    grad_W = torch.empty((R, C), dtype=torch.float32, pin_memory=pin) if grad_W is None else grad_W
    grad_delta = torch.empty((R, C // 32), dtype=torch.float32, pin_memory=pin) if grad_delta is None else grad_delta
    need = lsq_fwd_bwd_host_workspace_bytes(R, C, gd)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=torch.cuda.current_device())
    cs = copy_stream if copy_stream is not None else _copy_stream()
    _check(L.qat4_lsq_fwd_bwd_host(_host(W, "W"), _host(delta, "delta"), _host(G, "G"), gd, R, C,
                                   ct.c_float(grad_scale), _host(Q, "Q", torch.float32, (R, C)),
                                   _host(grad_W, "grad_W", torch.float32, (R, C)),
                                   _host(grad_delta, "grad_delta", torch.float32, (R, C // 32)),
                                   _dev(workspace, "workspace"), workspace.numel(), _stream(stream),
                                   ct.c_void_p(cs.cuda_stream)), "qat4_lsq_fwd_bwd_host")
    return Q, grad_W, grad_delta


_copy_streams = {}


def _copy_stream():
    """One side stream per device for the downloads of lsq_fwd_bwd_host."""
    import torch
    d = torch.cuda.current_device()
    if d not in _copy_streams:
        _copy_streams[d] = torch.cuda.Stream(device=d)
    return _copy_streams[d]


def pack_w4a16(W, delta, packed=None, scales=None, stream=None):
    """Returns (packed uint8 [R, C/2], scales float16 [R, C/32])."""
    import torch
    L = lib()
    _dev(W, "W", torch.float32)
    R, C = W.shape
    _dev(delta, "delta", torch.float32, (R, C // 32))
    packed = _out(packed, "packed", (R, C // 2), torch.uint8, W)
    scales = _out(scales, "scales", (R, C // 32), torch.float16, W)
    _check(L.qat4_pack_w4a16(_dev(W, "W"), _dev(delta, "delta"), R, C, _dev(packed, "packed"),
                             _dev(scales, "scales"), _stream(stream)), "qat4_pack_w4a16")
    return packed, scales


# ------------------------------------------------------------------ per-channel
def rowwise_grad_scale(C: int) -> float:
    """float32(1/sqrt(C * 7)): the per-channel step-gradient normalisation."""
    return struct.unpack("<f", struct.pack("<f", 1.0 / math.sqrt(C * 7.0)))[0]


def lsq_fwd_rowwise(W, delta, Q=None, stream=None):
    """Q with one scale per row: delta float32 [R]."""
    import torch
    L = lib()
    _dev(W, "W", torch.float32)
    R, C = W.shape
    _dev(delta, "delta", torch.float32, (R,))
    Q = _out(Q, "Q", (R, C), torch.float32, W)
    _check(L.qat4_lsq_fwd_rowwise(_dev(W, "W"), _dev(delta, "delta"), R, C, _dev(Q, "Q"), _stream(stream)),
           "qat4_lsq_fwd_rowwise")
    return Q


def lsq_bwd_rowwise(W, delta, G, grad_scale=None, grad_W=None, grad_delta=None, stream=None):
    import torch
    L = lib()
    _dev(W, "W", torch.float32)
    R, C = W.shape
    _dev(delta, "delta", torch.float32, (R,))
    _dev(G, "G", None, (R, C))
    gs = rowwise_grad_scale(C) if grad_scale is None else grad_scale
    grad_W = _out(grad_W, "grad_W", (R, C), torch.float32, W)
    grad_delta = _out(grad_delta, "grad_delta", (R,), torch.float32, W)
    _check(L.qat4_lsq_bwd_rowwise(_dev(W, "W"), _dev(delta, "delta"), _dev(G, "G"), _gdtype(G), R, C,
                                  ct.c_float(gs), _dev(grad_W, "grad_W"), _dev(grad_delta, "grad_delta"),
                                  _stream(stream)), "qat4_lsq_bwd_rowwise")
    return grad_W, grad_delta


def lsq_fwd_bwd_rowwise(W, delta, G, grad_scale=None, Q=None, grad_W=None, grad_delta=None, stream=None):
    import torch
    L = lib()
    _dev(W, "W", torch.float32)
    R, C = W.shape
    _dev(delta, "delta", torch.float32, (R,))
    _dev(G, "G", None, (R, C))
    gs = rowwise_grad_scale(C) if grad_scale is None else grad_scale
    Q = _out(Q, "Q", (R, C), torch.float32, W)
    grad_W = _out(grad_W, "grad_W", (R, C), torch.float32, W)
    grad_delta = _out(grad_delta, "grad_delta", (R,), torch.float32, W)
    _check(L.qat4_lsq_fwd_bwd_rowwise(_dev(W, "W"), _dev(delta, "delta"), _dev(G, "G"), _gdtype(G), R, C,
                                      ct.c_float(gs), _dev(Q, "Q"), _dev(grad_W, "grad_W"),
                                      _dev(grad_delta, "grad_delta"), _stream(stream)), "qat4_lsq_fwd_bwd_rowwise")
    return Q, grad_W, grad_delta


def pack_w4a16_rowwise(W, delta, packed=None, scales=None, stream=None):
    """Returns (packed uint8 [R, C/2], scales float16 [R])."""
    import torch
    L = lib()
    _dev(W, "W", torch.float32)
    R, C = W.shape
    _dev(delta, "delta", torch.float32, (R,))
    packed = _out(packed, "packed", (R, C // 2), torch.uint8, W)
    scales = _out(scales, "scales", (R,), torch.float16, W)
    _check(L.qat4_pack_w4a16_rowwise(_dev(W, "W"), _dev(delta, "delta"), R, C, _dev(packed, "packed"),
                                     _dev(scales, "scales"), _stream(stream)), "qat4_pack_w4a16_rowwise")
    return packed, scales


def scale_search_rowwise(W, H, alpha, delta=None, idx=None, best_err=None, workspace=None, stream=None):
    """Per-channel search with the full H.  Returns (delta f32 [R], idx i32 [R], best_err f32 [R])."""
    import torch
    L = lib()
    _dev(W, "W", torch.float32)
    R, C = W.shape
    _dev(H, "H", torch.float32)
    if H.dim() != 2 or H.shape[0] < C or H.shape[1] < C:
        raise ValueError("H must be at least [C, C]")
    _dev(alpha, "alpha", torch.float32)
    delta = _out(delta, "delta", (R,), torch.float32, W)
    idx = _out(idx, "idx", (R,), torch.int32, W)
    best_err = _out(best_err, "best_err", (R,), torch.float32, W)
    need = int(L.qat4_scale_search_rowwise_workspace_bytes(R, C))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=W.device)
    _check(L.qat4_scale_search_rowwise(_dev(W, "W"), R, C, _dev(H, "H"), H.shape[1], _dev(alpha, "alpha"),
                                       alpha.numel(), _dev(delta, "delta"), _dev(idx, "idx"),
                                       _dev(best_err, "best_err"), _dev(workspace, "workspace", torch.uint8),
                                       workspace.numel(), _stream(stream)), "qat4_scale_search_rowwise")
    return delta, idx, best_err


def w4a16_gemv(x, packed, scales, y=None, stream=None):
    """y [M, R] float32 = x @ (scale * code)^T on the packed export; x bf16 [M, C] (or [C]);
    scales float16 [R, C/group] (group-32 export) or [R] (per-row export)."""
    import torch
    L = lib()
    if x.dim() == 1:
        x = x.unsqueeze(0)
    _dev(x, "x", torch.bfloat16)
    M, C = x.shape
    _dev(packed, "packed", torch.uint8)
    R = packed.shape[0]
    if tuple(packed.shape) != (R, C // 2):
        raise ValueError("packed must be [R, C/2]")
    _dev(scales, "scales", torch.float16)
    G = scales.numel() // R
    if G < 1 or scales.numel() != R * G or C % G != 0:
        raise ValueError("scales must hold C/group values per row")
    y = _out(y, "y", (M, R), torch.float32, x)
    _check(L.qat4_w4a16_gemv(_dev(x, "x"), M, _dev(packed, "packed"), _dev(scales, "scales"), R, C, C // G,
                             _dev(y, "y"), _stream(stream)), "qat4_w4a16_gemv")
    return y


def fq_gemm(X, W, delta, Y=None, stream=None, fused=False, workspace=None):
    """Y [T, R] float32 = X @ bf16(Q_delta(W))^T; X bf16 [T, C], W float32 [R, C], delta float32
    [R, C/32].  By default the staged call (the quantizer writes bf16 Q into `workspace`, allocated
    here when None, then a tcgen05 GEMM); fused=True runs the single kernel with the quantizer in
    the GEMM's producer (no workspace)."""
    import torch
    L = lib()
    _dev(X, "X", torch.bfloat16)
    T, C = X.shape
    _dev(W, "W", torch.float32)
    R = W.shape[0]
    if W.shape[1] != C:
        raise ValueError("W must be [R, C] with the C of X")
    _dev(delta, "delta", torch.float32, (R, C // 32))
    Y = _out(Y, "Y", (T, R), torch.float32, X)
    if fused:
        _check(L.qat4_fq_gemm(_dev(X, "X"), T, _dev(W, "W"), _dev(delta, "delta"), R, C, _dev(Y, "Y"),
                              _stream(stream)), "qat4_fq_gemm")
        return Y
    need = int(L.qat4_fq_gemm_staged_workspace_bytes(R, C))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    _check(L.qat4_fq_gemm_staged(_dev(X, "X"), T, _dev(W, "W"), _dev(delta, "delta"), R, C, _dev(Y, "Y"),
                                 _dev(workspace, "workspace"), workspace.numel(), _stream(stream)),
           "qat4_fq_gemm_staged")
    return Y


def refine(W, H, alpha, idx, sweeps=1, delta=None, obj=None, workspace=None, stream=None):
    """Full-objective coordinate descent over the groups of each row, starting from idx (int32
    [R, C/32], refined in place); returns (delta float32 [R, C/32], idx, obj float64 [R])."""
    import torch
    L = lib()
    _dev(W, "W", torch.float32)
    R, C = W.shape
    _dev(H, "H", torch.float32)
    _dev(alpha, "alpha", torch.float32)
    _dev(idx, "idx", torch.int32, (R, C // 32))
    delta = _out(delta, "delta", (R, C // 32), torch.float32, W)
    obj = _out(obj, "obj", (R,), torch.float64, W)
    need = L.qat4_refine_workspace_bytes(R, C)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    _check(L.qat4_refine(_dev(W, "W"), R, C, _dev(H, "H"), H.shape[1], _dev(alpha, "alpha"), alpha.numel(),
                         int(sweeps), _dev(idx, "idx"), _dev(delta, "delta"), _dev(obj, "obj"),
                         _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream)),
           "qat4_refine")
    return delta, idx, obj


def sync_check(stream=None):
    """Synchronise and raise Qat4Error(QAT4_ERR_TIMEOUT) if a kernel gave up a bounded wait."""
    _check(lib().qat4_sync_check(_stream(stream)), "qat4_sync_check")


def selftest_bounded_wait(limit_ns: int, stream=None) -> int:
    """Launch the bounded-wait self test; returns the status of the following sync_check."""
    L = lib()
    _check(L.qat4_selftest_bounded_wait(int(limit_ns), _stream(stream)), "qat4_selftest_bounded_wait")
    return int(L.qat4_sync_check(_stream(stream)))
