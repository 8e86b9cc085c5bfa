"""Second, independent NumPy statement of the quantizer (tiny inputs only).

TEST INFRASTRUCTURE.  Written separately from ``qat4_oracle.c`` (vectorised
NumPy instead of C loops) so that the two can be checked against each other on
small cases.  Same readings of the pages as the C oracle:

* Q_Delta(w) = Delta * clamp(rint(w / Delta), -8, 7) in float32, Delta = 0 -> 0
  ("Opt.Gear-QAT" blog, section 1 and section 3; model card "Quantization
  Configuration", symmetric zero-point 0);
* per-group objective e H_gg e^T over Delta_k = alpha_k * (max|w| / 7) (model
  card objective, block-diagonal reading);
* LSQ gradients (blog section 3; Esser et al. 2020);
* the fake-quant forward product X @ bf16(Q)^T (blog section 3, bf16 operands,
  round to nearest even).
"""
from __future__ import annotations

import numpy as np

f32 = np.float32


def _v(w, d):
    w = np.asarray(w, f32)
    d = np.asarray(d, f32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(d == 0, f32(0), w / np.where(d == 0, f32(1), d))
    return v.astype(f32)


def codes(w, d):
    return np.clip(np.rint(_v(w, d)), f32(-8), f32(7)).astype(f32)


def fake_quant(w, d):
    return (np.asarray(d, f32) * codes(w, d)).astype(f32)


def search(W, H, alpha):
    """Exhaustive grid search; returns (delta, idx, best_err float64, all_err)."""
    W = np.asarray(W, f32)
    R, C = W.shape
    G = C // 32
    alpha = np.asarray(alpha, f32)
    K = alpha.size
    Wg = W.reshape(R, G, 32)
    m = np.abs(Wg).max(axis=2)                          # [R, G]
    base = (m / f32(7)).astype(f32)
    dk = (alpha[None, None, :] * base[:, :, None]).astype(f32)   # [R, G, K]
    q = fake_quant(Wg[:, :, None, :], dk[:, :, :, None])         # [R, G, K, 32]
    e = Wg[:, :, None, :].astype(np.float64) - q.astype(np.float64)     # exact difference
    Hb = np.stack([np.asarray(H, np.float64)[32 * g:32 * g + 32, 32 * g:32 * g + 32]
                   for g in range(G)])                           # [G, 32, 32]
    E = np.einsum("rgki,gij,rgkj->rgk", e, Hb, e)
    idx = np.argmin(E, axis=2).astype(np.int32)                  # first minimum
    best = np.take_along_axis(E, idx[:, :, None].astype(np.int64), axis=2)[:, :, 0]
    delta = np.take_along_axis(dk, idx[:, :, None].astype(np.int64), axis=2)[:, :, 0]
    return delta.astype(f32), idx, best, E


def lsq_bwd(W, delta, G, s):
    W = np.asarray(W, f32)
    R, C = W.shape
    d = np.repeat(np.asarray(delta, f32), 32, axis=1)
    v = _v(W, d)
    G = np.asarray(G, f32)
    gW = np.where((v >= -8) & (v <= 7), G, f32(0)).astype(f32)
    dq = np.where(v <= -8, f32(-8), np.where(v >= 7, f32(7), (np.rint(v) - v).astype(f32)))
    gD = float(s) * (G.astype(np.float64) * dq.astype(np.float64)).reshape(R, C // 32, 32).sum(axis=2)
    return gW, gD


def pack(W, delta):
    W = np.asarray(W, f32)
    R, C = W.shape
    q = codes(W, np.repeat(np.asarray(delta, f32), 32, axis=1)).astype(np.int8)
    nib = (q.astype(np.int16) & 0xF).astype(np.uint8)
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    with np.errstate(over="ignore"):
        s16 = np.asarray(delta, f32).astype(np.float16).view(np.uint16)
    return packed, s16


def _bf16_rne(a):
    """float32 -> float32 holding the nearest bf16 value (ties to even), by integer rounding of
    the bit pattern."""
    u = np.asarray(a, f32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(f32)


def fq_gemm(X, W, delta):
    """X float32 (bf16-valued) [T, C], W [R, C], delta [R, C/32] -> float64 [T, R]."""
    W = np.asarray(W, f32)
    D = np.repeat(np.asarray(delta, f32), 32, axis=1)
    Qb = _bf16_rne(fake_quant(W, D)).astype(np.float64)
    return np.asarray(X, np.float64) @ Qb.T


def refine(W, H, alpha, idx_start, sweeps):
    """Coordinate descent on the full objective e H e^T (groups in order, ties to the smallest k),
    every candidate's objective evaluated with a float64 matrix product."""
    W = np.asarray(W, f32)
    H = np.asarray(H, np.float64)
    alpha = np.asarray(alpha, f32)
    R, C = W.shape
    G = C // 32
    idx = np.array(idx_start, np.int32, copy=True)
    obj = np.empty(R)
    for r in range(R):
        wg = W[r].reshape(G, 32)
        base = (np.abs(wg).max(axis=1) / f32(7)).astype(f32)

        def err(g, k):
            return wg[g].astype(np.float64) - fake_quant(wg[g], (alpha[k] * base[g]).astype(f32)).astype(np.float64)

        e = np.concatenate([err(g, idx[r, g]) for g in range(G)])
        for _ in range(sweeps):
            for g in range(G):
                best_k, best = -1, 0.0
                for k in range(alpha.size):
                    e[32 * g:32 * g + 32] = err(g, k)
                    E = float(e @ H @ e)
                    if best_k < 0 or E < best:
                        best_k, best = k, E
                idx[r, g] = best_k
                e[32 * g:32 * g + 32] = err(g, best_k)
        obj[r] = float(e @ H @ e)
    return idx, obj
