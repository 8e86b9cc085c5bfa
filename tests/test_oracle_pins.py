"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle (and its NumPy twin) against something other than
its own formula: hand-worked values (tests/golden), closed forms, invariants,
special cases that reduce to a textbook computation, and brute force on tiny
inputs.  No GPU is involved.
"""
import os

import numpy as np
import pytest

from oracle import twin
from int4_group_wise_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
f32 = np.float32
S_LSQ = float(f32(1.0 / np.sqrt(32 * 7)))


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _bits(a):
    return np.asarray(a, f32).view(np.uint32)


def _group_row(vals):
    """Pad a list of values to a multiple of 32 columns (one row)."""
    v = np.zeros(((len(vals) + 31) // 32) * 32, f32)
    v[:len(vals)] = vals
    return v[None, :]


# ----------------------------------------------------------------- quantizer

def test_codes_hand_values(oracle_mod):
    rows = _golden_rows("quantize_codes.txt")
    w = _group_row([float(r[0]) for r in rows])
    exp = np.array([int(r[1]) for r in rows], np.int8)
    delta = np.ones((1, w.shape[1] // 32), f32)
    got = oracle_mod.codes(w, delta)[0, :len(rows)]
    np.testing.assert_array_equal(got, exp)
    np.testing.assert_array_equal(twin.codes(w, 1.0)[0, :len(rows)].astype(np.int8), exp)
    # forward value with Delta = 1 equals the code
    np.testing.assert_array_equal(oracle_mod.lsq_fwd(w, delta)[0, :len(rows)], exp.astype(f32))


def test_fixed_points_on_grid(oracle_mod):
    """w = fl(Delta*q) is reproduced bit-exactly with code q, for every q in [-8, 7]."""
    rng = np.random.default_rng(1)
    R = 64
    deltas = (10.0 ** rng.uniform(-6, 2, size=R)).astype(f32)
    q = np.tile(np.arange(-8, 8, dtype=f32), 2)           # 32 codes per row
    W = (deltas[:, None] * q[None, :]).astype(f32)
    D = deltas[:, None]
    np.testing.assert_array_equal(oracle_mod.codes(W, D), np.broadcast_to(q, W.shape).astype(np.int8))
    np.testing.assert_array_equal(_bits(oracle_mod.lsq_fwd(W, D)), _bits(W))


def test_idempotent_and_odd(oracle_mod):
    rng = np.random.default_rng(2)
    W = rng.standard_normal((16, 256)).astype(f32)
    D = (np.abs(W).reshape(16, 8, 32).max(axis=2) / f32(7) * rng.uniform(0.4, 1.2, (16, 8))).astype(f32)
    Q = oracle_mod.lsq_fwd(W, D)
    np.testing.assert_array_equal(_bits(oracle_mod.lsq_fwd(Q, D)), _bits(Q))
    # odd symmetry wherever neither side reaches the asymmetric clamp (|round(v)| <= 7)
    v = W / np.repeat(D, 32, axis=1)
    ok = np.abs(np.rint(v)) <= 7
    Qn = oracle_mod.lsq_fwd(-W, D)
    np.testing.assert_array_equal(Qn[ok], -Q[ok])
    # zero maps to zero; an all-zero Delta maps everything to zero
    np.testing.assert_array_equal(oracle_mod.lsq_fwd(np.zeros_like(W), D), 0)
    np.testing.assert_array_equal(oracle_mod.lsq_fwd(np.zeros_like(W), np.zeros_like(D)), 0)
    c = oracle_mod.codes(W, D)
    assert c.min() >= -8 and c.max() <= 7


def test_twin_agrees_forward(oracle_mod):
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((8, 128)) * 0.02).astype(f32)
    D = (np.abs(W).reshape(8, 4, 32).max(axis=2) / f32(7) * f32(0.8)).astype(f32)
    D[0, 0] = 0  # all-zero-group convention applied to a non-zero group
    np.testing.assert_array_equal(_bits(oracle_mod.lsq_fwd(W, D)),
                                  _bits(twin.fake_quant(W, np.repeat(D, 32, axis=1))))


# --------------------------------------------------------------- LSQ backward

def test_lsq_hand_values(oracle_mod):
    rows = _golden_rows("lsq_grad_cases.txt")
    n = len(rows)
    v = _group_row([float(r[0]) for r in rows])
    exp_gw = np.array([float(r[1]) for r in rows], f32)
    exp_d = np.array([float(r[2]) for r in rows], np.float64)
    D = np.ones((1, v.shape[1] // 32), f32)
    G = np.zeros_like(v)
    G[0, :n] = 1.0
    gW, gD = oracle_mod.lsq_bwd(v, D, G, S_LSQ)
    np.testing.assert_array_equal(gW[0, :n], exp_gw)
    # grad_Delta of the (single) group = s * sum of the hand dQ/dDelta values
    assert n <= 32
    np.testing.assert_allclose(gD[0, 0], S_LSQ * exp_d.sum(), rtol=1e-12, atol=0)
    # element by element: put G = 1 on one element at a time
    for i in range(n):
        Gi = np.zeros_like(v)
        Gi[0, i] = 1.0
        _, gDi = oracle_mod.lsq_bwd(v, D, Gi, 1.0)
        assert gDi[0, 0] == exp_d[i], (rows[i], gDi[0, 0])


def test_lsq_step_gradient_identity(oracle_mod):
    """Inside the range, round(v) - v == (Q - w) / Delta: a second formula for the same value."""
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((8, 64)) * 0.02).astype(f32)
    D = (np.abs(W).reshape(8, 2, 32).max(axis=2) / f32(7)).astype(f32)
    Dfull = np.repeat(D, 32, axis=1)
    Q = oracle_mod.lsq_fwd(W, D)
    for r in range(8):
        for c in range(64):
            G = np.zeros_like(W)
            G[r, c] = 1.0
            _, gD = oracle_mod.lsq_bwd(W, D, G, 1.0)
            v = W[r, c] / Dfull[r, c]
            if -8 < v < 7:
                ref = (float(Q[r, c]) - float(W[r, c])) / float(Dfull[r, c])
                assert abs(gD[r, c // 32] - ref) <= 1e-6 * max(1.0, abs(ref))
            else:
                assert gD[r, c // 32] == (7.0 if v >= 7 else -8.0)


def test_lsq_bf16_grad_and_twin(oracle_mod):
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((6, 96)) * 0.02).astype(f32)
    D = (np.abs(W).reshape(6, 3, 32).max(axis=2) / f32(7) * f32(0.7)).astype(f32)
    Gf = (rng.standard_normal(W.shape) * 1e-3).astype(f32)
    Gb = inputs.f32_to_bf16_bits(Gf)
    Gw = inputs.bf16_bits_to_f32(Gb)
    gW1, gD1 = oracle_mod.lsq_bwd(W, D, Gb, S_LSQ)
    gW2, gD2 = oracle_mod.lsq_bwd(W, D, Gw, S_LSQ)
    np.testing.assert_array_equal(_bits(gW1), _bits(gW2))
    np.testing.assert_array_equal(gD1, gD2)
    gW3, gD3 = twin.lsq_bwd(W, D, Gw, S_LSQ)
    np.testing.assert_array_equal(_bits(gW1), _bits(gW3))
    np.testing.assert_allclose(gD1, gD3, rtol=1e-12, atol=1e-18)
    # clamped elements get zero weight gradient, the rest get G unchanged
    v = W / np.repeat(D, 32, axis=1)
    inside = (v >= -8) & (v <= 7)
    np.testing.assert_array_equal(gW1[inside], Gw[inside])
    assert np.all(gW1[~inside] == 0)
    assert (~inside).any()


# ------------------------------------------------------------------- Hessian

def _bf16(x):
    return inputs.f32_to_bf16_bits(np.asarray(x, f32))


def test_hessian_hand_2x2(oracle_mod):
    # X = [[1, 2], [3, 4]]: X^T X = [[10, 14], [14, 20]], n = 2 -> [[5, 7], [7, 10]]
    H = oracle_mod.hessian(_bf16([[1, 2], [3, 4]]))
    np.testing.assert_array_equal(H, [[5.0, 7.0], [7.0, 10.0]])


def test_hessian_quadratic_form_and_diag(oracle_mod):
    """v^T H v == ||X v||^2 / n (matvec, no X^T X) and diag(H) = column mean squares."""
    rng = np.random.default_rng(6)
    n, C = 96, 40
    Xb = _bf16(rng.standard_normal((n, C)) * np.linspace(0.5, 3, C))
    X = inputs.bf16_bits_to_f32(Xb).astype(np.float64)
    H = oracle_mod.hessian(Xb)
    for _ in range(5):
        v = rng.standard_normal(C)
        lhs = v @ H @ v
        rhs = np.sum((X @ v) ** 2) / n
        assert abs(lhs - rhs) <= 1e-12 * rhs
    np.testing.assert_allclose(np.diag(H), (X * X).mean(axis=0), rtol=1e-14)
    np.testing.assert_array_equal(H, H.T)
    np.linalg.cholesky(H + 1e-9 * np.eye(C))    # positive semi-definite


def test_hessian_one_hot_rows_diagonal(oracle_mod):
    """Rows with a single non-zero a_t in column c_t give H = diag(sum_t a_t^2 [c_t = i]) / n."""
    rng = np.random.default_rng(7)
    n, C = 64, 32
    cols = rng.integers(0, C, n)
    a = rng.choice([-2.0, -1.0, 0.5, 1.0, 3.0], n)
    X = np.zeros((n, C), f32)
    X[np.arange(n), cols] = a
    H = oracle_mod.hessian(_bf16(X))
    exp = np.zeros((C, C))
    for t in range(n):
        exp[cols[t], cols[t]] += a[t] ** 2
    np.testing.assert_array_equal(H, exp / n)


def test_hessian_entries_and_block_consistent(oracle_mod):
    rng = np.random.default_rng(8)
    Xb = _bf16(rng.standard_normal((50, 64)))
    H = oracle_mod.hessian(Xb)
    ii = rng.integers(0, 64, 30)
    jj = rng.integers(0, 64, 30)
    np.testing.assert_array_equal(oracle_mod.hessian_entries(Xb, ii, jj), H[ii, jj])
    np.testing.assert_array_equal(oracle_mod.hessian_block(Xb, 32, 32, 0, 64), H[32:64, 0:64])


def test_hessian_blocks_closed_forms(oracle_mod):
    """The batched block call (used by the full-size GPU checks) against closed forms that do not
    form X^T X: a bilinear form u^T H_blk v = (X_r u) . (X_c v) / n from two matrix-vector
    products, the one-hot diagonal case, and the hand 2x2 case inside a larger matrix."""
    rng = np.random.default_rng(9)
    n, C = 300, 192
    Xb = _bf16(rng.standard_normal((n, C)) * np.linspace(0.3, 4, C))
    X = inputs.bf16_bits_to_f32(Xb).astype(np.float64)
    r0 = [0, 32, 160, 96]
    c0 = [64, 32, 0, 128]
    blocks = oracle_mod.hessian_blocks(Xb, r0, c0, 32)
    for b, r, c in zip(blocks, r0, c0):
        for _ in range(3):
            u, v = rng.standard_normal(32), rng.standard_normal(32)
            lhs = u @ b @ v
            rhs = (X[:, r:r + 32] @ u) @ (X[:, c:c + 32] @ v) / n
            assert abs(lhs - rhs) <= 1e-12 * (np.abs(X[:, r:r + 32] @ np.abs(u)) @ np.abs(X[:, c:c + 32] @ np.abs(v)) / n)
    # one-hot rows: every off-diagonal block is exactly zero, diagonal blocks are diag(sum a_t^2)/n
    cols = rng.integers(0, C, 64)
    a = rng.choice([-2.0, 0.5, 1.0, 3.0], 64)
    Xo = np.zeros((64, C), f32)
    Xo[np.arange(64), cols] = a
    bo = oracle_mod.hessian_blocks(_bf16(Xo), [0, 64, 32], [32, 64, 160], 32)
    assert not bo[0].any() and not bo[2].any()
    exp = np.zeros(C)
    np.add.at(exp, cols, a ** 2)
    np.testing.assert_array_equal(bo[1], np.diag(exp[64:96] / 64))
    # hand 2x2 case [[1, 2], [3, 4]] placed in columns 40, 41 of zeros: H[40:42, 40:42] = [[5, 7], [7, 10]]
    Xh = np.zeros((2, 96), f32)
    Xh[:, 40:42] = [[1, 2], [3, 4]]
    bh = oracle_mod.hessian_blocks(_bf16(Xh), [32], [32], 32)[0]
    np.testing.assert_array_equal(bh[8:10, 8:10], [[5.0, 7.0], [7.0, 10.0]])


# --------------------------------------------------------------- scale search

def _integer_calibration(rng, n, C):
    """Small-integer X with n a power of two: H = X^T X / n is exact in float32."""
    X = rng.integers(-3, 4, size=(n, C)).astype(f32)
    return X, _bf16(X)


def test_search_objective_equals_output_error_from_X(oracle_mod):
    """E_k = e H_gg e^T equals ||e X_g^T||^2 / n computed from X directly (model-card objective).

    Two groups with different statistics, so a wrong block index or a transposed block fails.
    """
    rng = np.random.default_rng(9)
    n, C, R = 64, 64, 5
    X, Xb = _integer_calibration(rng, n, C)
    X[:, 32:] *= 2        # second group's block differs from the first
    X[:, 5] += X[:, 7]    # correlated columns: non-trivial off-diagonals
    Xb = _bf16(X)
    H64 = oracle_mod.hessian(Xb)
    H = H64.astype(f32)
    assert np.array_equal(H.astype(np.float64), H64)   # exact in float32
    W = (rng.standard_normal((R, C)) * 0.02).astype(f32)
    alpha = inputs.alpha_grid(0.5, 0.05, 11)
    delta, idx, best, allE = oracle_mod.scale_search(W, H, alpha, all_err=True)
    Xd = X.astype(np.float64)
    for r in range(R):
        for g in range(2):
            w = W[r, 32 * g:32 * g + 32]
            m = np.abs(w).max()
            for k in range(alpha.size):
                dk = f32(alpha[k] * f32(m / f32(7)))
                e = w.astype(np.float64) - twin.fake_quant(w, dk).astype(np.float64)
                direct = np.sum((Xd[:, 32 * g:32 * g + 32] @ e) ** 2) / n
                assert abs(allE[r, g, k] - direct) <= 1e-12 * direct
            assert idx[r, g] == int(np.argmin(allE[r, g]))
            assert best[r, g] == allE[r, g].min()


def test_search_identity_hessian_is_mse(oracle_mod):
    """H = I reduces the search to plain squared error over the grid."""
    rng = np.random.default_rng(10)
    R, C = 6, 96
    W = (rng.standard_normal((R, C)) * 0.02).astype(f32)
    alpha = inputs.alpha_grid(0.5, 0.005, 101)
    delta, idx, best = oracle_mod.scale_search(W, np.eye(C, dtype=f32), alpha)
    for r in range(R):
        for g in range(C // 32):
            w = W[r, 32 * g:32 * g + 32]
            base = f32(np.abs(w).max() / f32(7))
            mse = []
            for a in alpha:
                d = f32(a * base)
                e = w.astype(np.float64) - twin.fake_quant(w, d).astype(np.float64)
                mse.append(float(e @ e))
            k = int(np.argmin(mse))
            assert idx[r, g] == k
            assert delta[r, g] == f32(alpha[k] * base)
            assert abs(best[r, g] - min(mse)) <= 1e-12 * min(mse)


def test_search_single_candidate_is_rtn(oracle_mod):
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((4, 64)) * 0.02).astype(f32)
    H = np.eye(64, dtype=f32) * f32(3)
    delta, idx, _ = oracle_mod.scale_search(W, H, np.array([1.0], f32))
    rtn = (np.abs(W).reshape(4, 2, 32).max(axis=2) / f32(7)).astype(f32)
    np.testing.assert_array_equal(_bits(delta), _bits(rtn))
    assert np.all(idx == 0)
    # every |w| equal: codes are +-7 at the RTN scale
    Weq = np.sign(W).astype(f32) * f32(0.013)
    d_eq, _, _ = oracle_mod.scale_search(Weq, H, np.array([1.0], f32))
    c = oracle_mod.codes(Weq, d_eq)
    assert set(np.unique(np.abs(c))) == {7}


def test_search_on_grid_weights_pick_exact_candidate(oracle_mod):
    """Weights that lie on the alpha=1 grid (power-of-two step) have zero error there."""
    rng = np.random.default_rng(12)
    R, C = 8, 64
    step = f32(2.0 ** -7)
    q = rng.integers(-6, 7, size=(R, C)).astype(f32)
    q[:, 0] = 7
    q[:, 32] = -7                                        # max |code| = 7 in each group
    W = (step * q).astype(f32)
    X, Xb = _integer_calibration(rng, 32, C)
    H = oracle_mod.hessian(Xb).astype(f32) + np.eye(C, dtype=f32)
    alpha = inputs.alpha_grid(0.5, 0.005, 101)
    delta, idx, best = oracle_mod.scale_search(W, H, alpha)
    assert np.all(idx == 100) and np.all(best == 0.0)
    assert np.all(delta == step)


def test_search_rtn_never_better_and_scale_covariance(oracle_mod):
    rng = np.random.default_rng(13)
    R, C = 16, 128
    W = inputs.student_t((R, C), 3.0, 0.01, seed=0, cfg=99, name="t")
    Xb = inputs.activations(256, C, seed=0, cfg=99, name="x", outliers=3)
    H = oracle_mod.hessian(Xb).astype(f32)
    alpha = inputs.alpha_grid(0.3, 0.0035, 201)
    assert alpha[-1] == f32(1.0)
    delta, idx, best, allE = oracle_mod.scale_search(W, H, alpha, all_err=True)
    assert np.all(best <= allE[:, :, -1])
    # doubling W (exact in binary) doubles Delta, keeps the index, quadruples the error
    d2, i2, b2 = oracle_mod.scale_search((W * f32(2)).astype(f32), H, alpha)
    np.testing.assert_array_equal(i2, idx)
    np.testing.assert_array_equal(d2, delta * f32(2))
    np.testing.assert_allclose(b2, 4 * best, rtol=1e-12)
    # whole-group permutation permutes outputs
    perm = [2, 0, 3, 1]
    cols = np.concatenate([np.arange(32 * p, 32 * p + 32) for p in perm])
    d3, i3, b3 = oracle_mod.scale_search(W[:, cols], H[np.ix_(cols, cols)], alpha)
    np.testing.assert_array_equal(i3, idx[:, perm])
    np.testing.assert_array_equal(d3, delta[:, perm])
    # a change inside group 1 alters only group 1's outputs
    W4 = W.copy()
    W4[:, 40] *= f32(1.5)
    d4, i4, _ = oracle_mod.scale_search(W4, H, alpha)
    keep = [0, 2, 3]
    np.testing.assert_array_equal(d4[:, keep], delta[:, keep])


def test_search_error_is_exact_difference(oracle_mod):
    """Heavily clipped weights (|w| > 2|Q|) make the binary32 difference w - Q inexact; the
    objective uses the exact difference (model-card objective on W - Q_Delta(W))."""
    w = np.zeros((1, 32), f32)
    w[0, 0] = f32(1.0)                         # sets the scale: base = fl(1/7)
    w[0, 1] = f32(0.3333333432674408)          # moderate weight
    w[0, 2] = f32(-1.0)
    alpha = np.array([0.1], f32)               # Delta = 0.1/7: both +-1 clip at codes 7 / -8
    H = np.eye(32, dtype=f32)
    d, i, best, allE = oracle_mod.scale_search(w, H, alpha, all_err=True)
    dk = f32(alpha[0] * f32(w[0, 0] / f32(7)))
    Q = twin.fake_quant(w[0], dk)
    e_exact = w[0].astype(np.float64) - Q.astype(np.float64)
    assert allE[0, 0, 0] == float(e_exact @ e_exact)
    e_f32 = (w[0] - Q).astype(np.float64)      # binary32 difference, rounded where clipped
    assert float(e_f32 @ e_f32) != float(e_exact @ e_exact)


def test_search_zero_group_and_twin(oracle_mod):
    rng = np.random.default_rng(14)
    R, C = 5, 64
    W = (rng.standard_normal((R, C)) * 0.02).astype(f32)
    W[2, 32:64] = 0
    X, Xb = _integer_calibration(rng, 64, C)
    H = oracle_mod.hessian(Xb).astype(f32)
    alpha = inputs.alpha_grid(0.5, 0.005, 101)
    d, i, b = oracle_mod.scale_search(W, H, alpha)
    assert d[2, 1] == 0 and i[2, 1] == 0 and b[2, 1] == 0
    dt, it, bt, _ = twin.search(W, H, alpha)
    np.testing.assert_array_equal(i, it)
    np.testing.assert_array_equal(d, dt)
    np.testing.assert_allclose(b, bt, rtol=1e-12)


# ---------------------------------------------------------------------- pack

def test_pack_hand_bytes(oracle_mod):
    rows = _golden_rows("pack_bytes.txt")
    codes = np.array([int(x) for x in rows[0]], f32)[None, :]
    exp = np.array([int(x, 16) for x in rows[1]], np.uint8)
    packed, s16 = oracle_mod.pack_w4a16(codes, np.ones((1, 1), f32))
    np.testing.assert_array_equal(packed[0], exp)
    assert s16[0, 0] == np.float16(1.0).view(np.uint16)
    np.testing.assert_array_equal(twin.pack(codes, np.ones((1, 1), f32))[0][0], exp)


def test_pack_unpack_roundtrip_and_fp16(oracle_mod):
    rng = np.random.default_rng(15)
    R, C = 12, 256
    W = (rng.standard_normal((R, C)) * 0.02).astype(f32)
    D = (np.abs(W).reshape(R, 8, 32).max(axis=2) / f32(7) * rng.uniform(0.5, 1.0, (R, 8))).astype(f32)
    D[0, 0] = 0
    D[1, 1] = f32(70000.0)   # overflows binary16 -> inf
    D[1, 2] = f32(1e-8)      # binary16 subnormal range
    packed, s16 = oracle_mod.pack_w4a16(W, D)
    lo = (packed & 0xF).astype(np.int16)
    hi = (packed >> 4).astype(np.int16)
    un = np.empty((R, C), np.int16)
    un[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    un[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    np.testing.assert_array_equal(un, oracle_mod.codes(W, D))
    with np.errstate(over="ignore"):
        s16_ref = D.astype(np.float16).view(np.uint16)   # NumPy's RNE conversion
    np.testing.assert_array_equal(s16, s16_ref)
    p2, s2 = twin.pack(W, D)
    np.testing.assert_array_equal(packed, p2)
    np.testing.assert_array_equal(s16, s2)


# ------------------------------------------------------------ per-channel variant

def test_rowwise_lsq_hand_row(oracle_mod):
    """One 64-weight row with the hand cases: grad_Delta = (sum of dQ/dDelta) / sqrt(64 * 7)."""
    cases = _golden_rows("lsq_grad_cases.txt")
    C, total = (int(x) if i == 0 else float(x) for i, x in enumerate(_golden_rows("lsq_grad_rowwise.txt")[0]))
    v = np.zeros((1, C), f32)
    v[0, :len(cases)] = [float(r[0]) for r in cases]
    G = np.ones_like(v)
    s = float(f32(1.0 / np.sqrt(C * 7)))
    gW, gD = oracle_mod.lsq_bwd_rowwise(v, np.ones(1, f32), G, s)
    assert abs(gD[0] - s * total) <= 1e-12 * abs(s * total)
    np.testing.assert_array_equal(gW[0, :len(cases)], [float(r[1]) for r in cases])


def test_rowwise_equals_group32_with_broadcast_scale(oracle_mod):
    """A per-row scale broadcast to every group of the row reproduces the group-32 functions."""
    rng = np.random.default_rng(21)
    R, C = 9, 32 * 11
    W = (rng.standard_normal((R, C)) * 0.02).astype(f32)
    Dr = (np.abs(W).max(axis=1) / f32(7) * rng.uniform(0.4, 1.1, R)).astype(f32)
    Dr[3] = 0                                   # Delta = 0 convention
    Dg = np.repeat(Dr[:, None], C // 32, axis=1)
    Gb = inputs.f32_to_bf16_bits((rng.standard_normal((R, C)) * 1e-3).astype(f32))
    np.testing.assert_array_equal(_bits(oracle_mod.lsq_fwd_rowwise(W, Dr)), _bits(oracle_mod.lsq_fwd(W, Dg)))
    s_row, s_grp = float(f32(1 / np.sqrt(C * 7))), float(f32(1 / np.sqrt(32 * 7)))
    gWr, gDr = oracle_mod.lsq_bwd_rowwise(W, Dr, Gb, s_row)
    gWg, gDg = oracle_mod.lsq_bwd(W, Dg, Gb, s_grp)
    np.testing.assert_array_equal(_bits(gWr), _bits(gWg))
    np.testing.assert_allclose(gDr / s_row, (gDg / s_grp).sum(axis=1), rtol=1e-12, atol=1e-300)
    pr, sr = oracle_mod.pack_w4a16_rowwise(W, Dr)
    pg, sg = oracle_mod.pack_w4a16(W, Dg)
    np.testing.assert_array_equal(pr, pg)
    np.testing.assert_array_equal(sr, sg[:, 0])
    with np.errstate(over="ignore"):
        np.testing.assert_array_equal(sr, Dr.astype(np.float16).view(np.uint16))


def test_rowwise_single_group_row_is_group32(oracle_mod):
    rng = np.random.default_rng(22)
    W = (rng.standard_normal((7, 32)) * 0.02).astype(f32)
    D = (np.abs(W).max(axis=1) / f32(7)).astype(f32)
    G = (rng.standard_normal((7, 32)) * 1e-3).astype(f32)
    gWr, gDr = oracle_mod.lsq_bwd_rowwise(W, D, G, S_LSQ)
    gWg, gDg = oracle_mod.lsq_bwd(W, D[:, None], G, S_LSQ)
    np.testing.assert_array_equal(gDr, gDg[:, 0])
    np.testing.assert_array_equal(_bits(gWr), _bits(gWg))


def test_rowwise_search_pins(oracle_mod):
    rng = np.random.default_rng(23)
    alpha = inputs.alpha_grid(0.5, 0.01, 51)
    # a one-group row is the group-32 search
    W1 = (rng.standard_normal((6, 32)) * 0.02).astype(f32)
    X1, X1b = _integer_calibration(rng, 64, 32)
    H1 = oracle_mod.hessian(X1b).astype(f32)
    d_r, i_r, b_r = oracle_mod.scale_search_rowwise(W1, H1, alpha)
    d_g, i_g, b_g = oracle_mod.scale_search(W1, H1, alpha)
    np.testing.assert_array_equal(i_r, i_g[:, 0])
    np.testing.assert_array_equal(d_r, d_g[:, 0])
    np.testing.assert_allclose(b_r, b_g[:, 0], rtol=1e-12)
    # objective from X directly over the whole row (cross-group terms included)
    R, C, n = 4, 96, 64
    X, Xb = _integer_calibration(rng, n, C)
    X[:, 40] += X[:, 70]                      # couples two groups
    Xb = _bf16(X)
    H = oracle_mod.hessian(Xb).astype(f32)
    W = (rng.standard_normal((R, C)) * 0.02).astype(f32)
    d, i, b, allE = oracle_mod.scale_search_rowwise(W, H, alpha, all_err=True)
    Xd = X.astype(np.float64)
    for r in range(R):
        base = f32(np.abs(W[r]).max() / f32(7))
        for k in range(0, alpha.size, 5):
            dk = f32(alpha[k] * base)
            e = W[r].astype(np.float64) - twin.fake_quant(W[r], dk).astype(np.float64)
            direct = np.sum((Xd @ e) ** 2) / n
            assert abs(allE[r, k] - direct) <= 1e-12 * direct
        assert i[r] == int(np.argmin(allE[r]))
    # H = I: plain squared error over the row
    d0, i0, b0 = oracle_mod.scale_search_rowwise(W, np.eye(C, dtype=f32), alpha)
    for r in range(R):
        base = f32(np.abs(W[r]).max() / f32(7))
        mse = [float(np.sum((W[r].astype(np.float64) - twin.fake_quant(W[r], f32(a * base)).astype(np.float64)) ** 2))
               for a in alpha]
        assert i0[r] == int(np.argmin(mse))
    # weights on the alpha = 1 grid (power-of-two step) pick alpha = 1 with zero error
    q = rng.integers(-6, 7, size=(3, 64)).astype(f32)
    q[:, 5] = 7
    Wg = (f32(2.0 ** -8) * q).astype(f32)
    dg, ig, bg = oracle_mod.scale_search_rowwise(Wg, np.eye(64, dtype=f32) + f32(0.25), alpha)
    assert np.all(ig == alpha.size - 1) and np.all(bg == 0) and np.all(dg == f32(2.0 ** -8))


# ------------------------------------------------------------- W4A16 inference GEMV

def test_w4a16_gemv_hand_row(oracle_mod):
    rows = _golden_rows("w4a16_gemv.txt")
    packed = np.array([[int(b, 16) for b in rows[0]]], np.uint8)
    scale = np.array([[np.float16(float(rows[1][0])).view(np.uint16)]], np.uint16)
    x = inputs.f32_to_bf16_bits(np.arange(1, 33, dtype=f32)[None, :])
    y = oracle_mod.w4a16_gemv(x, packed, scale, 32)
    assert y.shape == (1, 1) and y[0, 0] == float(rows[2][0])


def test_w4a16_gemv_export_roundtrip_and_linearity(oracle_mod):
    """Weights already on the exported grid (binary16-exact scale times a code) pack and
    multiply back to x W^T exactly; the product is linear in x; both scale layouts agree."""
    rng = np.random.default_rng(31)
    R, C, M = 6, 128, 3
    scale = rng.uniform(0.01, 0.05, (R, C // 32)).astype(np.float16).astype(f32)
    codes = rng.integers(-8, 8, (R, C)).astype(f32)
    W = (np.repeat(scale, 32, axis=1) * codes).astype(f32)          # exact
    packed, s16 = oracle_mod.pack_w4a16(W, scale)
    xf = inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(rng.standard_normal((M, C)).astype(f32)))
    xb = inputs.f32_to_bf16_bits(xf)
    y = oracle_mod.w4a16_gemv(xb, packed, s16, 32)
    np.testing.assert_allclose(y, xf.astype(np.float64) @ W.astype(np.float64).T, rtol=1e-13, atol=1e-13)
    y2 = oracle_mod.w4a16_gemv(inputs.f32_to_bf16_bits(2 * xf), packed, s16, 32)
    np.testing.assert_array_equal(y2, 2 * y)
    # per-channel scales (group = C) through the row-wise export
    rs = scale[:, 0]
    Wr = (rs[:, None] * codes).astype(f32)
    pr, sr = oracle_mod.pack_w4a16_rowwise(Wr, rs)
    yr = oracle_mod.w4a16_gemv(xb, pr, sr, C)
    np.testing.assert_allclose(yr, xf.astype(np.float64) @ Wr.astype(np.float64).T, rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------- fake-quant forward GEMM
def _golden_fq():
    rows = []
    for ln in open(os.path.join(GOLDEN, "fq_gemm_operand.txt")).read().splitlines():
        if ln.strip() and not ln.startswith("#"):
            rows.append([float.fromhex(v) for v in ln.split()])
    return rows


def test_fq_gemm_golden_bf16_operand(oracle_mod):
    """Hand-worked bf16 roundings of Q (ties to even, clamp, zero group): one weight per row,
    x = 2 on that column, so Y = 2 * Qb exactly."""
    rows = _golden_fq()
    R, C = len(rows), 32
    W = np.zeros((R, C), np.float32)
    D = np.zeros((R, 1), np.float32)
    for r, (w, d, _) in enumerate(rows):
        W[r, r % C] = w
        D[r, 0] = d
    X = np.zeros((1, C), np.float32)
    X[0, :R] = 2.0
    Y = oracle_mod.fq_gemm(inputs.f32_to_bf16_bits(X), W, D)
    np.testing.assert_array_equal(Y[0], [2.0 * e for _, _, e in rows])


def test_fq_gemm_equals_export_product_on_exact_grids(oracle_mod):
    """With power-of-two scales, fl(Delta*q) is a bf16 and a binary16 value, so the fake-quant
    forward and the W4A16 product of the packed export are the same sum in the same order:
    bitwise equal, although one goes through the LSQ forward and the other through packing and
    nibble decoding."""
    rng = np.random.default_rng(11)
    T, R, C = 3, 7, 96
    D = (2.0 ** -rng.integers(4, 9, (R, C // 32))).astype(np.float32)
    W = (rng.standard_normal((R, C)) * 0.1).astype(np.float32)
    Xb = inputs.f32_to_bf16_bits(rng.standard_normal((T, C)).astype(np.float32))
    Y = oracle_mod.fq_gemm(Xb, W, D)
    packed, scales = oracle_mod.pack_w4a16(W, D)
    Yg = oracle_mod.w4a16_gemv(Xb, packed, scales, 32)
    np.testing.assert_array_equal(Y, Yg)
    assert np.count_nonzero(Y) == Y.size


def test_fq_gemm_twin_and_entries(oracle_mod):
    """The C oracle against the NumPy twin (own fake-quant, own bf16 rounding, BLAS product), and
    its sampled-entry form against the full product (same sum order: bitwise)."""
    rng = np.random.default_rng(12)
    T, R, C = 5, 9, 64
    W = (rng.standard_normal((R, C)) * 0.05).astype(np.float32)
    D = (np.abs(W).reshape(R, C // 32, 32).max(axis=2) / 7 * rng.uniform(0.5, 1.0, (R, C // 32))).astype(np.float32)
    Xb = inputs.f32_to_bf16_bits(rng.standard_normal((T, C)).astype(np.float32))
    Y = oracle_mod.fq_gemm(Xb, W, D)
    Yt = twin.fq_gemm(inputs.bf16_bits_to_f32(Xb), W, D)
    np.testing.assert_allclose(Y, Yt, rtol=1e-12, atol=1e-15)
    tt = rng.integers(0, T, 20)
    rr = rng.integers(0, R, 20)
    np.testing.assert_array_equal(oracle_mod.fq_gemm_entries(Xb, W, D, tt, rr), Y[tt, rr])


# --------------------------------------------------------- full-objective refinement
def _refine_problem(R, C, K, seed, coupled=True):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((R, C)) * 0.02).astype(np.float32)
    if coupled:
        X = rng.standard_normal((4 * C, C)).astype(np.float32)
        X[:, :C // 2] += X[:, C // 2:]                      # correlate channels across groups
        H = (X.astype(np.float64).T @ X / X.shape[0]).astype(np.float32)
    else:
        H = np.zeros((C, C), np.float32)
        for g in range(C // 32):
            B = rng.standard_normal((64, 32))
            H[32 * g:32 * g + 32, 32 * g:32 * g + 32] = (B.T @ B / 64).astype(np.float32)
    alpha = inputs.alpha_grid(0.5, 0.5 / (K - 1), K)
    return W, H, alpha


def test_refine_keeps_the_search_when_H_is_block_diagonal(oracle_mod):
    """Without cross-group blocks the full objective is the sum of the groups' own objectives,
    which the search already minimises group by group: no sweep changes anything, and the final
    objective is the sum of the search's per-group minima."""
    W, H, alpha = _refine_problem(8, 128, 11, seed=31, coupled=False)
    _, idx0, best, _ = oracle_mod.scale_search(W, H, alpha, all_err=True)
    _, idx, obj = oracle_mod.refine(W, H, alpha, idx0, sweeps=3)
    np.testing.assert_array_equal(idx, idx0)
    np.testing.assert_allclose(obj, best.sum(axis=1), rtol=1e-12)


def test_refine_agrees_with_twin(oracle_mod):
    W, H, alpha = _refine_problem(5, 128, 9, seed=32)
    _, idx0, _, _ = oracle_mod.scale_search(W, H, alpha, all_err=True)
    _, idx, obj = oracle_mod.refine(W, H, alpha, idx0, sweeps=2)
    idx_t, obj_t = twin.refine(W, H, alpha, idx0, 2)
    np.testing.assert_array_equal(idx, idx_t)
    np.testing.assert_allclose(obj, obj_t, rtol=1e-11)


def test_refine_descends_to_a_coordinate_minimum(oracle_mod):
    """From the search's scales, sweeps never raise the full objective, lower it where groups are
    coupled, and stop at a point where no single group can improve it (checked by brute force
    with the twin's objective)."""
    W, H, alpha = _refine_problem(6, 96, 7, seed=33)
    _, idx0, _, _ = oracle_mod.scale_search(W, H, alpha, all_err=True)
    _, _, obj0 = oracle_mod.refine(W, H, alpha, idx0, sweeps=0)
    _, idx, obj = oracle_mod.refine(W, H, alpha, idx0, sweeps=20)
    assert np.all(obj <= obj0 * (1 + 1e-12))
    assert np.any(obj < obj0 * (1 - 1e-6))
    Hd = H.astype(np.float64)
    for r in range(W.shape[0]):
        wg = W[r].reshape(-1, 32)
        base = (np.abs(wg).max(axis=1) / np.float32(7)).astype(np.float32)
        err = lambda g, k: wg[g].astype(np.float64) - twin.fake_quant(wg[g], (alpha[k] * base[g]).astype(np.float32))
        e = np.concatenate([err(g, idx[r, g]) for g in range(wg.shape[0])])
        E = e @ Hd @ e
        for g in range(wg.shape[0]):
            for k in range(alpha.size):
                e2 = e.copy()
                e2[32 * g:32 * g + 32] = err(g, k)
                assert e2 @ Hd @ e2 >= E * (1 - 1e-12)


def test_refine_replay_of_its_own_sweep(oracle_mod):
    W, H, alpha = _refine_problem(4, 128, 9, seed=34)
    _, idx0, _, _ = oracle_mod.scale_search(W, H, alpha, all_err=True)
    _, idx1, _ = oracle_mod.refine(W, H, alpha, idx0, sweeps=1)
    emin, epick = oracle_mod.refine_replay(W, H, alpha, idx0, idx1)
    np.testing.assert_array_equal(emin, epick)
    assert np.any(idx1 != idx0)
