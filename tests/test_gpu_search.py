"""GPU parity of the Hessian-weighted scale search against the CPU oracle.

Tolerances: idx exact, except where the oracle's own objective at the GPU's
choice is within 1e-6 relative of the oracle's minimum (a near-tie); Delta
bit-exact wherever idx matches; best_err within 1e-4 relative of the
oracle's objective at the chosen candidate."""
import numpy as np
import pytest
import torch

import int4_group_wise_b200 as q4
from int4_group_wise_b200 import inputs

pytestmark = pytest.mark.gpu
f32 = np.float32


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def check_search(W, H, alpha, oracle_mod, rows=None):
    """Run the GPU search on all of W; compare the given rows (default all) with the oracle."""
    d, i, e = q4.scale_search(_dev(W), _dev(H), _dev(alpha))
    q4.sync_check()
    d, i, e = d.cpu().numpy(), i.cpu().numpy(), e.cpu().numpy()
    if rows is not None:
        W, d, i, e = W[rows], d[rows], i[rows], e[rows]
    dr, ir, br, allE = oracle_mod.scale_search(W, H, alpha, all_err=True)
    same = i == ir
    if not same.all():
        # near-ties only: the oracle's error at the GPU's pick is within 1e-6 of its minimum
        at_gpu = np.take_along_axis(allE, i[..., None].astype(np.int64), axis=2)[..., 0]
        rel = (at_gpu[~same] - br[~same]) / np.maximum(br[~same], 1e-300)
        assert np.all(rel <= 1e-6), (int((~same).sum()), float(rel.max()))
    np.testing.assert_array_equal(d[same].view(np.uint32), dr[same].view(np.uint32))
    at_gpu = np.take_along_axis(allE, i[..., None].astype(np.int64), axis=2)[..., 0]
    np.testing.assert_allclose(e.astype(np.float64), at_gpu, rtol=1e-4, atol=1e-30)
    return int((~same).sum())


def _hessian_fp32(oracle_mod, Xb):
    return oracle_mod.hessian(Xb).astype(f32)


@pytest.mark.parametrize("R,C,K,seed", [(1, 32, 101, 1), (3, 64, 1, 2), (5, 96, 3, 3), (130, 160, 101, 4),
                                        (129, 64, 201, 5), (7, 32 * 9, 17, 6)])
def test_search_small(R, C, K, seed, oracle_mod):
    rng = np.random.default_rng(seed)
    W = inputs.student_t((R, C), 3.0, 0.01, seed=seed, cfg=50, name="W")
    W[0, :32] = 0                                   # all-zero group
    if R > 2:
        W[2, :32] = np.sign(W[2, :32]) * f32(0.02)  # equal magnitudes
    Xb = inputs.activations(256, C, seed=seed, cfg=50, name="X", outliers=max(1, C // 64))
    H = _hessian_fp32(oracle_mod, Xb)
    alpha = inputs.alpha_grid(0.5, 0.5 / max(K - 1, 1), K) if K > 1 else np.array([1.0], f32)
    check_search(W, H, alpha, oracle_mod)


def test_search_identity_and_ongrid(oracle_mod):
    rng = np.random.default_rng(9)
    R, C = 64, 128
    W = (rng.standard_normal((R, C)) * 0.02).astype(f32)
    check_search(W, np.eye(C, dtype=f32), inputs.alpha_grid(0.5, 0.005, 101), oracle_mod)
    q = rng.integers(-6, 7, size=(R, C)).astype(f32)
    q[:, ::32] = 7
    Wg = (f32(2.0 ** -7) * q).astype(f32)
    d, i, e = q4.scale_search(_dev(Wg), _dev(np.eye(C, dtype=f32) * f32(2)), _dev(inputs.alpha_grid(0.5, 0.005, 101)))
    torch.cuda.synchronize()
    assert torch.all(i == 100) and torch.all(e == 0) and torch.all(d == f32(2.0 ** -7))


def test_search_exact_division_path(oracle_mod):
    """Weights at exact half-integer multiples of a power-of-two step land on rounding ties at
    alpha = 1 (the exact-division path), and alpha = 0 gives Delta = 0 (1/Delta not finite)."""
    rng = np.random.default_rng(11)
    R, C = 70, 96
    step = f32(2.0 ** -7)
    q = rng.integers(-7, 7, size=(R, C)).astype(f32) + f32(0.5)
    q[:, ::32] = 7.0                                   # max |w| = 7 steps: base = step exactly
    W = (step * q).astype(f32)
    X, Xb = None, inputs.activations(128, C, seed=3, cfg=51, name="X")
    H = oracle_mod.hessian(Xb).astype(f32)
    alpha = np.array([0.0, 0.5, 0.75, 1.0, 1.25], f32)
    check_search(W, H, alpha, oracle_mod)


def test_search_non_psd_and_padded_ldh(oracle_mod):
    """A symmetric indefinite H (kappa > 1) and a row stride larger than C."""
    rng = np.random.default_rng(10)
    R, C = 40, 64
    W = (rng.standard_normal((R, C)) * 0.02).astype(f32)
    A = rng.standard_normal((C, C)).astype(f32)
    H = ((A + A.T) * f32(0.5)).astype(f32)
    check_search(W, H, inputs.alpha_grid(0.5, 0.005, 101), oracle_mod)
    Hp = np.zeros((C, C + 12), f32)
    Hp[:, :C] = H
    d1, i1, e1 = q4.scale_search(_dev(W), _dev(H), _dev(inputs.alpha_grid(0.5, 0.005, 101)))
    d2, i2, e2 = q4.scale_search(_dev(W), _dev(Hp), _dev(inputs.alpha_grid(0.5, 0.005, 101)))
    torch.cuda.synchronize()
    assert torch.equal(i1, i2) and torch.equal(d1, d2) and torch.equal(e1, e2)


def _diag_block_hessian(cache, cfg, oracle_mod, x_name="x"):
    """H with the oracle's 32x32 diagonal blocks (all the search reads) and zeros elsewhere."""
    def make():
        wl = inputs.workload(cfg)
        Xb = cache.get(("X", cfg, x_name), lambda: wl.activations(x_name))
        C = Xb.shape[1]
        H = np.zeros((C, C), f32)
        for g in range(C // 32):
            H[32 * g:32 * g + 32, 32 * g:32 * g + 32] = oracle_mod.hessian_block(Xb, 32 * g, 32, 32 * g, 32)
        return H
    return cache.get(("Hdiag", cfg, x_name), make)


def test_search_config0_full(cache, oracle_mod):
    wl = inputs.workload(0)
    W = wl.weight(wl.matrices[0])
    Xb = cache.get(("X", 0, "x"), lambda: wl.activations("x"))
    H = _hessian_fp32(oracle_mod, Xb)
    check_search(W, H, wl.alpha(), oracle_mod)


@pytest.mark.parametrize("cfg", [1, 2])
def test_search_full_size_sampled_rows(cfg, cache, oracle_mod):
    """All rows run on the GPU; every 32nd row (all groups, all candidates) checked."""
    wl = inputs.workload(cfg)
    W = wl.weight(wl.matrices[0])
    H = _diag_block_hessian(cache, cfg, oracle_mod)
    rows = np.arange(0, W.shape[0], 32)
    check_search(W, H, wl.alpha(), oracle_mod, rows=rows)


def test_search_degenerate_blocks_rows_and_ties(oracle_mod):
    """Paths the tensor-core screen hands to the float64 re-score: a 32x32 block of H that is
    all zero (every candidate ties, so every row is re-scored over all K by its warp), rows whose
    weights are too small for the power-of-two row scale (|w| < 2^-100), and a grid with repeated
    multipliers (equal objectives: the smallest index wins)."""
    rng = np.random.default_rng(12)
    R, C = 200, 96
    W = (rng.standard_normal((R, C)) * 0.02).astype(f32)
    W[5, :] = (rng.standard_normal(C) * 1e-33).astype(f32)          # m ~ 2^-108
    W[77, 64:96] = (rng.standard_normal(32) * 1e-36).astype(f32)     # one tiny group, H_gg nonzero
    Xb = inputs.activations(256, C, seed=12, cfg=52, name="X", outliers=2)
    H = oracle_mod.hessian(Xb).astype(f32)
    H[32:64, 32:64] = 0.0                                            # group 1: H_gg = 0
    alpha = inputs.alpha_grid(0.5, 0.01, 51)
    check_search(W, H, alpha, oracle_mod)
    d, i, e = q4.scale_search(_dev(W), _dev(H), _dev(alpha))
    torch.cuda.synchronize()
    assert torch.all(i[:, 1] == 0) and torch.all(e[:, 1] == 0)       # zero block: all tie at k = 0
    rep = np.repeat(inputs.alpha_grid(0.6, 0.05, 9), 3).astype(f32)  # each multiplier three times
    _, i2, _ = q4.scale_search(_dev(W), _dev(H), _dev(rep))
    torch.cuda.synchronize()
    assert torch.all(i2 % 3 == 0)                                     # first of each equal triple
    check_search(W, H, rep, oracle_mod)


@pytest.mark.parametrize("spread,seed", [(8, 11), (14, 12), (20, 13)])
def test_search_widely_scaled_channels(spread, seed, oracle_mod):
    """Channel scales spread over 2^-spread/2 .. 2^spread/2 (and lognormal channels with a strongly
    correlated pair): the binary16 split of such blocks puts the small entries below binary16's
    normal range, so the kernel equilibrates them (H' = D^-1 H D^-1, e' = D e) before the screen.
    Every row and group against the oracle."""
    rng = np.random.default_rng(seed)
    R, C, n = 200, 128, 4096
    X = rng.standard_normal((n, C)).astype(f32)
    X *= (2.0 ** rng.uniform(-spread / 2, spread / 2, C)).astype(f32)
    X[:, 5] = X[:, 4] * f32(1e-3) + X[:, 5] * f32(1e-6)      # nearly collinear pair, very different scales
    Xb = inputs.f32_to_bf16_bits(X)
    H = _hessian_fp32(oracle_mod, Xb)
    W = inputs.gaussian((R, C), 0.02, seed=seed, cfg=51, name="W")
    W[1] *= f32(1e-20)                                          # tiny rows
    W[2, :32] = f32(0.02) * np.sign(W[2, :32])                 # equal magnitudes
    alpha = inputs.alpha_grid(0.3, 0.0035, 201)
    check_search(W, H, alpha, oracle_mod)
