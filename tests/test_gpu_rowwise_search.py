"""GPU parity of the per-channel (one scale per row) Hessian-weighted search
against the CPU oracle's full C x C quadratic form: idx exact outside
1e-6-relative near-ties, delta bit-exact where idx matches, best_err within
1e-4 relative of the oracle's objective at the chosen candidate."""
import numpy as np
import pytest
import torch

import int4_group_wise_b200 as q4
from int4_group_wise_b200 import inputs

pytestmark = pytest.mark.gpu
f32 = np.float32


def _check(W, H, alpha, oracle_mod, rows=None):
    d, i, e = q4.scale_search_rowwise(torch.from_numpy(W).cuda(), torch.from_numpy(H).cuda(),
                                      torch.from_numpy(alpha).cuda())
    q4.sync_check()
    d, i, e = d.cpu().numpy(), i.cpu().numpy(), e.cpu().numpy()
    if rows is not None:
        W, d, i, e = W[rows], d[rows], i[rows], e[rows]
    dr, ir, br, allE = oracle_mod.scale_search_rowwise(W, H, alpha, all_err=True)
    at = allE[np.arange(len(i)), i]
    same = i == ir
    assert np.all((at[~same] - br[~same]) <= 1e-6 * np.abs(br[~same])), (int((~same).sum()),)
    np.testing.assert_array_equal(d[same].view(np.uint32), dr[same].view(np.uint32))
    np.testing.assert_allclose(e.astype(np.float64), at, rtol=1e-4, atol=1e-30)
    return i


def _H(oracle_mod, n, C, seed, outliers=1):
    Xb = inputs.activations(n, C, seed=seed, cfg=80, name="X", outliers=outliers)
    return oracle_mod.hessian(Xb).astype(f32)


def test_rowwise_search_one_group_rows_equal_group32(oracle_mod):
    W = inputs.gaussian((40, 32), 0.02, seed=1, cfg=80, name="W")
    H = _H(oracle_mod, 128, 32, 1)
    alpha = inputs.alpha_grid(0.5, 0.005, 101)
    i_row = _check(W, H, alpha, oracle_mod)
    d_g, i_g, _ = q4.scale_search(torch.from_numpy(W).cuda(), torch.from_numpy(H).cuda(), torch.from_numpy(alpha).cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(i_row, i_g.cpu().numpy()[:, 0])


@pytest.mark.parametrize("R,C,K,kind", [(7, 96, 101, "grid"), (5, 160, 1, "one"), (9, 288, 17, "unsorted"),
                                        (3, 512, 101, "zero-row"), (6, 256, 51, "indefinite")])
def test_rowwise_search_small(R, C, K, kind, oracle_mod):
    W = inputs.student_t((R, C), 3.0, 0.01, seed=R, cfg=81, name="W")
    if kind == "one":
        alpha = np.array([1.0], f32)
    elif kind == "unsorted":
        alpha = np.random.default_rng(3).permutation(inputs.alpha_grid(0.3, 0.05, K)).astype(f32)
        alpha[0] = 0.0                                     # Delta = 0 candidate first
    else:
        alpha = inputs.alpha_grid(0.5, 0.5 / max(K - 1, 1), K)
    if kind == "zero-row":
        W[1] = 0
    if kind == "indefinite":
        A = np.random.default_rng(5).standard_normal((C, C)).astype(f32)
        H = ((A + A.T) * f32(0.5)).astype(f32)
    else:
        H = _H(oracle_mod, 256, C, R, outliers=2)
    _check(W, H, alpha, oracle_mod)


def test_rowwise_search_layer_shape_sampled(oracle_mod):
    """All 8192 rows of the 1B-class up-projection on the GPU; 24 sampled rows checked."""
    wl = inputs.workload(1)
    W = wl.weight(wl.matrices[0])
    Xb = wl.activations("x", n=4096)
    H = oracle_mod.hessian(Xb).astype(f32)
    rows = np.arange(0, W.shape[0], 8192 // 24)[:24]
    _check(W, H, wl.alpha(), oracle_mod, rows=rows)
