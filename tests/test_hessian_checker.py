"""CPU test of the per-block Hessian checker used by the GPU parity tests: it
must accept the oracle's own H (rounded to float32, as the kernel stores it)
and reject an H in which one off-diagonal 256x256 tile (with its mirror) holds
the wrong values -- another tile's values, its own transpose, or a copy
shifted by 32 columns.  At full size (n = 262144, outlier channels near 400 on
the diagonal, off-diagonal entries near 2e-3) such a tile moves a Frobenius
ratio pooled over the diagonal blocks by less than 1e-3; judged block by block
it fails with an error near 1.  The planted mistakes are made in a NumPy copy
of the oracle's H; no GPU is involved."""
import numpy as np
import pytest

from int4_group_wise_b200 import inputs
from hessian_check import check_hessian, tile_blocks

T = 256


@pytest.fixture(scope="module")
def case(oracle_mod):
    n, C = 2048, 768                     # 3 x 3 tiles of 256, 6 of them upper-triangle
    Xb = inputs.activations(n, C, seed=11, cfg=64, name="Xcheck", outliers=8)
    H = oracle_mod.hessian(Xb).astype(np.float32)
    return Xb, H


def _set_tile(H, I, J, vals):
    H = H.copy()
    H[I * T:(I + 1) * T, J * T:(J + 1) * T] = vals
    H[J * T:(J + 1) * T, I * T:(I + 1) * T] = vals.T        # the mirror stays consistent
    return H


def test_every_upper_tile_is_sampled():
    C = 768
    starts = tile_blocks(C, np.random.default_rng(0))
    seen = {(r // T, c // T) for r, c in starts}
    assert seen == {(I, J) for I in range(3) for J in range(I, 3)}
    assert all(c >= r for r, c in starts)


def test_checker_accepts_the_oracles_own_hessian(case, oracle_mod):
    Xb, H = case
    assert check_hessian(H, Xb, oracle_mod, np.random.default_rng(1), n_random=8) <= 1e-6


@pytest.mark.parametrize("mistake", ["misplaced", "transposed", "shifted"])
def test_checker_rejects_a_wrong_tile(case, oracle_mod, mistake):
    Xb, H = case
    if mistake == "misplaced":          # tile (0, 2) receives tile (0, 1)'s values
        bad = _set_tile(H, 0, 2, H[0:T, T:2 * T])
    elif mistake == "transposed":       # tile (1, 2) stored transposed
        bad = _set_tile(H, 1, 2, H[T:2 * T, 2 * T:3 * T].T)
    else:                               # tile (0, 1) read 32 columns too far to the right
        bad = _set_tile(H, 0, 1, H[0:T, T + 32:2 * T + 32])
    with pytest.raises(AssertionError, match="blocks above"):
        check_hessian(bad, Xb, oracle_mod, np.random.default_rng(1), n_random=0)


def test_checker_tolerance_edges(case, oracle_mod):
    """A 1e-5 relative perturbation of one tile passes; 1e-2 fails."""
    Xb, H = case
    tile = H[0:T, 2 * T:3 * T].astype(np.float64)
    ok = _set_tile(H, 0, 2, (tile * (1 + 1e-5)).astype(np.float32))
    check_hessian(ok, Xb, oracle_mod, np.random.default_rng(1), n_random=0)
    bad = _set_tile(H, 0, 2, (tile * (1 + 1e-2)).astype(np.float32))
    with pytest.raises(AssertionError):
        check_hessian(bad, Xb, oracle_mod, np.random.default_rng(1), n_random=0)
