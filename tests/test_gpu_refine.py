"""GPU parity of the full-objective refinement (coordinate descent over the groups of each row)
against the binary64 oracle.  Each sweep of the GPU is replayed by the oracle: at every step the
GPU's pick must minimise the full objective e H e^T over the group's candidates to within 1e-9
relative (the two sides order their binary64 sums differently, so only true near-ties may
resolve differently); the final objectives and scales must match the oracle's evaluation of the
GPU's indices, and no sweep may raise a row's objective."""
import numpy as np
import pytest
import torch

import int4_group_wise_b200 as q4
from int4_group_wise_b200 import inputs

pytestmark = pytest.mark.gpu
f32 = np.float32


def _problem(R, C, K, seed):
    W = inputs.gaussian((R, C), 0.02, seed=seed, cfg=93, name="W")
    Xb = inputs.activations(4 * C, C, seed=seed, cfg=93, name="X", outliers=max(1, C // 50))
    return W, Xb, inputs.alpha_grid(0.5, 0.5 / (K - 1), K)


def _gpu_refine(W, H, alpha, idx, sweeps):
    ti = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda()
    d, i, o = q4.refine(torch.from_numpy(W).cuda(), torch.from_numpy(H).cuda(), torch.from_numpy(alpha).cuda(),
                        ti, sweeps=sweeps)
    q4.sync_check()
    return d.cpu().numpy(), i.cpu().numpy(), o.cpu().numpy()


def _check_sweep(W, H, alpha, start, picked, oracle_mod):
    emin, epick = oracle_mod.refine_replay(W, H, alpha, start, picked)
    assert np.all(epick <= emin + 1e-9 * np.abs(emin) + 1e-30), float(np.max((epick - emin) / np.abs(emin)))


@pytest.mark.parametrize("R,C,K,sweeps", [(8, 128, 11, 1), (33, 96, 21, 2), (64, 256, 101, 1), (5, 1056, 9, 2)])
def test_refine_matches_oracle(R, C, K, sweeps, oracle_mod):
    W, Xb, alpha = _problem(R, C, K, seed=R + C + K)
    H = oracle_mod.hessian(Xb).astype(f32)
    _, idx0, _, _ = oracle_mod.scale_search(W, H, alpha, all_err=True)
    _, _, obj0 = oracle_mod.refine(W, H, alpha, idx0, sweeps=0)
    start = idx0.copy()
    for _ in range(sweeps):                   # one GPU sweep at a time, each replayed
        d, idx, obj = _gpu_refine(W, H, alpha, start, 1)
        _check_sweep(W, H, alpha, start, idx, oracle_mod)
        start = idx
    dr, _, objr = oracle_mod.refine(W, H, alpha, idx, sweeps=0)   # the oracle's evaluation of the GPU's state
    np.testing.assert_array_equal(d.view(np.uint32), dr.view(np.uint32))
    np.testing.assert_allclose(obj, objr, rtol=1e-9)
    assert np.all(obj <= obj0 * (1 + 1e-12))
    # and the same result as the oracle's own sweeps wherever no near-tie intervened
    _, idx_o, _ = oracle_mod.refine(W, H, alpha, idx0, sweeps=sweeps)
    assert np.mean(idx == idx_o) > 0.99


def test_refine_zero_sweeps_and_block_diagonal(oracle_mod):
    """sweeps = 0 only evaluates the start; with H block-diagonal nothing moves."""
    W, Xb, alpha = _problem(16, 128, 11, seed=4)
    H = oracle_mod.hessian(Xb).astype(f32)
    Hb = np.zeros_like(H)
    for g in range(4):
        Hb[32 * g:32 * g + 32, 32 * g:32 * g + 32] = H[32 * g:32 * g + 32, 32 * g:32 * g + 32]
    _, idx0, best, _ = oracle_mod.scale_search(W, Hb, alpha, all_err=True)
    _, idx, obj = _gpu_refine(W, Hb, alpha, idx0, 3)
    np.testing.assert_array_equal(idx, idx0)
    np.testing.assert_allclose(obj, best.sum(axis=1), rtol=1e-9)
    _, idx, obj = _gpu_refine(W, H, alpha, idx0, 0)
    np.testing.assert_array_equal(idx, idx0)
    np.testing.assert_allclose(obj, oracle_mod.refine(W, H, alpha, idx0, sweeps=0)[2], rtol=1e-9)


@pytest.mark.slow
def test_refine_up_projection_full_size():
    """The 1B-class up-projection (W 8192x2048, H of its 262144 calibration rows, K = 101),
    starting from the GPU search: the objective of no row rises, and the reported objectives
    equal e H e^T of the returned scales (binary64 product on the host)."""
    wl = inputs.workload(1)
    m = wl.matrices[0]
    W = wl.weight(m)
    X = torch.from_numpy(wl.activations(m.x_name).view(np.int16)).cuda().view(torch.bfloat16)
    H = q4.hessian(X)
    del X
    alpha = torch.from_numpy(wl.alpha()).cuda()
    tW = torch.from_numpy(W).cuda()
    _, idx0, _ = q4.scale_search(tW, H, alpha)
    ti = idx0.clone()
    _, _, obj0 = q4.refine(tW, H, alpha, ti, sweeps=0)
    d, idx, obj = q4.refine(tW, H, alpha, idx0.clone(), sweeps=1)
    q4.sync_check()
    obj0, obj = obj0.cpu().numpy(), obj.cpu().numpy()
    assert np.all(obj <= obj0 * (1 + 1e-12))
    assert np.mean(obj < obj0 * (1 - 1e-9)) > 0.5          # the coupled objective does improve
    Q = q4.lsq_fwd(tW, d).double()
    E = tW.double() - Q
    ref = (E @ H.double() * E).sum(dim=1).cpu().numpy()
    np.testing.assert_allclose(obj, ref, rtol=1e-8)
