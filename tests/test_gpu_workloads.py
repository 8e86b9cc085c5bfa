"""GPU parity on the two decoder-stack workloads, at their full sizes.

1B-class stack (16 layers, 112 matrices, 973 M weights): layer 0's four
calibration Hessians (n = 65536), block by block over every upper-triangle tile; the scale search of all
seven layer-0 matrices on sampled rows; one fused LSQ step over every matrix of
the stack with every output compared.

8B-class stack (32 layers, 224 matrices, 6.98 G weights): layer 0's Hessians
for both input widths (n = 131072, C = 4096 block by block over every upper
tile, C = 14336 over 256 sampled tiles); the
scale search of a 14336-row and a 14336-column matrix on sampled rows; the
fused LSQ step streamed over all 224 matrices, a row sample of each compared.

Oracle inputs are the same seeded tensors; the search's H is the oracle's own
(diagonal blocks), never the GPU's."""
import numpy as np
import pytest
import torch

import int4_group_wise_b200 as q4
from int4_group_wise_b200 import inputs
from hessian_check import check_hessian

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
f32 = np.float32


def _x_dev(Xb):
    return torch.from_numpy(Xb.view(np.int16)).cuda().view(torch.bfloat16)


def _diag_blocks(oracle_mod, Xb, groups):
    C = Xb.shape[1]
    H = np.zeros((C, C), f32)
    starts = [32 * g for g in groups]
    blocks = oracle_mod.hessian_blocks(Xb, starts, starts, 32)
    for g, b in zip(groups, blocks):
        H[32 * g:32 * g + 32, 32 * g:32 * g + 32] = b
    return H


def _check_hessian(Xb, oracle_mod, rng, tile_sample=None, n_random=16):
    """GPU H against the oracle block by block (each 32x32 / 128x128 block within 1e-3 relative
    Frobenius error on its own): every diagonal block, one block in every upper-triangle 256x256
    tile (or in `tile_sample` seeded tiles), and n_random seeded 128x128 tiles."""
    Hg = q4.hessian(_x_dev(Xb))
    q4.sync_check()
    Hg = Hg.cpu().numpy()
    np.testing.assert_array_equal(Hg, Hg.T)
    check_hessian(Hg, Xb, oracle_mod, rng, n_random=n_random, every_tile=tile_sample is None,
                  tile_sample=tile_sample)


def _check_search_rows(W, H, alpha, rows, oracle_mod):
    d, i, e = q4.scale_search(torch.from_numpy(W).cuda(), torch.from_numpy(H).cuda(),
                              torch.from_numpy(alpha).cuda())
    q4.sync_check()
    d, i, e = d.cpu().numpy()[rows], i.cpu().numpy()[rows], e.cpu().numpy()[rows]
    dr, ir, br, allE = oracle_mod.scale_search(W[rows], H, alpha, all_err=True)
    at = np.take_along_axis(allE, i[..., None].astype(np.int64), axis=2)[..., 0]
    same = i == ir
    assert np.all((at[~same] - br[~same]) <= 1e-6 * br[~same]), int((~same).sum())
    np.testing.assert_array_equal(d[same].view(np.uint32), dr[same].view(np.uint32))
    np.testing.assert_allclose(e.astype(np.float64), at, rtol=1e-4, atol=1e-30)


def _rtn_spread_delta(W, seed):
    rng = np.random.default_rng(seed)
    R, C = W.shape
    return (np.abs(W).reshape(R, C // 32, 32).max(axis=2) / f32(7) *
            rng.uniform(0.5, 1.0, (R, C // 32))).astype(f32)


def _check_lsq(W, D, G, oracle_mod, rows=None):
    tG = torch.from_numpy(G.view(np.int16)).cuda().view(torch.bfloat16)
    Q, gW, gD = q4.lsq_fwd_bwd(torch.from_numpy(W).cuda(), torch.from_numpy(D).cuda(), tG)
    q4.sync_check()
    Q, gW, gD = Q.cpu().numpy(), gW.cpu().numpy(), gD.cpu().numpy()
    if rows is not None:
        W, D, G, Q, gW, gD = W[rows], D[rows], G[rows], Q[rows], gW[rows], gD[rows]
    np.testing.assert_array_equal(Q.view(np.uint32), oracle_mod.lsq_fwd(W, D).view(np.uint32))
    gWr, gDr = oracle_mod.lsq_bwd(W, D, G, q4.GRAD_SCALE)
    np.testing.assert_array_equal(gW.view(np.uint32), gWr.view(np.uint32))
    Gf = inputs.bf16_bits_to_f32(G).astype(np.float64)
    v = W / np.repeat(np.where(D == 0, 1, D), 32, axis=1)
    dq = np.where(v <= -8, 8.0, np.where(v >= 7, 7.0, np.abs(np.rint(v) - v)))
    denom = q4.GRAD_SCALE * (np.abs(Gf) * dq).reshape(gD.shape[0], -1, 32).sum(axis=2)
    assert np.all(np.abs(gD - gDr) <= 1e-4 * denom + 1e-30)


# --------------------------------------------------------------- 1B-class stack
def test_stack_1b_layer0_hessians_and_searches(oracle_mod):
    wl = inputs.workload(3)
    rng = np.random.default_rng(3)
    alpha = wl.alpha()
    for x_name in ["L0.attn_in", "L0.o_in", "L0.mlp_in", "L0.down_in"]:
        Xb = wl.activations(x_name)
        assert Xb.shape == (65536, wl.calib[x_name])
        groups = range(Xb.shape[1] // 32)
        H = _diag_blocks(oracle_mod, Xb, groups)
        _check_hessian(Xb, oracle_mod, rng)
        for m in [m for m in wl.matrices if m.x_name == x_name]:
            W = wl.weight(m)
            rows = np.arange(0, m.d_out, 64)
            _check_search_rows(W, H, alpha, rows, oracle_mod)


def test_stack_1b_lsq_step_over_all_matrices(oracle_mod):
    wl = inputs.workload(3)
    total = 0
    for k, m in enumerate(wl.matrices):
        W, G = wl.weight(m), wl.grad(m)
        _check_lsq(W, _rtn_spread_delta(W, k), G, oracle_mod)
        total += W.size
    assert total == 16 * (2 * 2048 * 2048 + 2 * 512 * 2048 + 2 * 8192 * 2048 + 2048 * 8192)


# --------------------------------------------------------------- 8B-class stack
def test_stack_8b_layer0_hessians_and_searches(oracle_mod):
    wl = inputs.workload(4)
    rng = np.random.default_rng(4)
    alpha = wl.alpha()
    for x_name, mname in [("L0.mlp_in", "L0.gate"), ("L0.down_in", "L0.down")]:
        Xb = wl.activations(x_name)
        assert Xb.shape == (131072, wl.calib[x_name])
        m = next(mm for mm in wl.matrices if mm.name == mname)
        groups = range(0, Xb.shape[1] // 32, 7)
        H = _diag_blocks(oracle_mod, Xb, groups)
        # C = 4096: all 136 upper tiles; C = 14336: 1596 upper tiles, 256 of them sampled
        _check_hessian(Xb, oracle_mod, rng, tile_sample=None if Xb.shape[1] <= 4096 else 256, n_random=8)
        W = wl.weight(m)
        keep = np.zeros(W.shape[1] // 32, bool)
        keep[list(groups)] = True
        # rows sampled; the search runs on all groups but only the sampled groups' H blocks are
        # filled, so compare those groups only
        d, i, e = q4.scale_search(torch.from_numpy(W).cuda(), torch.from_numpy(H).cuda(),
                                  torch.from_numpy(alpha).cuda())
        q4.sync_check()
        rows = np.arange(0, m.d_out, 256)
        cols = np.concatenate([np.arange(32 * g, 32 * g + 32) for g in groups])
        Ws = W[rows][:, cols]
        Hs = H[np.ix_(cols, cols)]
        dr, ir, br, allE = oracle_mod.scale_search(Ws, Hs, alpha, all_err=True)
        gi = i.cpu().numpy()[rows][:, keep]
        gd = d.cpu().numpy()[rows][:, keep]
        ge = e.cpu().numpy()[rows][:, keep]
        at = np.take_along_axis(allE, gi[..., None].astype(np.int64), axis=2)[..., 0]
        same = gi == ir
        assert np.all((at[~same] - br[~same]) <= 1e-6 * br[~same])
        np.testing.assert_array_equal(gd[same].view(np.uint32), dr[same].view(np.uint32))
        np.testing.assert_allclose(ge.astype(np.float64), at, rtol=1e-4, atol=1e-30)


def test_stack_8b_lsq_streamed_over_all_matrices(oracle_mod):
    wl = inputs.workload(4)
    total = 0
    for k, m in enumerate(wl.matrices):
        W, G = wl.weight(m), wl.grad(m)
        rows = np.arange(k % 97, m.d_out, 97)
        _check_lsq(W, _rtn_spread_delta(W, k), G, oracle_mod, rows=rows)
        total += W.size
        torch.cuda.empty_cache()
    assert total == 6_979_321_856
