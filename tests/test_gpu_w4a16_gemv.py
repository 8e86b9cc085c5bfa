"""GPU parity of the W4A16 inference product on the packed export against the
binary64 oracle.  Products are exact and sums float32, so each output is
within 5e-5 of sum_c |x_c| |scale * code_c| (about 1 + C/32 + 5 float32
roundings on the longest path, C <= 14336)."""
import numpy as np
import pytest
import torch

import int4_group_wise_b200 as q4
from int4_group_wise_b200 import inputs

pytestmark = pytest.mark.gpu
f32 = np.float32


def _export(R, C, seed, rowwise=False):
    W = inputs.gaussian((R, C), 0.02, seed=seed, cfg=90, name="W")
    if rowwise:
        D = (np.abs(W).max(axis=1) / f32(7)).astype(f32)
        return W, D
    D = (np.abs(W).reshape(R, C // 32, 32).max(axis=2) / f32(7) * f32(0.85)).astype(f32)
    return W, D


def _check(W, D, M, oracle_mod, rowwise=False):
    R, C = W.shape
    tW, tD = torch.from_numpy(W).cuda(), torch.from_numpy(D).cuda()
    packed, scales = (q4.pack_w4a16_rowwise(tW, tD) if rowwise else q4.pack_w4a16(tW, tD))
    xb = inputs.activations(M, C, seed=M + C, cfg=91, name="x", outliers=max(1, C // 100))
    tx = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    y = q4.w4a16_gemv(tx, packed, scales)
    q4.sync_check()
    pk, sc = packed.cpu().numpy(), scales.cpu().numpy().view(np.uint16)
    group = C if rowwise else 32
    yr = oracle_mod.w4a16_gemv(xb, pk, sc.reshape(R, -1), group)
    # magnitude bound sum_c |x_c| |scale * code_c| (float64, from the export's bytes)
    lo, hi = (pk & 0xF).astype(np.int16), (pk >> 4).astype(np.int16)
    codes = np.empty((R, C), np.float64)
    codes[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    codes[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    sf = np.repeat(sc.view(np.float16).astype(np.float64).reshape(R, -1), group, axis=1)
    bound = np.abs(inputs.bf16_bits_to_f32(xb).astype(np.float64)) @ np.abs(codes * sf).T
    err = np.abs(y.cpu().numpy().astype(np.float64) - yr)
    assert np.all(err <= 5e-5 * bound + 1e-30), float(np.max(err / np.maximum(bound, 1e-30)))


@pytest.mark.parametrize("R,C,M", [(1, 32, 1), (33, 96, 2), (70, 2080, 3), (64, 4096, 4), (45, 32 * 129, 5),
                                   (31, 14336, 1), (50, 30016, 4), (100, 4096, 8), (17, 1056, 9),
                                   (300, 14336, 7)])
def test_gemv_group32(R, C, M, oracle_mod):
    """Ragged rows and columns, 1..9 tokens (more than 8 take two passes); C = 30016 leaves room
    for 3 tokens per pass only, C = 14336 for 6."""
    _check(*_export(R, C, seed=R * 7 + C), M, oracle_mod)


@pytest.mark.parametrize("R,C,M", [(17, 64, 1), (40, 4096, 4)])
def test_gemv_rowwise_scales(R, C, M, oracle_mod):
    _check(*_export(R, C, seed=R + C, rowwise=True), M, oracle_mod, rowwise=True)


def test_gemv_layer_shape(oracle_mod):
    """The 8B-class gate projection (14336 x 4096), one token and four tokens."""
    W, D = _export(14336, 4096, seed=5)
    for M in (1, 4):
        _check(W, D, M, oracle_mod)


def test_gemv_deterministic():
    """Repeated launches give bitwise identical y (two partial sums per cut row block at most,
    and no ring slot is refilled before its codes are used)."""
    W, D = _export(14336, 4096, seed=6)
    packed, scales = q4.pack_w4a16(torch.from_numpy(W).cuda(), torch.from_numpy(D).cuda())
    for M in (1, 4):
        xb = inputs.activations(M, 4096, seed=M, cfg=91, name="xdet", outliers=40)
        tx = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
        y0 = q4.w4a16_gemv(tx, packed, scales).clone()
        for _ in range(30):
            assert torch.equal(q4.w4a16_gemv(tx, packed, scales), y0)
    q4.sync_check()
