"""GPU parity of the fake-quant forward GEMM Y = X bf16(Q_Delta(W))^T against the binary64
oracle, for both calls: the staged one (quantizer, then a persistent tcgen05 GEMM) and the fused
one (the quantizer in the GEMM's producer).  The operand bf16(Q) is formed on the GPU from the same code decision as the oracle;
products of bf16 values are exact in float32, so the only difference is the float32 summation
of C products: |Y - Y_ref| <= C * 2^-23 * sum_c |x_c| |b_c| (the classical bound for a
recursively summed dot product, doubled to cover a truncating accumulator)."""
import numpy as np
import pytest
import torch

import int4_group_wise_b200 as q4
from int4_group_wise_b200 import inputs
from oracle import twin

pytestmark = pytest.mark.gpu
f32 = np.float32


def _problem(T, R, C, seed):
    W = inputs.gaussian((R, C), 0.02, seed=seed, cfg=92, name="W")
    rng = np.random.default_rng(seed)
    D = (np.abs(W).reshape(R, C // 32, 32).max(axis=2) / f32(7) *
         rng.uniform(0.5, 1.0, (R, C // 32))).astype(f32)
    Xb = inputs.activations(T, C, seed=seed, cfg=92, name="X", outliers=max(1, C // 100))
    return Xb, W, D


def _run(Xb, W, D, fused=False):
    tX = torch.from_numpy(Xb.view(np.int16)).cuda().view(torch.bfloat16)
    Y = q4.fq_gemm(tX, torch.from_numpy(W).cuda(), torch.from_numpy(D).cuda(), fused=fused)
    q4.sync_check()
    return Y.cpu().numpy().astype(np.float64)


def _abs_bound(Xb, W, D, tt=None, rr=None):
    Qb = twin._bf16_rne(twin.fake_quant(W, np.repeat(D, 32, axis=1))).astype(np.float64)
    ax = np.abs(inputs.bf16_bits_to_f32(Xb).astype(np.float64))
    if tt is None:
        return ax @ np.abs(Qb).T
    return np.einsum("mc,mc->m", ax[tt], np.abs(Qb[rr]))


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("T,R,C", [(256, 256, 64), (1, 33, 32), (300, 300, 96), (513, 257, 2080),
                                   (128, 512, 4096), (260, 1000, 512), (2048, 2560, 384), (600, 19030, 160)])
def test_fq_gemm_matches_oracle(T, R, C, fused, oracle_mod):
    """Single and multiple 256x256 tiles (more tiles than SM pairs in the last two, so the staged
    GEMM's pairs take several tiles and alternate accumulators), ragged tokens, rows (R % 4 != 0)
    and columns (C % 128 == 32 or 96)."""
    Xb, W, D = _problem(T, R, C, seed=T + R + C)
    Y = _run(Xb, W, D, fused)
    Yr = oracle_mod.fq_gemm(Xb, W, D)
    bound = C * 2.0 ** -23 * _abs_bound(Xb, W, D) + 1e-30
    err = np.abs(Y - Yr)
    assert np.all(err <= bound), float(np.max(err / bound))


@pytest.mark.parametrize("fused", [False, True])
def test_fq_gemm_zero_groups_and_clamps(fused, oracle_mod):
    """All-zero groups (Delta = 0) give Q = 0; scales far below max|w|/7 clamp most codes."""
    T, R, C = 256, 256, 128
    Xb, W, D = _problem(T, R, C, seed=5)
    W[:, 32:64] = 0.0
    D[:, 1] = 0.0
    D[:, 2] *= f32(0.1)
    Y = _run(Xb, W, D, fused)
    Yr = oracle_mod.fq_gemm(Xb, W, D)
    bound = C * 2.0 ** -23 * _abs_bound(Xb, W, D) + 1e-30
    assert np.all(np.abs(Y - Yr) <= bound)


@pytest.mark.slow
@pytest.mark.parametrize("fused", [False, True])
def test_fq_gemm_up_projection_full_size(fused, oracle_mod):
    """The 1B-class up-projection (W 8192x2048) on a micro-batch of 8192 tokens, the size the
    benchmark times; 4096 sampled outputs against the oracle."""
    wl = inputs.workload(1)
    m = wl.matrices[0]
    W = wl.weight(m)
    rng = np.random.default_rng(1)
    D = (np.abs(W).reshape(W.shape[0], -1, 32).max(axis=2) / f32(7) *
         rng.uniform(0.5, 1.0, (W.shape[0], W.shape[1] // 32))).astype(f32)
    Xb = wl.activations(m.x_name, n=8192)
    Y = _run(Xb, W, D, fused)
    tt = rng.integers(0, Xb.shape[0], 4096)
    rr = rng.integers(0, W.shape[0], 4096)
    ref = oracle_mod.fq_gemm_entries(Xb, W, D, tt, rr)
    bound = W.shape[1] * 2.0 ** -23 * _abs_bound(Xb, W, D, tt, rr) + 1e-30
    assert np.all(np.abs(Y[tt, rr] - ref) <= bound)


@pytest.mark.parametrize("fused", [False, True])
def test_fq_gemm_deterministic(fused):
    """Repeated launches give bitwise identical Y (the ring slots are reused only after their
    contents are consumed; a race there shows up as whole W rows differing), and both calls give
    the same products up to the float32 summation order."""
    Xb, W, D = _problem(1024, 2048, 2048, seed=9)
    tX = torch.from_numpy(Xb.view(np.int16)).cuda().view(torch.bfloat16)
    tW, tD = torch.from_numpy(W).cuda(), torch.from_numpy(D).cuda()
    Y0 = q4.fq_gemm(tX, tW, tD, fused=fused).clone()
    for _ in range(30):
        assert torch.equal(q4.fq_gemm(tX, tW, tD, fused=fused), Y0)
    Y1 = q4.fq_gemm(tX, tW, tD, fused=not fused)
    q4.sync_check()
    bound = 2048 * 2.0 ** -22 * torch.from_numpy(_abs_bound(Xb, W, D)).cuda()
    assert torch.all((Y1.double() - Y0.double()).abs() <= bound)
