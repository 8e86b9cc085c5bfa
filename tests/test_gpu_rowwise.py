"""GPU parity of the per-channel (one scale per row) LSQ and W4A16 export
against the CPU oracle: bit-exact Q, grad_W, packed bytes and scales; the row
step gradient within 1e-4 relative to s * sum |G_i dQ_i/dDelta| of the row."""
import numpy as np
import pytest
import torch

import int4_group_wise_b200 as q4
from int4_group_wise_b200 import inputs

pytestmark = pytest.mark.gpu
f32 = np.float32


def _case(R, C, seed, *, zero_rows=0, ties=False, g_dtype="bf16"):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((R, C)) * 0.02).astype(f32)
    D = (np.abs(W).max(axis=1) / f32(7) * rng.uniform(0.3, 1.1, R)).astype(f32)
    for r in range(zero_rows):
        W[r] = 0
        D[r] = 0
    if ties:
        D[:] = f32(0.125)
        W[:, ::4] = (rng.integers(-20, 20, (R, C // 4)) + 0.5).astype(f32) * f32(0.125)
        W[:, 1::8] = f32(7.0 * 0.125)
        W[:, 3::8] = f32(-8.0 * 0.125)
    Gf = (rng.standard_normal((R, C)) * 1e-3).astype(f32)
    G = inputs.f32_to_bf16_bits(Gf) if g_dtype == "bf16" else Gf
    return W, D, G


def _run_and_check(W, D, G, oracle_mod):
    tG = torch.from_numpy(G.view(np.int16)).cuda().view(torch.bfloat16) if G.dtype == np.uint16 \
        else torch.from_numpy(G).cuda()
    tW, tD = torch.from_numpy(W).cuda(), torch.from_numpy(D).cuda()
    C = W.shape[1]
    s = q4.rowwise_grad_scale(C)
    Q, gW, gD = q4.lsq_fwd_bwd_rowwise(tW, tD, tG)
    Q1 = q4.lsq_fwd_rowwise(tW, tD)
    gW1, gD1 = q4.lsq_bwd_rowwise(tW, tD, tG)
    packed, scales = q4.pack_w4a16_rowwise(tW, tD)
    q4.sync_check()
    Qr = oracle_mod.lsq_fwd_rowwise(W, D)
    gWr, gDr = oracle_mod.lsq_bwd_rowwise(W, D, G, s)
    for a in (Q, Q1):
        np.testing.assert_array_equal(a.cpu().numpy().view(np.uint32), Qr.view(np.uint32))
    for a in (gW, gW1):
        np.testing.assert_array_equal(a.cpu().numpy().view(np.uint32), gWr.view(np.uint32))
    assert torch.equal(gD, gD1)
    Gf = (inputs.bf16_bits_to_f32(G) if G.dtype == np.uint16 else G).astype(np.float64)
    v = W / np.where(D == 0, 1, D)[:, None]
    dq = np.where(v <= -8, 8.0, np.where(v >= 7, 7.0, np.abs(np.rint(v) - v)))
    dq[D == 0] = 0
    denom = s * (np.abs(Gf) * dq).sum(axis=1)
    err = np.abs(gD.cpu().numpy().astype(np.float64) - gDr)
    assert np.all(err <= 1e-4 * denom + 1e-30), float(np.max(err / np.maximum(denom, 1e-30)))
    pr, sr = oracle_mod.pack_w4a16_rowwise(W, D)
    np.testing.assert_array_equal(packed.cpu().numpy(), pr)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint16), sr)


@pytest.mark.parametrize("R,C,kw", [
    (1, 32, {}), (3, 96, {"zero_rows": 1}), (7, 160, {"ties": True}), (5, 32 * 37, {"g_dtype": "f32"}),
    (33, 2080, {}), (2, 14336, {"zero_rows": 1}),
])
def test_rowwise_small_and_ragged(R, C, kw, oracle_mod):
    _run_and_check(*_case(R, C, seed=R + C, **kw), oracle_mod)


def test_rowwise_full_layer_shapes(oracle_mod):
    """The 1B-class up-projection (8192 x 2048) and 8B-class down-projection rows (x 14336)."""
    wl = inputs.workload(1)
    W, G = wl.weight(wl.matrices[0]), wl.grad(wl.matrices[0])
    D = (np.abs(W).max(axis=1) / f32(7)).astype(f32)
    _run_and_check(W, D, G, oracle_mod)
    W2 = inputs.gaussian((512, 14336), 0.015, seed=0, cfg=4, name="W/rowwise-long")
    G2 = inputs.grad((512, 14336), dtype="bf16", seed=0, cfg=4, name="G/rowwise-long")
    D2 = (np.abs(W2).max(axis=1) / f32(7) * f32(0.8)).astype(f32)
    _run_and_check(W2, D2, G2, oracle_mod)
