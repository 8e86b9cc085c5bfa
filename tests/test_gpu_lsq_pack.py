"""GPU parity of the streaming kernels (LSQ forward, backward, fused, W4A16
pack) against the CPU oracle, through the C ABI.  Codes, Q, grad_W and
packed bytes are bit-exact; grad_Delta is within 1e-4 relative to
s * sum |G_i dQ_i/dDelta| of its group."""
import numpy as np
import pytest
import torch

import int4_group_wise_b200 as q4
from int4_group_wise_b200 import inputs

pytestmark = pytest.mark.gpu
f32 = np.float32
S = q4.GRAD_SCALE


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.view(dtype) if dtype is not None else t


def _bits(a):
    return np.ascontiguousarray(a, f32).view(np.uint32)


def _case(R, C, seed, *, zero_groups=0, ties=False, scale=0.02, alpha=(0.4, 1.1), g_dtype="bf16"):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((R, C)) * scale).astype(f32)
    D = (np.abs(W).reshape(R, C // 32, 32).max(axis=2) / f32(7) *
         rng.uniform(*alpha, (R, C // 32))).astype(f32)
    if zero_groups:
        for _ in range(zero_groups):
            r, g = rng.integers(R), rng.integers(C // 32)
            W[r, 32 * g:32 * g + 32] = 0
            D[r, g] = 0
    if ties:
        # half-integer multiples of Delta and clamp edges, exactly representable
        D[:] = f32(0.125)
        W[:, ::4] = (rng.integers(-20, 20, (R, C // 4)) + 0.5).astype(f32) * f32(0.125)
        W[:, 1::8] = f32(7.0 * 0.125)
        W[:, 3::8] = f32(-8.0 * 0.125)
    Gf = (rng.standard_normal((R, C)) * 1e-3).astype(f32)
    G = inputs.f32_to_bf16_bits(Gf) if g_dtype == "bf16" else Gf
    return W, D, G


def _check_grad_delta(gd_gpu, W, D, G, oracle_mod):
    _, gd_ref = oracle_mod.lsq_bwd(W, D, G, S)
    # condition-aware denominator: s * sum |G_i * dQ_i/dDelta| per group
    Gf = inputs.bf16_bits_to_f32(G) if G.dtype == np.uint16 else G
    absG = np.abs(Gf).astype(f32)
    v = W / np.repeat(np.where(D == 0, 1, D), 32, axis=1)
    dq = np.where(v <= -8, -8.0, np.where(v >= 7, 7.0, np.rint(v) - v))
    dq[np.repeat(D == 0, 32, axis=1)] = 0
    denom = S * (absG.astype(np.float64) * np.abs(dq)).reshape(gd_ref.shape[0], -1, 32).sum(axis=2)
    err = np.abs(gd_gpu.astype(np.float64) - gd_ref)
    assert np.all(err <= 1e-4 * denom + 1e-30), float((err / np.maximum(denom, 1e-30)).max())


@pytest.mark.parametrize("R,C,kw", [
    (1, 32, {}), (3, 64, {}), (3, 96, {"zero_groups": 2}), (7, 160, {"ties": True}),
    (5, 32 * 37, {"g_dtype": "f32"}), (33, 224, {"alpha": (0.05, 3.0)}),
    (257, 512, {"zero_groups": 5, "g_dtype": "f32"}),
])
def test_lsq_small_shapes(R, C, kw, oracle_mod):
    W, D, G = _case(R, C, seed=R * 1000 + C, **kw)
    tW, tD = _dev(W), _dev(D)
    tG = _dev(G, torch.bfloat16) if G.dtype == np.uint16 else _dev(G)
    Q = q4.lsq_fwd(tW, tD)
    gW, gD = q4.lsq_bwd(tW, tD, tG)
    Q2, gW2, gD2 = q4.lsq_fwd_bwd(tW, tD, tG)
    q4.sync_check()
    Qr = oracle_mod.lsq_fwd(W, D)
    gWr, _ = oracle_mod.lsq_bwd(W, D, G, S)
    np.testing.assert_array_equal(_bits(Q.cpu().numpy()), _bits(Qr))
    np.testing.assert_array_equal(_bits(gW.cpu().numpy()), _bits(gWr))
    np.testing.assert_array_equal(_bits(Q2.cpu().numpy()), _bits(Qr))
    np.testing.assert_array_equal(_bits(gW2.cpu().numpy()), _bits(gWr))
    _check_grad_delta(gD.cpu().numpy(), W, D, G, oracle_mod)
    np.testing.assert_array_equal(gD.cpu().numpy(), gD2.cpu().numpy())


@pytest.mark.parametrize("R,C,kw", [
    (1, 32, {}), (3, 96, {"zero_groups": 2}), (7, 160, {"ties": True}), (33, 224, {"alpha": (0.05, 3.0)}),
])
def test_pack_small_shapes(R, C, kw, oracle_mod):
    W, D, _ = _case(R, C, seed=R * 7 + C, **kw)
    D[0, 0] = f32(70000.0)            # binary16 overflow -> inf
    if D.shape[1] > 1:
        D[0, 1] = f32(3e-7)           # binary16 subnormal
    packed, scales = q4.pack_w4a16(_dev(W), _dev(D))
    q4.sync_check()
    pr, sr = oracle_mod.pack_w4a16(W, D)
    np.testing.assert_array_equal(packed.cpu().numpy(), pr)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint16), sr)


def _workload_weights(cache, cfg):
    def make():
        wl = inputs.workload(cfg)
        m = wl.matrices[0]
        W = wl.weight(m)
        G = wl.grad(m)
        # scales at the RTN point times a spread, so some groups clamp
        rng = np.random.default_rng(cfg)
        D = (np.abs(W).reshape(W.shape[0], -1, 32).max(axis=2) / f32(7) *
             rng.uniform(0.5, 1.0, (W.shape[0], W.shape[1] // 32))).astype(f32)
        return W, D, G
    return cache.get(("lsq", cfg), make)


@pytest.mark.parametrize("cfg", [0, 1, 2])
def test_lsq_pack_full_workloads(cfg, cache, oracle_mod):
    """Full-size layer shapes (16.8 M elements for the 1B-class layers), every output compared."""
    W, D, G = _workload_weights(cache, cfg)
    tW, tD = _dev(W), _dev(D)
    tG = _dev(G, torch.bfloat16) if G.dtype == np.uint16 else _dev(G)
    Q, gW, gD = q4.lsq_fwd_bwd(tW, tD, tG)
    packed, scales = q4.pack_w4a16(tW, tD)
    q4.sync_check()
    Qr = oracle_mod.lsq_fwd(W, D)
    gWr, _ = oracle_mod.lsq_bwd(W, D, G, S)
    np.testing.assert_array_equal(_bits(Q.cpu().numpy()), _bits(Qr))
    np.testing.assert_array_equal(_bits(gW.cpu().numpy()), _bits(gWr))
    _check_grad_delta(gD.cpu().numpy(), W, D, G, oracle_mod)
    pr, sr = oracle_mod.pack_w4a16(W, D)
    np.testing.assert_array_equal(packed.cpu().numpy(), pr)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint16), sr)
    # run-to-run determinism (same bytes twice)
    Q2, gW2, gD2 = q4.lsq_fwd_bwd(tW, tD, tG)
    torch.cuda.synchronize()
    assert torch.equal(Q, Q2) and torch.equal(gW, gW2) and torch.equal(gD, gD2)


@pytest.mark.parametrize("R,C,gdt,pinned", [(3000, 1024, "bf16", True), (5000, 1024, "f32", True),
                                           (70, 96, "bf16", False), (1, 32, "f32", True)])
def test_lsq_fwd_bwd_host_matches_device_path(R, C, gdt, pinned):
    """The host-buffer pipeline (row chunks uploaded, run and downloaded on two streams) gives the
    same bits as the device call: 1 to 3 chunks, a ragged last chunk, pageable and pinned memory."""
    W = inputs.student_t((R, C), 3.0, 0.01, seed=R, cfg=60, name="W")
    d = (np.abs(W).reshape(R, C // 32, 32).max(axis=2) / np.float32(7)).astype(np.float32)
    G = (np.random.default_rng(R).standard_normal((R, C)) * 1e-3).astype(np.float32)
    Wt, dt = torch.from_numpy(W), torch.from_numpy(d)
    Gt = torch.from_numpy(G).to(torch.bfloat16) if gdt == "bf16" else torch.from_numpy(G)
    if pinned:
        Wt, dt, Gt = Wt.pin_memory(), dt.pin_memory(), Gt.pin_memory()
    Qh, gWh, gDh = q4.lsq_fwd_bwd_host(Wt, dt, Gt)
    torch.cuda.current_stream().synchronize()
    Qd, gWd, gDd = q4.lsq_fwd_bwd(Wt.cuda(), dt.cuda(), Gt.cuda())
    q4.sync_check()
    assert torch.equal(Qh, Qd.cpu()) and torch.equal(gWh, gWd.cpu()) and torch.equal(gDh, gDd.cpu())
