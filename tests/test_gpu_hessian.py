"""GPU parity of the calibration Hessian against the float64 oracle:
relative Frobenius error <= 1e-3 (tensor-core fp32 accumulation of exact
bf16 products), bitwise symmetry, and run-to-run determinism."""
import numpy as np
import pytest
import torch

import int4_group_wise_b200 as q4
from int4_group_wise_b200 import inputs

pytestmark = pytest.mark.gpu
f32 = np.float32


def _gpu_h(Xb):
    X = torch.from_numpy(np.ascontiguousarray(Xb).view(np.int16)).cuda().view(torch.bfloat16)
    H = q4.hessian(X)
    q4.sync_check()
    return X, H


def _frob(a, b):
    return float(np.linalg.norm(a.astype(np.float64) - b) / np.linalg.norm(b))


@pytest.mark.parametrize("n,C", [(1, 32), (63, 32), (65, 96), (200, 160), (64, 128), (129, 256),
                                 (1000, 288), (4096, 384)])
def test_hessian_small(n, C, oracle_mod):
    Xb = inputs.activations(n, C, seed=n, cfg=60, name="X", outliers=max(1, C // 100))
    X, H = _gpu_h(Xb)
    Hg = H.cpu().numpy()
    Hr = oracle_mod.hessian(Xb)
    assert _frob(Hg, Hr) <= 1e-3
    np.testing.assert_array_equal(Hg, Hg.T)
    assert np.all(np.isfinite(Hg))


def test_hessian_exact_small_integers(oracle_mod):
    """Small-integer X: every partial sum is an exactly representable integer, so fp32 accumulation is exact."""
    rng = np.random.default_rng(3)
    n, C = 256, 192
    Xb = inputs.f32_to_bf16_bits(rng.integers(-4, 5, size=(n, C)).astype(f32))
    X, H = _gpu_h(Xb)
    np.testing.assert_array_equal(H.cpu().numpy().astype(np.float64), oracle_mod.hessian(Xb))


def test_hessian_config0_full_and_deterministic(cache, oracle_mod):
    wl = inputs.workload(0)
    Xb = cache.get(("X", 0, "x"), lambda: wl.activations("x"))
    X, H = _gpu_h(Xb)
    Hr = oracle_mod.hessian(Xb)
    Hg = H.cpu().numpy()
    assert _frob(Hg, Hr) <= 1e-3
    np.testing.assert_array_equal(Hg, Hg.T)
    H2 = q4.hessian(X)
    torch.cuda.synchronize()
    assert torch.equal(H, H2)


@pytest.mark.parametrize("cfg", [1, 2])
def test_hessian_full_size_sampled(cfg, cache, oracle_mod):
    """Full n x C on the GPU; the oracle recomputes every 32x32 diagonal block
    plus seeded random 128x128 tiles (upper and lower), Frobenius over the sample."""
    wl = inputs.workload(cfg)
    Xb = cache.get(("X", cfg, "x"), lambda: wl.activations("x"))
    X, H = _gpu_h(Xb)
    Hg = H.cpu().numpy()
    C = Xb.shape[1]
    np.testing.assert_array_equal(Hg, Hg.T)
    num = den = 0.0
    for g in range(C // 32):
        ref = oracle_mod.hessian_block(Xb, 32 * g, 32, 32 * g, 32)
        got = Hg[32 * g:32 * g + 32, 32 * g:32 * g + 32]
        num += float(np.sum((got - ref) ** 2))
        den += float(np.sum(ref ** 2))
    rng = np.random.default_rng(cfg)
    for _ in range(4):
        r0, c0 = (int(v) * 128 for v in rng.integers(0, C // 128, 2))
        ref = oracle_mod.hessian_block(Xb, r0, 128, c0, 128)
        got = Hg[r0:r0 + 128, c0:c0 + 128]
        num += float(np.sum((got - ref) ** 2))
        den += float(np.sum(ref ** 2))
    assert (num / den) ** 0.5 <= 1e-3, (num / den) ** 0.5


@pytest.mark.parametrize("n,C", [(40000, 3072), (50000, 2048), (20000, 512)])
def test_hessian_multi_chunk_ragged(n, C, oracle_mod):
    """n spans several 16384-row promotion chunks with a ragged last chunk and a ragged last
    64-row stage; (40000, 3072) stores H directly, the others split n and reduce partials."""
    Xb = inputs.activations(n, C, seed=n, cfg=62, name="X", outliers=C // 100)
    X, H = _gpu_h(Xb)
    Hg = H.cpu().numpy()
    np.testing.assert_array_equal(Hg, Hg.T)
    rng = np.random.default_rng(n)
    num = den = 0.0
    blocks = [(0, 0), (C - 128, C - 128)] + [tuple(int(v) * 64 for v in rng.integers(0, C // 64 - 1, 2))
                                             for _ in range(3)]
    for r0, c0 in blocks:
        ref = oracle_mod.hessian_block(Xb, r0, 128 if r0 + 128 <= C else 64, c0, 128 if c0 + 128 <= C else 64)
        got = Hg[r0:r0 + ref.shape[0], c0:c0 + ref.shape[1]]
        num += float(np.sum((got - ref) ** 2))
        den += float(np.sum(ref ** 2))
    assert (num / den) ** 0.5 <= 1e-3, (num / den) ** 0.5


def test_hessian_workspace_contract():
    """The call rejects a missing or short workspace when n is split, and ignores it otherwise."""
    Xb = inputs.activations(4096, 512, seed=5, cfg=63, name="X")
    X = torch.from_numpy(Xb.view(np.int16)).cuda().view(torch.bfloat16)
    need = q4.hessian_workspace_bytes(4096, 512)
    assert need > 0
    H = torch.empty((512, 512), dtype=torch.float32, device="cuda")
    L = q4.lib()
    st = torch.cuda.current_stream().cuda_stream
    import ctypes as ct
    assert L.qat4_hessian(ct.c_void_p(X.data_ptr()), 4096, 512, ct.c_void_p(H.data_ptr()), None, 0,
                          ct.c_void_p(st)) == 5
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    assert L.qat4_hessian(ct.c_void_p(X.data_ptr()), 4096, 512, ct.c_void_p(H.data_ptr()),
                          ct.c_void_p(ws.data_ptr()), need - 16, ct.c_void_p(st)) == 5
    assert L.qat4_hessian(ct.c_void_p(X.data_ptr()), 4096, 512, ct.c_void_p(H.data_ptr()),
                          ct.c_void_p(ws.data_ptr()), need, ct.c_void_p(st)) == 0
    q4.sync_check()


def test_bounded_wait_reports_timeout_and_context_survives():
    assert q4.selftest_bounded_wait(20_000_000) == 7      # QAT4_ERR_TIMEOUT after ~20 ms
    q4.sync_check()                                        # cleared
    Xb = inputs.activations(64, 64, seed=1, cfg=61, name="X")
    _gpu_h(Xb)                                             # kernels still run afterwards


def test_split_n_partials_sum_to_the_hessian(oracle_mod):
    """The split-n exchange step: partials X_r^T X_r / n over 4 ragged row shards (one of them
    spanning several promotion chunks) add up to H within the same bound; small-integer X makes
    every partial and their sum exact, so there it is bitwise."""
    from int4_group_wise_b200 import distributed
    n, C = 40000, 256
    Xb = inputs.activations(n, C, seed=21, cfg=60, name="Xsplit", outliers=3)
    X = torch.from_numpy(Xb.view(np.int16)).cuda().view(torch.bfloat16)
    parts = [q4.hessian_partial(X[lo:hi], n) for lo, hi in (distributed.shard_rows(n, 4, r) for r in range(4))]
    q4.sync_check()
    Hs = sum(p.double() for p in parts).cpu().numpy()
    assert _frob(Hs, oracle_mod.hessian(Xb)) <= 1e-3
    # exact case: integer-valued X and n a power of two (1/n exact)
    rng = np.random.default_rng(5)
    Xi = inputs.f32_to_bf16_bits(rng.integers(-3, 4, (4096, 64)).astype(np.float32))
    Xt = torch.from_numpy(Xi.view(np.int16)).cuda().view(torch.bfloat16)
    Hfull = q4.hessian(Xt)
    Hsum = q4.hessian_partial(Xt[:1000], 4096) + q4.hessian_partial(Xt[1000:], 4096)
    q4.sync_check()
    assert torch.equal(Hsum, Hfull)


def test_hessian_sharded_single_rank_nccl():
    """hessian_sharded end to end (partial on the tensor cores, then the NCCL all-reduce) in a
    one-rank process group: the all-reduce is the identity, so H equals qat4_hessian's."""
    import os
    import socket
    import torch.distributed as dist
    from int4_group_wise_b200 import distributed
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        Xb = inputs.activations(3000, 512, seed=2, cfg=60, name="Xnccl", outliers=5)
        X = torch.from_numpy(Xb.view(np.int16)).cuda().view(torch.bfloat16)
        H = distributed.hessian_sharded(X, 3000)
        torch.cuda.synchronize()
        q4.sync_check()
        assert torch.equal(H, q4.hessian(X))
    finally:
        dist.destroy_process_group()
