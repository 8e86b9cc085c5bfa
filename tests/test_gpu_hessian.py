"""GPU parity of the calibration Hessian against the float64 oracle:
relative Frobenius error <= 1e-3 (tensor-core fp32 accumulation of exact
bf16 products) over the whole matrix AND over every checked 32x32 block on
its own (hessian_check), bitwise symmetry, and run-to-run determinism."""
import numpy as np
import pytest
import torch

import int4_group_wise_b200 as q4
from int4_group_wise_b200 import inputs
from hessian_check import check_blocks, check_hessian

pytestmark = pytest.mark.gpu
f32 = np.float32


def _gpu_h(Xb):
    X = torch.from_numpy(np.ascontiguousarray(Xb).view(np.int16)).cuda().view(torch.bfloat16)
    H = q4.hessian(X)
    q4.sync_check()
    return X, H


def _frob(a, b):
    return float(np.linalg.norm(a.astype(np.float64) - b) / np.linalg.norm(b))


def _every_block(Hg, Hr):
    """Each 32x32 block of a fully computed H within 1e-3 relative Frobenius error on its own."""
    C = Hr.shape[0]
    starts = [(r, c) for r in range(0, C, 32) for c in range(0, C, 32)]
    check_blocks(Hg, np.stack([Hr[r:r + 32, c:c + 32] for r, c in starts]), starts, 32)


@pytest.mark.parametrize("n,C", [(1, 32), (63, 32), (65, 96), (200, 160), (64, 128), (129, 256),
                                 (1000, 288), (4096, 384)])
def test_hessian_small(n, C, oracle_mod):
    Xb = inputs.activations(n, C, seed=n, cfg=60, name="X", outliers=max(1, C // 100))
    X, H = _gpu_h(Xb)
    Hg = H.cpu().numpy()
    Hr = oracle_mod.hessian(Xb)
    assert _frob(Hg, Hr) <= 1e-3
    _every_block(Hg, Hr)
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
    _every_block(Hg, Hr)
    np.testing.assert_array_equal(Hg, Hg.T)
    H2 = q4.hessian(X)
    torch.cuda.synchronize()
    assert torch.equal(H, H2)


@pytest.mark.parametrize("cfg", [1, 2])
def test_hessian_full_size_every_tile(cfg, cache, oracle_mod):
    """Full n x C on the GPU (config 1: C = 2048, 36 upper tiles, n split in two and the
    partials reduced; config 2: C = 8192, 528 upper tiles stored directly).  The oracle
    recomputes every 32x32 diagonal block, one seeded 32x32 block inside every upper-triangle
    256x256 tile, and seeded random 128x128 tiles (64 at config 2) anywhere in H; each block
    must be within 1e-3 relative Frobenius error on its own."""
    wl = inputs.workload(cfg)
    Xb = cache.get(("X", cfg, "x"), lambda: wl.activations("x"))
    X, H = _gpu_h(Xb)
    Hg = H.cpu().numpy()
    del X, H
    np.testing.assert_array_equal(Hg, Hg.T)
    assert np.all(np.isfinite(Hg))
    check_hessian(Hg, Xb, oracle_mod, np.random.default_rng(cfg), n_random=64 if cfg == 2 else 16)


@pytest.mark.parametrize("n,C", [(40000, 3072), (50000, 2048), (20000, 512)])
def test_hessian_multi_chunk_ragged(n, C, oracle_mod):
    """n spans several 16384-row promotion chunks with a ragged last chunk and a ragged last
    128-row stage; (40000, 3072) stores H directly, the others split n and reduce partials."""
    Xb = inputs.activations(n, C, seed=n, cfg=62, name="X", outliers=C // 100)
    X, H = _gpu_h(Xb)
    Hg = H.cpu().numpy()
    np.testing.assert_array_equal(Hg, Hg.T)
    check_hessian(Hg, Xb, oracle_mod, np.random.default_rng(n), n_random=6)


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
