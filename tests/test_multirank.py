"""Multi-process host logic of bench.py on CPU (gloo, world size 2): per-rank
layers, whole-job aggregation (units summed, time = slowest rank) and the
reference arm running on rank 0 only."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        units, ms = bench.aggregate_over_ranks(100.0 * (rank + 1), 2.0 + rank)
        out.put((rank, units, ms, bench.layer_seed(rank)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_aggregation_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, units, ms, seed in res:
        assert units == 300.0          # units of both ranks
        assert ms == 3.0               # the slowest rank's time
    assert res[0][3] != res[1][3]      # each rank quantizes its own layer


def test_single_process_aggregation_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate_over_ranks(5.0, 1.5) == (5.0, 1.5)


def test_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` without a launcher re-executes itself under torch.distributed.run with
    two ranks (gloo on CPU for the reference arm): exactly one JSON line, from rank 0, reporting
    both ranks; the other rank exits 0 without work."""
    import json
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--config", "0", "--steps", "1", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert set(rec["stages"]) == {"hessian_gflops", "scale_search_groups_per_s", "lsq_fwd_bwd_gbs",
                                  "pack_w4a16_gbs"}


def test_gpus_flag_must_match_the_launchers_world_size():
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "4", "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300, cwd=ROOT)
    assert r.returncode != 0 and "WORLD_SIZE=2" in r.stderr


# ------------------------------------------------------------- split-n Hessian plumbing
def _hessian_worker(rank, world, port, n, C, out):
    """Each rank takes its shard of the calibration rows, forms its partial X_r^T X_r / n with
    the oracle (CPU stand-in for the kernel's qat4_hessian_partial), and the all-reduce of the
    distributed module sums them."""
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from int4_group_wise_b200 import distributed, inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        Xb = inputs.activations(n, C, seed=3, cfg=0, name="split", outliers=2)
        lo, hi = distributed.shard_rows(n, world, rank)
        part = oracle.hessian(Xb[lo:hi]) * ((hi - lo) / n)
        H = torch.from_numpy(part.astype(np.float32))
        distributed.allreduce_partials(H)
        out.put((rank, lo, hi, H.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_split_n_hessian_allreduce_two_gloo_ranks():
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    from int4_group_wise_b200 import inputs
    n, C = 1001, 64
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_hessian_worker, args=(r, 2, port, n, C, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the shards tile [0, n) exactly, and both ranks hold the same, full H
    assert [(lo, hi) for _, lo, hi, _ in res] == [(0, 500), (500, 1001)]
    np.testing.assert_array_equal(res[0][3], res[1][3])
    Href = oracle.hessian(inputs.activations(n, C, seed=3, cfg=0, name="split", outliers=2))
    np.testing.assert_allclose(res[0][3], Href, rtol=1e-6, atol=1e-6 * np.abs(Href).max())


def test_shard_rows_partition():
    sys.path.insert(0, ROOT)
    from int4_group_wise_b200 import distributed
    for n in (1, 7, 64, 262144, 1000003):
        for world in (1, 2, 3, 4, 8):
            bounds = [distributed.shard_rows(n, world, r) for r in range(world)]
            assert bounds[0][0] == 0 and bounds[-1][1] == n
            assert all(bounds[r][1] == bounds[r + 1][0] for r in range(world - 1))
            sizes = [hi - lo for lo, hi in bounds]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        distributed.shard_rows(10, 2, 2)
