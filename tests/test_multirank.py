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


def test_reference_arm_prints_only_on_rank0(tmp_path):
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0 and r.stdout.strip() == ""
