"""Benchmark of the group-32 INT4 quantizer path on B200.

One step = one pass of the whole path over one 1B-class MLP up-projection
(W fp32 8192x2048, calibration X bf16 262144x2048 with 1% outlier channels,
101-candidate grid, upstream gradient bf16):

    H = hessian(X) -> (delta, idx, err) = scale_search(W, H, alpha)
      -> (Q, grad_W, grad_delta) = lsq_fwd_bwd(W, delta, G) -> pack_w4a16(W, delta)

Every input is resident in HBM before timing starts.  Before each stage the
L2 cache (126 MB) is flushed by a read sweep over a 512 MB buffer, so no
stage reads its inputs from L2; the flushes are inside ms_per_step but not
inside the per-kernel times.  Per-kernel times are CUDA events on the stream
the kernels run on.

The headline `value` is the first metric of the path, LSQ fwd+bwd GB/s
(14.25 algorithmic bytes per weight); the Hessian TFLOP/s, scale-search
groups/s and pack GB/s are in `stages`, each with its roofline.  With N GPUs
every rank quantizes its own layer (independent problems, weak scaling, no
collective on the data path); the value is the bytes of all ranks divided by
the slowest rank's time.

`--impl reference` times the CPU oracle instead (test infrastructure, run
only here and in the tests) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "LSQ fwd+bwd GB/s (% HBM peak); scale-search groups/s; Hessian TFLOP/s"
LSQ_BYTES_PER_ELT = 14.25       # W 4 + G(bf16) 2 + Q 4 + grad_W 4 + (delta 4 + grad_delta 4)/32
PACK_BYTES_PER_ELT = 4.6875     # W 4 + delta 4/32 + nibbles 0.5 + fp16 scale 2/32
SEARCH_OPS_PER_CAND = 720       # 528 FMA quadratic form + 32 x (div, rint, min, max, mul, sub)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


# --------------------------------------------------------------------------- setup
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic_1b_up_proj.md")
# where the nvidia-smi clock samples of the timed region are written (one CSV per rank)
OUT_DIR = os.environ.get("QAT4_BENCH_OUT", os.path.join(ROOT, "bench_out"))
STAGE_KERNELS = {"hessian": ["hessian_pair_kernel", "hessian_reduce_kernel"],
                 "scale_search": ["scale_search_kernel"], "lsq_fwd_bwd": ["lsq_blocks_kernel"],
                 "pack_w4a16": ["pack_w4a16_blocks_kernel"]}


STEP_SOURCES = ("device_common.cuh", "hessian.cuh", "lsq_pack.cuh", "scale_search.cuh")


def source_hash() -> str:
    """Hash of the kernel sources of the group-32 step, matching the one recorded with the ncu
    traffic table."""
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "int4_group_wise_b200", "csrc")
    for f in STEP_SOURCES:
        h.update(f.encode())
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_traffic(config: int):
    """Per-stage DRAM bytes per launch from the committed ncu table, or {} when stale or absent."""
    if config != 1 or not os.path.exists(TRAFFIC_FILE):
        return {}
    text = open(TRAFFIC_FILE).read()
    recorded = next((ln.split(":", 1)[1].strip() for ln in text.splitlines() if ln.startswith("source_hash:")), None)
    if recorded != source_hash():
        return {}
    per_kernel = {}
    for ln in text.splitlines():
        f = [x.strip() for x in ln.strip().strip("|").split("|")]
        if len(f) == 2 and f[1].isdigit():
            per_kernel[f[0]] = int(f[1])
    return {st: sum(per_kernel.get(k, 0) for k in ks) for st, ks in STAGE_KERNELS.items()
            if all(k in per_kernel for k in ks)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def layer_seed(rank: int) -> int:
    """Every rank quantizes its own, independently seeded layer."""
    return rank


def aggregate_over_ranks(local_units: float, local_ms: float, group=None):
    """(sum of units over ranks, max of ms over ranks); plain values when not distributed."""
    import torch
    import torch.distributed as dist
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return float(local_units), float(local_ms)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend(group) == "nccl" else "cpu"
    u = torch.tensor([local_units], dtype=torch.float64, device=dev)
    t = torch.tensor([local_ms], dtype=torch.float64, device=dev)
    dist.all_reduce(u, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(u.item()), float(t.item())


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    def __init__(self, index: int, out_path: str | None = None):
        self.index = index
        self.proc = None
        self.out_path = out_path

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={CLOCK_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
            if self.out_path:
                os.makedirs(os.path.dirname(self.out_path), exist_ok=True)
                with open(self.out_path, "w") as fh:
                    fh.write(CLOCK_FIELDS + "\n" + "\n".join(self.lines) + "\n")

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        load = [s for s in sm if s > 500] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------ our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    import int4_group_wise_b200 as q4
    from int4_group_wise_b200 import inputs

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    peaks, peak_kind = load_peaks()

    wl = inputs.workload(args.config)
    m = wl.matrices[0]
    seed = layer_seed(rank)
    t0 = time.time()
    W_h = wl.weight(m, seed)
    X_h = wl.activations(m.x_name, seed)
    G_h = wl.grad(m, seed)
    alpha_h = wl.alpha()
    gen_s = time.time() - t0
    R, C = W_h.shape
    n = X_h.shape[0]
    groups = R * C // 32
    K = alpha_h.size

    # pinned host copies (for the end-to-end leg) and device-resident inputs
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    W_p, X_p, G_p, a_p = pin(W_h), pin(X_h.view(np.int16)), pin(G_h.view(np.int16)), pin(alpha_h)
    W = W_p.to(dev)
    X = X_p.to(dev).view(torch.bfloat16)
    G = G_p.to(dev).view(torch.bfloat16)
    alpha = a_p.to(dev)
    H = torch.empty((C, C), dtype=torch.float32, device=dev)
    ws_bytes = q4.hessian_workspace_bytes(n, C)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    delta = torch.empty((R, C // 32), dtype=torch.float32, device=dev)
    idx = torch.empty((R, C // 32), dtype=torch.int32, device=dev)
    err = torch.empty((R, C // 32), dtype=torch.float32, device=dev)
    Q = torch.empty_like(W)
    gW = torch.empty_like(W)
    gD = torch.empty_like(delta)
    packed = torch.empty((R, C // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((R, C // 32), dtype=torch.float16, device=dev)
    flush_buf = torch.ones(128 << 20, dtype=torch.float32, device=dev)   # 512 MB
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def flush():
        torch.sum(flush_buf, dim=0, out=flush_sink)

    stages = ["hessian", "scale_search", "lsq_fwd_bwd", "pack_w4a16"]

    def step(ev=None):
        def run(i, fn):
            flush()
            if ev is not None:
                ev[i][0].record(stream)
            fn()
            if ev is not None:
                ev[i][1].record(stream)
        run(0, lambda: q4.hessian(X, H, ws))
        run(1, lambda: q4.scale_search(W, H, alpha, delta, idx, err))
        run(2, lambda: q4.lsq_fwd_bwd(W, delta, G, q4.GRAD_SCALE, Q, gW, gD))
        run(3, lambda: q4.pack_w4a16(W, delta, packed, scales))

    for _ in range(args.warmup):
        step()
    q4.sync_check()

    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in stages] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    os.makedirs(OUT_DIR, exist_ok=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local, os.path.join(OUT_DIR, f"bench_clocks_r{rank}.csv")) as clk:
        start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        stop.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    q4.sync_check()
    total_ms = start.elapsed_time(stop)
    per = {s: [evs[k][i][0].elapsed_time(evs[k][i][1]) for k in range(args.steps)] for i, s in enumerate(stages)}
    mean = {s: sum(v) / len(v) for s, v in per.items()}

    # ---- end-to-end leg: the host-buffer LSQ call (qat4_lsq_fwd_bwd_host) from pinned host
    # memory and back; it streams row chunks through the GPU, uploads overlapping downloads
    Q_p = torch.empty(Q.shape, dtype=Q.dtype).pin_memory()
    gW_p = torch.empty(gW.shape, dtype=gW.dtype).pin_memory()
    gD_p = torch.empty(gD.shape, dtype=gD.dtype).pin_memory()
    d_p = delta.cpu().pin_memory()
    G_pb = G_p.view(torch.bfloat16)
    ws_host = torch.empty(q4.lsq_fwd_bwd_host_workspace_bytes(R, C, q4.QAT4_BF16), dtype=torch.uint8, device=dev)
    copy_stream = torch.cuda.Stream(device=dev)

    def e2e_step():
        q4.lsq_fwd_bwd_host(W_p, d_p, G_pb, q4.GRAD_SCALE, Q_p, gW_p, gD_p, workspace=ws_host,
                            copy_stream=copy_stream)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e2e_n = max(3, min(args.steps, 10))
    a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a_.record(stream)
    for _ in range(e2e_n):
        e2e_step()
    b_.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a_.elapsed_time(b_) / e2e_n
    h2d = W.numel() * 4 + G.numel() * 2 + delta.numel() * 4
    d2h = Q.numel() * 4 + gW.numel() * 4 + gD.numel() * 4

    # ---- whole-job aggregation (max time over ranks)
    lsq_bytes = LSQ_BYTES_PER_ELT * R * C
    job_lsq_bytes, job_lsq_ms = aggregate_over_ranks(lsq_bytes, mean["lsq_fwd_bwd"])
    job_step_units, job_total_ms = aggregate_over_ranks(1.0, total_ms)
    job_e2e_bytes, job_e2e_ms = aggregate_over_ranks(lsq_bytes, e2e_ms)
    job_h_flop, job_h_ms = aggregate_over_ranks(float(n) * C * (C + 1), mean["hessian"])
    job_groups, job_s_ms = aggregate_over_ranks(float(groups), mean["scale_search"])
    job_pack_bytes, job_p_ms = aggregate_over_ranks(PACK_BYTES_PER_ELT * R * C, mean["pack_w4a16"])

    if rank == 0:
        clocks = clk.summary()
        traffic = load_traffic(args.config)
        hbm = float(peaks["hbm_gbs"])
        tc_peak = float(peaks["bf16_tflops"])
        sm_max = float(peaks.get("sm_max_mhz", 1965.0))
        fp32_ops_peak = 148 * 128 * sm_max * 1e6            # one FP32 op per lane per clock
        search_roof = fp32_ops_peak / (SEARCH_OPS_PER_CAND * K)   # groups/s, one GPU
        lsq_gbs = job_lsq_bytes / job_lsq_ms / 1e6
        stage_lines = {
            "hessian": {"value": job_h_flop / job_h_ms / 1e9, "unit": "TFLOP/s", "ms": mean["hessian"],
                        "roofline": {"bound": "tensor", "peak": tc_peak * world, "unit": "TFLOP/s",
                                     "frac": job_h_flop / job_h_ms / 1e9 / (tc_peak * world),
                                     "algorithmic_per_launch": float(n) * C * (C + 1),
                                     "peak_kind": f"{peak_kind} bf16 burst"}},
            "scale_search": {"value": job_groups / job_s_ms * 1e3, "unit": "groups/s", "ms": mean["scale_search"],
                             "roofline": {"bound": "alu", "peak": search_roof * world, "unit": "groups/s",
                                          "frac": job_groups / job_s_ms * 1e3 / (search_roof * world),
                                          "ops_per_group": SEARCH_OPS_PER_CAND * K,
                                          "peak_kind": f"148 SM x 128 FP32 lanes x {sm_max:.0f} MHz"}},
            "lsq_fwd_bwd": {"value": lsq_gbs, "unit": "GB/s", "ms": mean["lsq_fwd_bwd"],
                            "roofline": {"bound": "hbm", "peak": hbm * world, "unit": "GB/s",
                                         "frac": lsq_gbs / (hbm * world), "bytes_per_launch": lsq_bytes,
                                         "peak_kind": f"{peak_kind} copy"}},
            "pack_w4a16": {"value": job_pack_bytes / job_p_ms / 1e6, "unit": "GB/s", "ms": mean["pack_w4a16"],
                           "roofline": {"bound": "hbm", "peak": hbm * world, "unit": "GB/s",
                                        "frac": job_pack_bytes / job_p_ms / 1e6 / (hbm * world),
                                        "bytes_per_launch": PACK_BYTES_PER_ELT * R * C,
                                        "peak_kind": f"{peak_kind} copy"}},
        }
        for st_name, line_st in stage_lines.items():
            line_st["roofline"]["traffic"] = traffic.get(st_name)
        dominant = max(stages, key=lambda s: mean[s])
        dom = stage_lines[dominant]["roofline"]
        if dominant == "hessian":
            achieved, dom_peak = job_h_flop / job_h_ms / 1e9 / world, tc_peak
        elif dominant == "scale_search":
            achieved, dom_peak = job_groups / job_s_ms * 1e3 * SEARCH_OPS_PER_CAND * K / 1e12 / world, \
                fp32_ops_peak / 1e12
        else:
            achieved = stage_lines[dominant]["value"] / world
            dom_peak = hbm
        roof_unit = {"hessian": "TFLOP/s", "scale_search": "Top/s"}.get(dominant, "GB/s")
        line = {
            "metric": METRIC, "value": lsq_gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": job_total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "1B-class MLP up-projection: W fp32 8192x2048, X bf16 262144x2048 "
                                   "(1% outlier channels x20), 101-candidate grid, G bf16",
                       "config_index": args.config, "R": R, "C": C, "n_calib": n, "K": K,
                       "parallelism": f"replicas x{world} (one layer per GPU)",
                       "l2": "flushed (512 MB read sweep) before every stage; flush time in ms_per_step only"},
            "roofline": {"kernel": dominant, "bound": dom["bound"], "achieved": achieved, "peak": dom_peak,
                         "unit": roof_unit, "frac": achieved / dom_peak,
                         "traffic": traffic.get(dominant), "traffic_unit": "bytes per launch (ncu DRAM read + write)",
                         "peak_kind": dom["peak_kind"]},
            "stages": stage_lines,
            "e2e": {"value": job_e2e_bytes / job_e2e_ms / 1e6, "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "what": "lsq_fwd_bwd_host (C ABI qat4_lsq_fwd_bwd_host) from pinned host W, G, delta to "
                            "pinned host Q, grad_W, grad_delta: row chunks of ~2 M weights, uploads on the "
                            "compute stream overlapping downloads on a copy stream"},
            # per step: Hessian pair kernel (+ the reduction of split partials when n is split),
            # search, fused LSQ, pack
            "gpu_launches": (4 + (1 if ws_bytes > 0 else 0)) * args.steps,
            "clocks": clocks,
            "input_gen_s": round(gen_s, 1),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(W_h, X_h, G_h, alpha_h)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ CPU oracle legs
def _oracle_sample(W, X, G, alpha, rows: int, hblocks: int):
    """One bounded sample of the step on the CPU oracle; returns per-stage (units, seconds)."""
    import oracle
    from int4_group_wise_b200.inputs import bf16_bits_to_f32  # noqa: F401  (inputs only)
    res = {}
    Ws, Gs = W[:rows], G[:rows]
    C = W.shape[1]
    t = time.perf_counter()
    Hd = np.zeros((C, C), np.float32)
    for g in range(hblocks):
        Hd[32 * g:32 * g + 32, 32 * g:32 * g + 32] = oracle.hessian_block(X, 32 * g, 32, 32 * g, 32)
    res["hessian"] = (float(X.shape[0]) * 32 * 33 * hblocks, time.perf_counter() - t)
    Wsearch = Ws[:, :32 * hblocks]
    t = time.perf_counter()
    d, i, b = oracle.scale_search(Wsearch, Hd[:32 * hblocks, :32 * hblocks], alpha)
    res["scale_search"] = (float(Wsearch.size // 32), time.perf_counter() - t)
    delta = (np.abs(Ws).reshape(rows, -1, 32).max(axis=2) / np.float32(7)).astype(np.float32)
    t = time.perf_counter()
    oracle.lsq_fwd(Ws, delta)
    oracle.lsq_bwd(Ws, delta, Gs, float(np.float32(1 / np.sqrt(224))))
    res["lsq_fwd_bwd"] = (LSQ_BYTES_PER_ELT * Ws.size, time.perf_counter() - t)
    t = time.perf_counter()
    oracle.pack_w4a16(Ws, delta)
    res["pack_w4a16"] = (PACK_BYTES_PER_ELT * Ws.size, time.perf_counter() - t)
    return res


def cpu_baseline(W, X, G, alpha, rows=2048, hblocks=8):
    import oracle
    cores = oracle.set_threads(0)
    res = _oracle_sample(W, X, G, alpha, rows, hblocks)
    u, s = res["lsq_fwd_bwd"]
    return {"value": u / s / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"rows 0..{rows - 1} of W for LSQ/pack ({rows}x{W.shape[1]}); "
                      f"{hblocks} diagonal 32x32 Hessian blocks over all {X.shape[0]} rows; "
                      f"scale search on those {hblocks} groups x {rows} rows",
            "stages": {"hessian_gflops": res["hessian"][0] * 1e-9 / res["hessian"][1] * 1.0,
                       "scale_search_groups_per_s": res["scale_search"][0] / res["scale_search"][1],
                       "lsq_fwd_bwd_gbs": u / s / 1e9,
                       "pack_w4a16_gbs": res["pack_w4a16"][0] / res["pack_w4a16"][1] / 1e9}}


def run_reference(args):
    """The oracle as it stands, on the host cores, on bounded samples of the same workload."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    from int4_group_wise_b200 import inputs
    wl = inputs.workload(args.config)
    m = wl.matrices[0]
    W, G, alpha = wl.weight(m), wl.grad(m), wl.alpha()
    X = wl.activations(m.x_name, n=16384)          # a row sample of the calibration set
    cores = oracle.set_threads(0)
    rows = 512
    for _ in range(args.warmup):
        _oracle_sample(W, X, G, alpha, rows, 2)
    tot_u = tot_s = 0.0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r = _oracle_sample(W, X, G, alpha, rows, 2)
        tot_u += r["lsq_fwd_bwd"][0]
        tot_s += r["lsq_fwd_bwd"][1]
    wall = time.perf_counter() - t0
    v = tot_u / tot_s / 1e9
    sample = (f"per step: rows 0..{rows - 1} of W (LSQ, pack); 2 diagonal Hessian blocks over 16384 "
              f"calibration rows; scale search on 2 groups x {rows} rows")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "1B-class MLP up-projection (CPU oracle, row sample)", "config_index": args.config},
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_stack(args):
    """A whole decoder stack: config 3 (1B-class, 16 layers, 112 matrices, every matrix searched,
    64 calibration Hessians of n = 65536) or config 4 (8B-class, 32 layers, 224 matrices, layer 0's
    4 Hessians of n = 131072 and 7 searches, RTN scales elsewhere).  A step is every Hessian, every
    search, one fused LSQ step over every weight and the W4A16 export of every matrix; each stage's
    launches (independent matrices) go round-robin to four streams and the stage is timed with CUDA
    events on the launching stream, which waits for all four (every stage's inputs are far larger
    than L2).  Inputs are drawn on the GPU with torch's CUDA generator (seed 0) with the workload's shapes
    and distributions (weights N(0, sigma); X rows N(0, 1) with round(1% d) outlier channels x20,
    rounded to bf16; G N(0, 1e-3) in bf16); parity at these shapes is covered by the workload tests
    on the host-seeded tensors.  One JSON line."""
    import torch

    import int4_group_wise_b200 as q4
    from int4_group_wise_b200 import inputs

    if args.config not in (3, 4):
        raise SystemExit("--variant stack runs config 3 or 4")
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks, peak_kind = load_peaks()
    wl = inputs.workload(args.config)
    gen = torch.Generator(device=dev).manual_seed(layer_seed(rank))
    t0 = time.time()

    def randn(shape, sigma):
        return torch.randn(shape, generator=gen, device=dev, dtype=torch.float32).mul_(sigma)

    X, H = {}, {}
    for x_name, d in wl.calib.items():
        x = torch.randn((wl.n_calib, d), generator=gen, device=dev, dtype=torch.float32)
        cols = torch.randperm(d, generator=gen, device=dev)[:wl.outliers.get(x_name, 0)]
        x[:, cols] *= 20.0
        X[x_name] = x.to(torch.bfloat16)
        del x
        H[x_name] = torch.empty((d, d), dtype=torch.float32, device=dev)
    ws = torch.empty(max([q4.hessian_workspace_bytes(wl.n_calib, d) for d in wl.calib.values()] + [16]),
                     dtype=torch.uint8, device=dev)
    alpha = torch.from_numpy(wl.alpha()).to(dev)
    mats = []
    for m in wl.matrices:
        W = randn((m.d_out, m.d_in), wl.weight_sigma)
        G = randn((m.d_out, m.d_in), 1e-3).to(torch.bfloat16)
        # scales of matrices that are not searched: round-to-nearest (alpha = 1), fl(max|w_g| / 7)
        delta = (W.abs().view(m.d_out, m.d_in // 32, 32).amax(-1) / 7.0).contiguous()
        mats.append(dict(m=m, W=W, G=G, delta=delta, idx=torch.empty(delta.shape, dtype=torch.int32, device=dev),
                         err=torch.empty_like(delta), Q=torch.empty_like(W), gW=torch.empty_like(W),
                         gD=torch.empty_like(delta),
                         packed=torch.empty((m.d_out, m.d_in // 2), dtype=torch.uint8, device=dev),
                         scales=torch.empty(delta.shape, dtype=torch.float16, device=dev)))
    gen_s = time.time() - t0
    searched = [e for e in mats if e["m"].name in wl.searched]
    n_weights = sum(e["W"].numel() for e in mats)
    hess_flop = sum(float(wl.n_calib) * d * (d + 1) for d in wl.calib.values())
    groups = sum(e["W"].numel() // 32 for e in searched)
    K = int(alpha.numel())
    stream = torch.cuda.current_stream(dev)
    # independent matrices go round-robin to NS side streams (the small k/v launches alone leave
    # most SMs idle); each stage starts after the previous one on every stream and ends when all
    # side streams are done; each stream has its own Hessian workspace
    NS = 4
    side = [torch.cuda.Stream(device=dev) for _ in range(NS)]
    wss = [ws] + [torch.empty_like(ws) for _ in range(NS - 1)]

    def fan(launches):
        go = torch.cuda.Event()
        go.record(stream)
        for s_ in side:
            s_.wait_event(go)
        for i, launch in enumerate(launches):
            with torch.cuda.stream(side[i % NS]):
                launch(i % NS)
        for s_ in side:
            done = torch.cuda.Event()
            done.record(s_)
            stream.wait_event(done)

    def stage_hessian():
        fan([lambda j, x=x_name: q4.hessian(X[x], H[x], wss[j]) for x_name in wl.calib])

    def stage_search():
        fan([lambda j, e=e: q4.scale_search(e["W"], H[e["m"].x_name], alpha, e["delta"], e["idx"], e["err"])
             for e in searched])

    def stage_lsq():
        fan([lambda j, e=e: q4.lsq_fwd_bwd(e["W"], e["delta"], e["G"], q4.GRAD_SCALE, e["Q"], e["gW"], e["gD"])
             for e in mats])

    def stage_pack():
        fan([lambda j, e=e: q4.pack_w4a16(e["W"], e["delta"], e["packed"], e["scales"]) for e in mats])

    stages = [("hessian", stage_hessian), ("scale_search", stage_search), ("lsq_fwd_bwd", stage_lsq),
              ("pack_w4a16", stage_pack)]

    def step(ev=None):
        for i, (_, fn) in enumerate(stages):
            if ev is not None:
                ev[i][0].record(stream)
            fn()
            if ev is not None:
                ev[i][1].record(stream)

    for _ in range(args.warmup):
        step()
    q4.sync_check()
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in stages] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with ClockSampler(local, os.path.join(OUT_DIR, f"bench_stack_clocks_r{rank}.csv")) as clk:
        start.record(stream)
        for k in range(args.steps):
            step(evs[k])
        stop.record(stream)
        torch.cuda.synchronize()
    q4.sync_check()
    total_ms = start.elapsed_time(stop) / args.steps
    mean = {name: sum(evs[k][i][0].elapsed_time(evs[k][i][1]) for k in range(args.steps)) / args.steps
            for i, (name, _) in enumerate(stages)}
    hbm = float(peaks["hbm_gbs"])
    tc_peak = float(peaks["bf16_tflops"])
    sm_max = float(peaks.get("sm_max_mhz", 1965.0))
    search_roof = 148 * 128 * sm_max * 1e6 / (SEARCH_OPS_PER_CAND * K)
    lsq_bytes = LSQ_BYTES_PER_ELT * n_weights
    pack_bytes = PACK_BYTES_PER_ELT * n_weights
    lsq_gbs = lsq_bytes / mean["lsq_fwd_bwd"] / 1e6
    st = {
        "hessian": {"value": hess_flop / mean["hessian"] / 1e9, "unit": "TFLOP/s", "ms": mean["hessian"],
                    "launches": len(wl.calib), "flop": hess_flop,
                    "frac": hess_flop / mean["hessian"] / 1e9 / tc_peak},
        "scale_search": {"value": groups / mean["scale_search"] * 1e3, "unit": "groups/s",
                         "ms": mean["scale_search"], "launches": len(searched), "groups": groups,
                         "frac": groups / mean["scale_search"] * 1e3 / search_roof},
        "lsq_fwd_bwd": {"value": lsq_gbs, "unit": "GB/s", "ms": mean["lsq_fwd_bwd"], "launches": len(mats),
                        "bytes": lsq_bytes, "frac": lsq_gbs / hbm},
        "pack_w4a16": {"value": pack_bytes / mean["pack_w4a16"] / 1e6, "unit": "GB/s", "ms": mean["pack_w4a16"],
                       "launches": len(mats), "bytes": pack_bytes,
                       "frac": pack_bytes / mean["pack_w4a16"] / 1e6 / hbm},
    }
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": lsq_gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "variant": "stack", "dtype": "f32", "data": "synthetic (drawn on the GPU)",
            "config": {"workload": wl.title, "config_index": args.config, "matrices": len(mats),
                       "weights": n_weights, "hessians": len(wl.calib), "n_calib": wl.n_calib,
                       "searched_matrices": len(searched), "K": K,
                       "streams": NS, "l2": "every stage's inputs are larger than L2; no flush"},
            "stages": st, "peaks": {"hbm_gbs": hbm, "bf16_tflops": tc_peak, "kind": peak_kind,
                                    "search_roof_groups_per_s": search_roof},
            "gpu_launches": (len(wl.calib) * 2 + len(searched) + 2 * len(mats)) * args.steps,
            "clocks": clk.summary(), "input_gen_s": round(gen_s, 1)}), flush=True)


def run_per_channel(args):
    """The per-channel variant (one scale per row) on the same layer shape: fused LSQ step and
    W4A16 export, each launch timed with CUDA events after an L2 flush; one JSON line."""
    import torch

    import int4_group_wise_b200 as q4
    from int4_group_wise_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    wl = inputs.workload(args.config)
    m = wl.matrices[0]
    W_h, G_h = wl.weight(m), wl.grad(m)
    R, C = W_h.shape
    W = torch.from_numpy(W_h).to(dev)
    G = torch.from_numpy(G_h.view(np.int16)).to(dev).view(torch.bfloat16)
    delta = (W.abs().amax(dim=1) / 7).contiguous()
    Q, gW = torch.empty_like(W), torch.empty_like(W)
    gD = torch.empty_like(delta)
    packed = torch.empty((R, C // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((R,), dtype=torch.float16, device=dev)
    flush_buf = torch.ones(128 << 20, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    lsq = lambda: q4.lsq_fwd_bwd_rowwise(W, delta, G, None, Q, gW, gD)
    pack = lambda: q4.pack_w4a16_rowwise(W, delta, packed, scales)

    def timed(fn, n):
        ts = []
        for _ in range(n):
            torch.sum(flush_buf, dim=0, out=sink)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            ts.append((a, b))
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ts) / n

    for _ in range(args.warmup):
        lsq()
        pack()
    q4.sync_check()
    lsq_ms = timed(lsq, args.steps)
    pack_ms = timed(pack, args.steps)
    q4.sync_check()
    lsq_bytes = (4 + 2 + 4 + 4) * R * C + 8 * R
    pack_bytes = 4.5 * R * C + 6 * R

    # per-channel scale search on the layer's Hessian (full C x C quadratic form per row)
    X = torch.from_numpy(wl.activations(m.x_name).view(np.int16)).to(dev).view(torch.bfloat16)
    H = q4.hessian(X)
    del X
    alpha_h = wl.alpha()
    alpha = torch.from_numpy(alpha_h).to(dev)
    sd = torch.empty((R,), dtype=torch.float32, device=dev)
    si = torch.empty((R,), dtype=torch.int32, device=dev)
    se = torch.empty((R,), dtype=torch.float32, device=dev)
    ws = torch.empty(q4.lib().qat4_scale_search_rowwise_workspace_bytes(R, C), dtype=torch.uint8, device=dev)
    search = lambda: q4.scale_search_rowwise(W, H, alpha, sd, si, se, ws)
    search()
    q4.sync_check()
    search_ms = timed(search, 3)
    q4.sync_check()
    # code changes between consecutive candidates, from a 64-row sample (the sweep's work model)
    rows = np.arange(0, R, max(1, R // 64))[:64]
    Ws = W_h[rows]
    bs = (np.abs(Ws).max(axis=1) / np.float32(7)).astype(np.float32)
    prev, changes = None, 0
    for a in alpha_h:
        dk = (a * bs).astype(np.float32)[:, None]
        qk = np.clip(np.rint(Ws / dk), -8, 7)
        if prev is not None:
            changes += int((qk != prev).sum())
        prev = qk
    changes_per_row = changes / len(rows)
    K = alpha_h.size
    dfma = 2.0 * R * C * C + R * changes_per_row * C + 3.0 * R * C * K
    h_row_bytes = R * changes_per_row * C * 4.0
    fp64_peak = 148 * 64 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
    hbm = float(peaks["hbm_gbs"])
    v_lsq, v_pack = lsq_bytes / lsq_ms / 1e6, pack_bytes / pack_ms / 1e6
    print(json.dumps({
        "metric": "per-channel LSQ fwd+bwd GB/s; per-channel W4A16 pack GB/s", "value": v_lsq, "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
        "variant": "per-channel (one scale per row)", "data": "synthetic", "dtype": "f32",
        "config": {"workload": f"W fp32 {R}x{C}, G bf16, one scale per row", "config_index": args.config,
                   "l2": "flushed (512 MB read sweep) before every launch"},
        "stages": {"lsq_fwd_bwd_rowwise": {"value": v_lsq, "unit": "GB/s", "ms": lsq_ms,
                                           "bytes_per_launch": lsq_bytes, "frac": v_lsq / hbm},
                   "pack_w4a16_rowwise": {"value": v_pack, "unit": "GB/s", "ms": pack_ms,
                                          "bytes_per_launch": pack_bytes, "frac": v_pack / hbm},
                   "scale_search_rowwise": {"value": R / search_ms * 1e3, "unit": "rows/s", "ms": search_ms,
                                            "K": K, "code_changes_per_row": changes_per_row,
                                            "fp64_fma_per_launch": dfma,
                                            "fp64_frac": dfma / (search_ms * 1e-3) / fp64_peak,
                                            "h_row_bytes_per_launch": h_row_bytes,
                                            "h_row_gbs": h_row_bytes / search_ms / 1e6,
                                            "note": "exact binary64 sweep; fp64_frac against 148 SM x 64 "
                                                    "FP64 FMA/clock; the H rows re-read per code change "
                                                    "come from L2"}},
        "peak": {"hbm_gbs": hbm, "kind": f"{peak_kind} copy"}}), flush=True)


def run_w4a16_decode(args):
    """Decode on the W4A16 export of the 8B-class stack (32 layers x {q, k, v, o, gate, up,
    down}): one step = the 224 GEMVs of one token batch (M = 1 and M = 4), replayed from a CUDA
    graph.  The seeded layer-0 weights, packed once, are copied into 32 distinct layer buffers
    (3.9 GB of codes and scales, 31x L2), so every step streams its bytes from HBM."""
    import torch

    import int4_group_wise_b200 as q4
    from int4_group_wise_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    wl = inputs.workload(4)
    layer0 = [m for m in wl.matrices if m.name.startswith("L0.")]
    n_layers = len(wl.matrices) // len(layer0) if args.layers is None else args.layers
    base = []
    for m in layer0:
        W = torch.from_numpy(wl.weight(m)).to(dev)
        R, C = W.shape
        delta = (W.abs().reshape(R, C // 32, 32).amax(dim=2) / 7).contiguous()
        base.append(q4.pack_w4a16(W, delta))
        del W, delta
    q4.sync_check()
    layers = [[(p.clone(), sc.clone()) for p, sc in base] for _ in range(n_layers)]
    del base
    torch.cuda.synchronize()
    shapes = [(m.d_out, m.d_in) for m in layer0]
    weights = sum(R * C for R, C in shapes) * n_layers
    code_bytes = sum(R * C // 2 + R * (C // 32) * 2 for R, C in shapes) * n_layers
    stream = torch.cuda.Stream(dev)
    flush_buf = torch.ones(128 << 20, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    results = {}
    for M in (1, 4):
        xs = {C: torch.from_numpy(inputs.activations(M, C, seed=M, cfg=4, name=f"decode_x/{C}").view(np.int16))
              .to(dev).view(torch.bfloat16) for C in sorted({C for _, C in shapes})}
        ys = [torch.empty((M, R), dtype=torch.float32, device=dev) for R, _ in shapes]

        def step():
            for lay in layers:
                for (R, C), (p, sc), y in zip(shapes, lay, ys):
                    q4.w4a16_gemv(xs[C], p, sc, y, stream=stream)

        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                step()
        stream.synchronize()
        q4.sync_check(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step()
        for _ in range(args.warmup):
            g.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            for _ in range(args.steps):
                g.replay()
            b.record(stream)
        torch.cuda.synchronize()
        q4.sync_check(stream)
        step_ms = a.elapsed_time(b) / args.steps
        step_bytes = code_bytes + n_layers * sum(M * C * 2 + M * R * 4 for R, C in shapes)
        # each shape on its own, L2 flushed before every launch (layer 0's buffers)
        per_shape = {}
        for m, (R, C), (p, sc), y in zip(layer0, shapes, layers[0], ys):
            ts = []
            with torch.cuda.stream(stream):
                for _ in range(max(args.steps, 10)):
                    torch.sum(flush_buf, dim=0, out=sink)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    q4.w4a16_gemv(xs[C], p, sc, y, stream=stream)
                    e1.record(stream)
                    ts.append((e0, e1))
            torch.cuda.synchronize()
            us = 1e3 * sum(e0.elapsed_time(e1) for e0, e1 in ts) / len(ts)
            nbytes = R * C // 2 + R * (C // 32) * 2 + M * C * 2 + M * R * 4
            per_shape[m.name.split(".")[1]] = {"shape": [R, C], "us": us, "gbs": nbytes / us / 1e3,
                                              "frac": nbytes / us / 1e3 / hbm}
        del g
        gbs = step_bytes / step_ms / 1e6
        results[M] = {"tokens_per_s": M * 1e3 / step_ms, "ms_per_step": step_ms, "gbs": gbs, "frac": gbs / hbm,
                      "bytes_per_step": step_bytes, "launches_per_step": len(shapes) * n_layers,
                      "per_shape_l2_flushed": per_shape}
    r1 = results[1]
    print(json.dumps({
        "metric": "W4A16 decode GEMV GB/s over the 8B-class stack (M = 1)", "value": r1["gbs"], "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": r1["ms_per_step"],
        "higher_is_better": True, "variant": "w4a16-decode", "data": "synthetic", "dtype": "bf16 x int4 -> f32",
        "config": {"workload": f"8B-class stack, {n_layers} layers x 7 matrices, {weights} weights, "
                               "group-32 export, decode batch M = 1 and 4",
                   "l2": "inputs 31x L2 (distinct layer buffers); per-shape times flush L2 before every launch"},
        "roofline": {"bound": "hbm", "achieved": r1["gbs"], "peak": hbm, "unit": "GB/s", "frac": r1["frac"],
                     "peak_kind": f"{peak_kind} copy"},
        "gpu_launches": r1["launches_per_step"] * args.steps,
        "stages": {f"M={M}": v for M, v in results.items()}}), flush=True)


def run_fq_gemm(args):
    """The fused fake-quant forward GEMM of a QAT step on the 1B-class up-projection (W fp32
    8192x2048, searched-range scales) for a micro-batch of --tokens tokens: TFLOP/s against the
    bf16 tensor peak, each launch timed with CUDA events after an L2 flush.  For context the
    same product is also timed unfused through libraries: the LSQ forward, a cast to bf16 and a
    cuBLAS bf16 GEMM."""
    import torch

    import int4_group_wise_b200 as q4
    from int4_group_wise_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    wl = inputs.workload(1)
    m = wl.matrices[0]
    W_h = wl.weight(m)
    R, C = W_h.shape
    T = args.tokens
    rng = np.random.default_rng(1)
    D_h = (np.abs(W_h).reshape(R, C // 32, 32).max(axis=2) / np.float32(7) *
           rng.uniform(0.5, 1.0, (R, C // 32))).astype(np.float32)
    X = torch.from_numpy(wl.activations(m.x_name, n=T).view(np.int16)).to(dev).view(torch.bfloat16)
    W = torch.from_numpy(W_h).to(dev)
    D = torch.from_numpy(D_h).to(dev)
    Y = torch.empty((T, R), dtype=torch.float32, device=dev)
    Q = torch.empty_like(W)
    flush_buf = torch.ones(128 << 20, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def timed(fn, n):
        ts = []
        for _ in range(n):
            torch.sum(flush_buf, dim=0, out=sink)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            ts.append((a, b))
        torch.cuda.synchronize()
        return sorted(a.elapsed_time(b) for a, b in ts)

    fused = lambda: q4.fq_gemm(X, W, D, Y)

    def unfused():
        q4.lsq_fwd(W, D, Q)
        torch.matmul(X, Q.to(torch.bfloat16).t())

    for _ in range(args.warmup):
        fused()
        unfused()
    q4.sync_check()
    with ClockSampler(0) as clk:
        t_f = timed(fused, args.steps)
    t_u = timed(unfused, max(3, args.steps // 2))
    q4.sync_check()
    flop = 2.0 * T * R * C
    ms = statistics.median(t_f)
    tf = flop / ms / 1e9
    peak = float(peaks["bf16_tflops"])
    print(json.dumps({
        "metric": "fused fake-quant GEMM TFLOP/s (Y = X bf16(Q_Delta(W))^T)", "value": tf, "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "variant": "fq-gemm", "data": "synthetic", "dtype": "bf16 x bf16 -> f32 (quantizer f32)",
        "config": {"workload": f"1B-class up-projection W fp32 {R}x{C}, X bf16 {T}x{C} (micro-batch of {T} tokens)",
                   "l2": "flushed (512 MB read sweep) before every launch"},
        "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                     "flop_per_launch": flop, "peak_kind": f"{peak_kind} bf16 burst"},
        "ms_min_median_max": [t_f[0], ms, t_f[-1]],
        "unfused_library_ms": statistics.median(t_u),
        "unfused_library": "qat4_lsq_fwd + cast to bf16 + torch.matmul (cuBLAS bf16), same product",
        "gpu_launches": args.steps, "clocks": clk.summary()}), flush=True)


def run_hessian_split(args):
    """The Hessian of the 1B-class up-projection's calibration set (X bf16 262144x2048) with its
    rows split across the N ranks: each rank computes the partial of its shard on the tensor
    cores, then one NCCL all-reduce sums the partials (16.8 MB).  Total work is fixed as N grows
    (strong scaling); the time of a step is the slowest rank's, measured with CUDA events around
    partial + all-reduce, L2 flushed before each step."""
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    import int4_group_wise_b200 as q4
    from int4_group_wise_b200 import distributed, inputs

    rank, world, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world == 1:   # a one-rank group still runs the all-reduce path
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29533")
    dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev, rank=rank, world_size=world)
    try:
        peaks, peak_kind = load_peaks()
        wl = inputs.workload(1)
        m = wl.matrices[0]
        n, C = wl.n_calib, wl.calib[m.x_name]
        lo, hi = distributed.shard_rows(n, world, rank)
        Xb = wl.activations(m.x_name)[lo:hi]
        X = torch.from_numpy(np.ascontiguousarray(Xb).view(np.int16)).to(dev).view(torch.bfloat16)
        del Xb
        H = torch.empty((C, C), dtype=torch.float32, device=dev)
        ws = torch.empty(max(1, q4.hessian_workspace_bytes(hi - lo, C)), dtype=torch.uint8, device=dev)
        flush_buf = torch.ones(128 << 20, dtype=torch.float32, device=dev)
        sink = torch.empty((), dtype=torch.float32, device=dev)
        stream = torch.cuda.current_stream(dev)
        step = lambda: distributed.hessian_sharded(X, n, H=H, workspace=ws)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        q4.sync_check()
        ts = []
        with ClockSampler(local) as clk:
            for _ in range(args.steps):
                torch.sum(flush_buf, dim=0, out=sink)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                dist.barrier()
                a.record(stream)
                step()
                b.record(stream)
                ts.append((a, b))
            torch.cuda.synchronize()
        q4.sync_check()
        ms_local = statistics.median(a.elapsed_time(b) for a, b in ts)
        _, ms = aggregate_over_ranks(0.0, ms_local)
        flop = float(n) * C * (C + 1)
        tf = flop / ms / 1e9
        peak = float(peaks["bf16_tflops"]) * world
        if rank == 0:
            print(json.dumps({
                "metric": "split-n Hessian TFLOP/s (partials + NCCL all-reduce)", "value": tf, "unit": "TFLOP/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "strong", "variant": "hessian-split", "data": "synthetic",
                "dtype": "bf16 x bf16 -> f32",
                "config": {"workload": f"1B-class up-projection calibration set X bf16 {n}x{C}, rows split "
                                       f"over {world} GPU(s)", "parallelism": f"split-n x{world} + all-reduce",
                           "l2": "flushed (512 MB read sweep) before every step"},
                "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                             "peak_kind": f"{peak_kind} bf16 burst x {world} GPU(s)"},
                "allreduce_bytes": C * C * 4, "gpu_launches": args.steps * (1 if q4.hessian_workspace_bytes(
                    hi - lo, C) == 0 else 2), "clocks": clk.summary()}), flush=True)
    finally:
        dist.destroy_process_group()


def run_refine(args):
    """The full-objective refinement (one coordinate-descent sweep over the groups of every row)
    on the 1B-class up-projection, starting from the GPU search's indices; each launch timed with
    CUDA events after an L2 flush.  Work model in binary64 FMAs: V = E H (R C^2), every
    candidate of every group (R G K (528 + 32)) and the v updates of the groups that move
    (moves x 32 C)."""
    import torch

    import int4_group_wise_b200 as q4
    from int4_group_wise_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    wl = inputs.workload(1)
    m = wl.matrices[0]
    W = torch.from_numpy(wl.weight(m)).to(dev)
    R, C = W.shape
    X = torch.from_numpy(wl.activations(m.x_name).view(np.int16)).to(dev).view(torch.bfloat16)
    H = q4.hessian(X)
    del X
    alpha = torch.from_numpy(wl.alpha()).to(dev)
    K = alpha.numel()
    _, idx0, _ = q4.scale_search(W, H, alpha)
    idx = idx0.clone()
    delta = torch.empty((R, C // 32), dtype=torch.float32, device=dev)
    obj = torch.empty((R,), dtype=torch.float64, device=dev)
    ws = torch.empty(q4.lib().qat4_refine_workspace_bytes(R, C), dtype=torch.uint8, device=dev)
    q4.refine(W, H, alpha, idx, 0, delta, obj, ws)
    obj0 = obj.clone()
    flush_buf = torch.ones(128 << 20, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def one():
        idx.copy_(idx0)
        q4.refine(W, H, alpha, idx, 1, delta, obj, ws)

    for _ in range(args.warmup):
        one()
    q4.sync_check()
    ts = []
    with ClockSampler(0) as clk:
        for _ in range(args.steps):
            idx.copy_(idx0)
            torch.sum(flush_buf, dim=0, out=sink)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            q4.refine(W, H, alpha, idx, 1, delta, obj, ws)
            b.record(stream)
            ts.append((a, b))
        torch.cuda.synchronize()
    q4.sync_check()
    ms = statistics.median(a.elapsed_time(b) for a, b in ts)
    G = C // 32
    moves = int((idx != idx0).sum().item())
    dfma = float(R) * C * C + float(R) * G * K * 560 + float(moves) * 32 * C
    fp64_peak = 148 * 64 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
    gain = (1.0 - obj / obj0)
    print(json.dumps({
        "metric": "full-objective refinement, one sweep: groups/s", "value": R * G / ms * 1e3, "unit": "groups/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "variant": "refine", "data": "synthetic", "dtype": "f64 (exact f32 codes)",
        "config": {"workload": f"1B-class up-projection W fp32 {R}x{C}, H of 262144 calibration rows, K={K}",
                   "l2": "flushed (512 MB read sweep) before every launch"},
        "roofline": {"bound": "fp64", "achieved": dfma / (ms * 1e-3) / 1e12, "peak": fp64_peak / 1e12,
                     "unit": "T FMA/s", "frac": dfma / (ms * 1e-3) / fp64_peak,
                     "peak_kind": "148 SM x 64 FP64 FMA/clock at max SM clock"},
        "fp64_fma_per_launch": dfma, "groups_moved": moves, "groups": R * G,
        "objective_gain_median": float(gain.median().item()), "objective_gain_max": float(gain.max().item()),
        "gpu_launches": 3 * args.steps, "clocks": clk.summary()}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--variant", choices=["group32", "per-channel", "w4a16-decode", "fq-gemm", "hessian-split",
                                          "refine", "stack"],
                    default="group32",
                    help="per-channel: time the one-scale-per-row LSQ step and export instead; "
                         "w4a16-decode: time the inference GEMV on the packed 8B-class stack; "
                         "fq-gemm: time the fused fake-quant forward GEMM; "
                         "hessian-split: the calibration Hessian with its rows split over the ranks; "
                         "refine: one sweep of the full-objective refinement; "
                         "stack: the whole decoder stack of --config 3 or 4")
    ap.add_argument("--tokens", type=int, default=8192, help="fq-gemm: tokens of the micro-batch")
    ap.add_argument("--layers", type=int, default=None,
                    help="w4a16-decode: number of layers of the 8B-class stack (default: all 32)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.variant == "per-channel":
        run_per_channel(args)
    elif args.variant == "w4a16-decode":
        run_w4a16_decode(args)
    elif args.variant == "fq-gemm":
        run_fq_gemm(args)
    elif args.variant == "hessian-split":
        run_hessian_split(args)
    elif args.variant == "refine":
        run_refine(args)
    elif args.variant == "stack":
        run_stack(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
