"""Benchmark of the group-32 INT4 quantizer path on B200.

One step = one pass of the whole path over a workload, inputs resident in HBM:

    H = hessian(X) for every calibration input
      -> (delta, idx, err) = scale_search(W, H, alpha) for every searched matrix
      -> (Q, grad_W, grad_delta) = lsq_fwd_bwd(W, delta, G) for every matrix
      -> (packed, scales) = pack_w4a16(W, delta) for every matrix

The headline step is the 8B-class decoder stack (hidden 4096, MLP 14336, 32
layers, 224 matrices, 6.98 G fp32 weights): layer 0's four calibration
Hessians from 131072 rows, layer 0's seven scale searches over the
101-candidate grid, one fused LSQ step over all 224 matrices (99.5 GB moved)
and the W4A16 export of all 224 (the largest configuration that fits one
GPU).  Each stage's launches go round-robin to four streams; every stage's
inputs are larger than L2.  After it, the 1B-class MLP up-projection
(8192x2048, X 262144x2048) and the heavy-tailed down-projection (2048x8192,
X 262144x8192, 201 candidates) are timed the same way, one launch per stage,
with L2 flushed before every stage, and reported under `stages.config1` and
`stages.config2`.  Per-stage times are CUDA events on the launching stream.

The headline `value` is the first metric of the path, LSQ fwd+bwd GB/s
(14.25 algorithmic bytes per weight); the Hessian TFLOP/s, scale-search
groups/s and pack GB/s are in `stages`, each with its roofline.  With N GPUs
every rank runs its own seeded copy of the workload (independent problems,
weak scaling, no collective on the data path); the value is the bytes of all
ranks divided by the slowest rank's time.  `--gpus N` started without a
launcher re-executes itself under torch.distributed.run with N ranks.

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
LSQ_BYTES_PER_ELT_F32G = 16.25  # the same with an fp32 G
PACK_BYTES_PER_ELT = 4.6875     # W 4 + delta 4/32 + nibbles 0.5 + fp16 scale 2/32
SEARCH_OPS_PER_CAND = 720       # 528 FMA quadratic form + 32 x (div, rint, min, max, mul, sub)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


# --------------------------------------------------------------------------- setup
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic_path.md")
# where the nvidia-smi clock samples of the timed regions are written (one CSV per config and rank)
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


def load_traffic(config: int, p=None):
    """Per-stage DRAM bytes per step from the committed table of ncu captures.

    The table holds, per configuration and kernel, dram__bytes_read.sum + dram__bytes_write.sum
    summed over the launches of one step, with the sources' hash at capture time.  It is a stored
    figure: a stage gets {"bytes", "source"} only while the kernel sources still hash to the
    recorded value, and nothing (null in the line) after any change to them."""
    if not os.path.exists(TRAFFIC_FILE):
        return {}
    text = open(TRAFFIC_FILE).read()
    recorded = next((ln.split(":", 1)[1].strip() for ln in text.splitlines() if ln.startswith("source_hash:")), None)
    if recorded is None or recorded != source_hash():
        return {}
    per = {}
    for ln in text.splitlines():
        f = [x.strip() for x in ln.strip().strip("|").split("|")]
        if len(f) == 3 and f[0].isdigit() and f[2].isdigit():
            per[(int(f[0]), f[1])] = int(f[2])
    src = f"stored ncu capture ({os.path.relpath(TRAFFIC_FILE, ROOT)}, source hash {recorded})"
    return {st: {"bytes": sum(per[(config, k)] for k in ks if (config, k) in per), "source": src}
            for st, ks in STAGE_KERNELS.items() if (config, ks[0]) in per}


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


def relaunch_ranks(n: int, argv) -> int:
    """Runs this script as n ranks on this node under torch.distributed.run (rendezvous on
    127.0.0.1, a free port); returns the launcher's exit status."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    return subprocess.run(cmd).returncode


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


# ------------------------------------------------------------ device workloads
class DeviceProblem:
    """One workload drawn on the GPU with torch's CUDA generator: every matrix's W (fp32,
    N(0, sigma) or Student-t(3) * 0.01), G (N(0, 1e-3); bf16, fp32 for the small layer), its
    scales (the search writes those of the searched matrices; the others get round-to-nearest
    scales fl(max|w_g| / 7)) and outputs, and per distinct layer input the calibration X (rows
    N(0, 1), round(1% d) outlier channels x20 or lognormal channel scales, rounded to bf16) and
    H.  Host-generating the 8B-class stack (28 GB of weights) would dominate the run; parity at
    these shapes is covered by the tests on the host-seeded tensors."""

    def __init__(self, cfg: int, dev, seed: int, q4, streams: int):
        import torch
        from int4_group_wise_b200 import inputs
        self.cfg = cfg
        self.wl = wl = inputs.workload(cfg)
        self.dev = dev
        gen = torch.Generator(device=dev).manual_seed(1000 * cfg + seed)
        randn = lambda shape: torch.randn(shape, generator=gen, device=dev, dtype=torch.float32)
        t0 = time.time()
        self.X, self.H = {}, {}
        for x_name, d in wl.calib.items():
            x = randn((wl.n_calib, d))
            scale = torch.ones(d, device=dev)
            k = wl.outliers.get(x_name) or 0
            if k:
                scale[torch.randperm(d, generator=gen, device=dev)[:k]] = 20.0
            if wl.lognormal_channels:
                scale *= randn((d,)).exp_()
            x *= scale
            self.X[x_name] = x.to(torch.bfloat16)
            del x
            self.H[x_name] = torch.empty((d, d), dtype=torch.float32, device=dev)
        self.n_ws = max([q4.hessian_workspace_bytes(wl.n_calib, d) for d in wl.calib.values()] + [16])
        self.ws = [torch.empty(self.n_ws, dtype=torch.uint8, device=dev) for _ in range(streams)]
        self.alpha = torch.from_numpy(wl.alpha()).to(dev)
        self.mats = []
        for m in wl.matrices:
            shape = (m.d_out, m.d_in)
            if wl.weight_student_t:
                chi2 = randn(shape).square_()
                chi2 += randn(shape).square_()
                chi2 += randn(shape).square_()
                W = randn(shape).div_(chi2.div_(3.0).sqrt_()).mul_(0.01)
                del chi2
            else:
                W = randn(shape).mul_(wl.weight_sigma)
            G = randn(shape).mul_(1e-3)
            if wl.g_dtype == "bf16":
                G = G.to(torch.bfloat16)
            delta = (W.abs().view(m.d_out, m.d_in // 32, 32).amax(-1) / 7.0).contiguous()
            self.mats.append(dict(
                m=m, W=W, G=G, delta=delta, idx=torch.empty(delta.shape, dtype=torch.int32, device=dev),
                err=torch.empty_like(delta), Q=torch.empty_like(W), gW=torch.empty_like(W),
                gD=torch.empty_like(delta), packed=torch.empty((m.d_out, m.d_in // 2), dtype=torch.uint8, device=dev),
                scales=torch.empty(delta.shape, dtype=torch.float16, device=dev)))
        torch.cuda.synchronize(dev)
        self.gen_s = time.time() - t0
        self.searched = [e for e in self.mats if e["m"].name in wl.searched]
        self.weights = sum(e["W"].numel() for e in self.mats)
        self.hess_flop = sum(float(wl.n_calib) * d * (d + 1) for d in wl.calib.values())
        self.groups = sum(e["W"].numel() // 32 for e in self.searched)
        self.K = int(self.alpha.numel())
        self.lsq_bpe = LSQ_BYTES_PER_ELT if wl.g_dtype == "bf16" else LSQ_BYTES_PER_ELT_F32G
        # kernel launches of one step: a Hessian is one launch, plus the reduction of its
        # partials when its calibration rows are split
        self.launches = (sum(1 + (q4.hessian_workspace_bytes(wl.n_calib, d) > 0) for d in wl.calib.values())
                         + len(self.searched) + 2 * len(self.mats))

    def units(self):
        return {"hessian": self.hess_flop, "scale_search": float(self.groups),
                "lsq_fwd_bwd": self.lsq_bpe * self.weights, "pack_w4a16": PACK_BYTES_PER_ELT * self.weights}


STAGES = ("hessian", "scale_search", "lsq_fwd_bwd", "pack_w4a16")


def time_problem(p: DeviceProblem, q4, steps: int, warmup: int, flush: bool, world: int, rank: int,
                 local: int, clock_name: str | None):
    """Warm-up, then exactly `steps` steps bracketed by a barrier and a device synchronize on both
    sides.  A step runs the four stages over every matrix of the workload: each stage's launches
    (independent matrices) go round-robin to side streams (one launch goes on the launching
    stream itself), the stage ends when all are done, and CUDA events on the launching stream
    bracket it.  With `flush`, a 512 MB read sweep evicts L2 before every stage (inside the step
    time, outside the stage times)."""
    import torch
    import torch.distributed as dist
    dev = p.dev
    stream = torch.cuda.current_stream(dev)
    ns = len(p.ws)
    side = [torch.cuda.Stream(device=dev) for _ in range(ns)] if ns > 1 else []
    flush_buf = torch.ones(128 << 20, dtype=torch.float32, device=dev) if flush else None
    sink = torch.empty((), dtype=torch.float32, device=dev)

    def fan(launches):
        if not side:
            for launch in launches:
                launch(0)
            return
        go = torch.cuda.Event()
        go.record(stream)
        for s_ in side:
            s_.wait_event(go)
        for i, launch in enumerate(launches):
            with torch.cuda.stream(side[i % ns]):
                launch(i % ns)
        for s_ in side:
            done = torch.cuda.Event()
            done.record(s_)
            stream.wait_event(done)

    stage_fn = {
        "hessian": lambda: fan([lambda j, x=x: q4.hessian(p.X[x], p.H[x], p.ws[j]) for x in p.wl.calib]),
        "scale_search": lambda: fan([lambda j, e=e: q4.scale_search(e["W"], p.H[e["m"].x_name], p.alpha, e["delta"],
                                                                    e["idx"], e["err"]) for e in p.searched]),
        "lsq_fwd_bwd": lambda: fan([lambda j, e=e: q4.lsq_fwd_bwd(e["W"], e["delta"], e["G"], q4.GRAD_SCALE, e["Q"],
                                                                  e["gW"], e["gD"]) for e in p.mats]),
        "pack_w4a16": lambda: fan([lambda j, e=e: q4.pack_w4a16(e["W"], e["delta"], e["packed"], e["scales"])
                                   for e in p.mats]),
    }

    def step(ev=None):
        for i, name in enumerate(STAGES):
            if flush:
                torch.sum(flush_buf, dim=0, out=sink)
            if ev is not None:
                ev[i][0].record(stream)
            stage_fn[name]()
            if ev is not None:
                ev[i][1].record(stream)

    for _ in range(warmup):
        step()
    q4.sync_check()
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in STAGES] for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    path = os.path.join(OUT_DIR, f"{clock_name}_r{rank}.csv") if clock_name else None
    with ClockSampler(local, path) as clk:
        start.record(stream)
        for k in range(steps):
            step(evs[k])
        stop.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    q4.sync_check()
    mean = {s: sum(evs[k][i][0].elapsed_time(evs[k][i][1]) for k in range(steps)) / steps
            for i, s in enumerate(STAGES)}
    floor = copy_floor(p, stage_fn, stream, flush_buf, sink, steps) if flush else None
    alone = stages_alone(stage_fn, stream, flush_buf, sink, steps) if flush else None
    del flush_buf
    return {"total_ms": start.elapsed_time(stop), "stage_ms": mean, "clocks": clk.summary(), "copy_floor": floor,
            "alone_ms": alone}


def stages_alone(stage_fn, stream, flush_buf, sink, steps: int):
    """Each stage of a single-layer step on its own: after a 0.2 s pause (the GPU leaves the
    power state that the previous stage's work put it in), two untimed launches, then `steps`
    launches, each after the L2 flush and bracketed by CUDA events.  Lightest stage first.
    Returns {stage: mean ms}."""
    import torch
    out = {}
    for name in ("pack_w4a16", "lsq_fwd_bwd", "scale_search", "hessian"):
        torch.cuda.synchronize()
        time.sleep(0.2)
        for _ in range(2):
            stage_fn[name]()
        tot = 0.0
        for _ in range(steps):
            torch.sum(flush_buf, dim=0, out=sink)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            stage_fn[name]()
            b.record(stream)
            b.synchronize()
            tot += a.elapsed_time(b)
        out[name] = tot / steps
    return out


def copy_floor(p: DeviceProblem, stage_fn, stream, flush_buf, sink, steps: int):
    """Reference for the single-launch streaming stages of a single-layer step: the same steps
    again, with the LSQ and export launches replaced by a device copy (torch's copy kernel, src ->
    dst) that moves the stage's algorithmic bytes (half read, half written), after the same L2
    flush and after the same Hessian and search launches, so that it runs in the same power
    state.  Returns the mean CUDA-event time of each copy in ms."""
    import torch
    units = p.units()
    bufs = {}
    for s in ("lsq_fwd_bwd", "pack_w4a16"):
        half = int(units[s] // 2) // 16 * 16
        bufs[s] = (torch.ones(half, dtype=torch.uint8, device=p.dev), torch.empty(half, dtype=torch.uint8, device=p.dev))
    tot = {s: 0.0 for s in bufs}
    for k in range(steps + 1):                    # the first pass is a warm-up
        for name in ("hessian", "scale_search"):
            torch.sum(flush_buf, dim=0, out=sink)
            stage_fn[name]()
        for s, (src, dst) in bufs.items():
            torch.sum(flush_buf, dim=0, out=sink)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            dst.copy_(src)
            b.record(stream)
            b.synchronize()
            if k > 0:
                tot[s] += a.elapsed_time(b)
    return {s: tot[s] / steps for s in bufs}


def stage_lines(p: DeviceProblem, res, world: int, peaks, peak_kind: str, long_step: bool, traffic: dict):
    """Per-stage whole-job rate and roofline: units of all ranks / the slowest rank's time.
    Every rank makes the same collective calls in the same order."""
    units = p.units()
    job = {s: aggregate_over_ranks(units[s], res["stage_ms"][s]) for s in STAGES}
    hbm = float(peaks["hbm_gbs"])
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    sm_max = float(peaks.get("sm_max_mhz", 1965.0))
    alu_peak = 148 * 128 * sm_max * 1e6                                  # FP32 ops/s, one per lane per clock
    search_roof = alu_peak / (SEARCH_OPS_PER_CAND * p.K)                 # groups/s
    tc = sustained if long_step else burst
    out = {}
    u, ms = job["hessian"]
    v = u / ms / 1e9
    out["hessian"] = {"value": v, "unit": "TFLOP/s", "ms": ms, "launches": len(p.wl.calib),
                      "roofline": {"bound": "tensor", "achieved": v / world, "peak": tc, "unit": "TFLOP/s",
                                   "frac": v / world / tc, "frac_of_burst": v / world / burst,
                                   "frac_of_sustained": v / world / sustained,
                                   "algorithmic_per_step": units["hessian"],
                                   "peak_kind": f"{peak_kind} bf16 {'sustained' if long_step else 'burst'}"}}
    u, ms = job["scale_search"]
    v = u / ms * 1e3
    out["scale_search"] = {"value": v, "unit": "groups/s", "ms": ms, "launches": len(p.searched), "K": p.K,
                           "roofline": {"bound": "alu", "achieved": v / world * SEARCH_OPS_PER_CAND * p.K / 1e12,
                                        "peak": alu_peak / 1e12, "unit": "Top/s", "frac": v / world / search_roof,
                                        "ops_per_group": SEARCH_OPS_PER_CAND * p.K, "groups_per_step": units["scale_search"],
                                        "peak_kind": f"148 SM x 128 FP32 lanes x {sm_max:.0f} MHz"}}
    floor = res.get("copy_floor")
    for s in ("lsq_fwd_bwd", "pack_w4a16"):
        u, ms = job[s]
        v = u / ms / 1e6
        out[s] = {"value": v, "unit": "GB/s", "ms": ms, "launches": len(p.mats),
                  "roofline": {"bound": "hbm", "achieved": v / world, "peak": hbm, "unit": "GB/s",
                               "frac": v / world / hbm, "bytes_per_step": units[s], "peak_kind": f"{peak_kind} copy"}}
        if floor is not None:
            fu, fms = aggregate_over_ranks(units[s], floor[s])
            fv = fu / fms / 1e6
            out[s]["copy_floor"] = {
                "what": "device copy of the same bytes (half read, half written) at the same point of the "
                        "step (after the flush, the Hessian and the search), CUDA-event timed",
                "ms": fms, "gbs": fv / world, "frac_of_peak": fv / world / hbm, "stage_over_copy": v / fv}
    alone = res.get("alone_ms")
    if alone is not None:
        for s in STAGES:
            au, ams = aggregate_over_ranks(units[s], alone[s])
            frac = out[s]["roofline"]["frac"] * out[s]["ms"] / ams     # same work, same peak
            out[s]["alone"] = {"what": "the stage's launch on its own (after a 0.2 s pause, L2 flushed before "
                                       "each launch, no other stage in between), CUDA-event timed",
                               "ms": ams, "frac": frac}
    for s in STAGES:
        t = traffic.get(s)
        out[s]["roofline"]["traffic"] = t["bytes"] if t else None
        if t:
            out[s]["roofline"]["traffic_source"] = t["source"]
    return out


def e2e_lsq_stack(p: DeviceProblem, q4, steps: int):
    """The LSQ step of the stack end to end through the host-buffer call qat4_lsq_fwd_bwd_host:
    each call uploads W, G and the scales from page-locked host memory, runs the fused kernel on
    row chunks and downloads Q, grad_W and grad_delta (uploads on the caller's stream overlap the
    downloads on a copy stream).  Layer 0's seven matrices are held on the host (3 GB page-locked)
    and stand in for every layer of the stack, so one e2e step moves the whole stack's bytes
    through PCIe.  Returns (ms per step, h2d bytes, d2h bytes, algorithmic bytes)."""
    import torch
    dev = p.dev
    layer0 = [e for e in p.mats if e["m"].name.startswith("L0.")] if p.cfg in (3, 4) else p.mats
    reps = len(p.mats) // len(layer0)
    host = []
    for e in layer0:
        h = {k: e[k].cpu().pin_memory() for k in ("W", "G", "delta")}
        h.update(Q=torch.empty(e["W"].shape, dtype=torch.float32).pin_memory(),
                 gW=torch.empty(e["W"].shape, dtype=torch.float32).pin_memory(),
                 gD=torch.empty(e["delta"].shape, dtype=torch.float32).pin_memory())
        host.append(h)
    gd = q4.QAT4_BF16 if p.wl.g_dtype == "bf16" else q4.QAT4_F32
    ws = torch.empty(max(q4.lsq_fwd_bwd_host_workspace_bytes(*e["W"].shape, gd) for e in layer0),
                     dtype=torch.uint8, device=dev)
    cs = torch.cuda.Stream(device=dev)
    stream = torch.cuda.current_stream(dev)

    def one():
        for _ in range(reps):
            for h in host:
                q4.lsq_fwd_bwd_host(h["W"], h["delta"], h["G"], q4.GRAD_SCALE, h["Q"], h["gW"], h["gD"],
                                    workspace=ws, copy_stream=cs)

    one()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        one()
    b.record(stream)
    torch.cuda.synchronize(dev)
    q4.sync_check()
    ms = a.elapsed_time(b) / steps
    gbytes = 2 if gd == q4.QAT4_BF16 else 4
    h2d = reps * sum(h["W"].numel() * (4 + gbytes) + h["delta"].numel() * 4 for h in host)
    d2h = reps * sum(h["W"].numel() * 8 + h["delta"].numel() * 4 for h in host)
    return ms, h2d, d2h, p.lsq_bpe * p.weights


def cpu_model() -> str:
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for ln in out.splitlines():
            if ln.lower().startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except (OSError, subprocess.SubprocessError):
        pass
    return "unknown"


# ------------------------------------------------------------------------ our arm
PATH_CONFIGS = (4, 1, 2)        # the headline step first, then the single-layer configurations


def run_ours(args):
    import torch
    import torch.distributed as dist

    import int4_group_wise_b200 as q4

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    peaks, peak_kind = load_peaks()
    os.makedirs(OUT_DIR, exist_ok=True)
    configs = PATH_CONFIGS if args.config is None else (args.config,)
    seed = layer_seed(rank)
    results = {}
    for i, cfg in enumerate(configs):
        stack = cfg in (3, 4)
        p = DeviceProblem(cfg, dev, seed, q4, streams=4 if stack else 1)
        res = time_problem(p, q4, args.steps, args.warmup, flush=not stack, world=world, rank=rank, local=local,
                           clock_name=f"bench_clocks_c{cfg}")
        job_steps, job_total = aggregate_over_ranks(1.0, res["total_ms"])
        traffic = load_traffic(cfg, p)
        lines = stage_lines(p, res, world, peaks, peak_kind, long_step=stack, traffic=traffic)
        entry = {"workload": p.wl.title, "config_index": cfg, "ms_per_step": job_total / args.steps,
                 "matrices": len(p.mats), "weights": p.weights, "hessians": len(p.wl.calib),
                 "n_calib": p.wl.n_calib, "searched_matrices": len(p.searched), "K": p.K,
                 "streams": len(p.ws), "stages": lines, "clocks": res["clocks"],
                 "gpu_launches": p.launches * args.steps, "input_gen_s": round(p.gen_s, 1),
                 "l2": ("every stage's inputs are larger than L2 (126 MB); no flush" if stack else
                        "flushed (512 MB read sweep) before every stage; flush time in ms_per_step only")}
        if i == 0 and not args.no_e2e:
            ms, h2d, d2h, alg = e2e_lsq_stack(p, q4, steps=2 if stack else max(3, min(args.steps, 10)))
            job_alg, job_ms = aggregate_over_ranks(alg, ms)
            entry["e2e"] = {"value": job_alg / job_ms / 1e6, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                            "d2h_bytes_per_step": d2h, "ms_per_step": job_ms,
                            "what": "the LSQ fwd+bwd step of the whole workload through the C ABI host-buffer "
                                    "call qat4_lsq_fwd_bwd_host (page-locked host W, G, delta in; Q, grad_W, "
                                    "grad_delta out; uploads overlap downloads)" +
                                    ("; layer 0's seven host matrices stand in for every layer" if stack else "")}
        if i == 0 and rank == 0 and world == 1 and not args.no_cpu_baseline:
            entry["cpu_baseline"] = cpu_baseline(p)
        results[cfg] = entry
        del p
        torch.cuda.empty_cache()

    head = results[configs[0]]
    if rank == 0:
        st = head["stages"]
        dominant = max(STAGES, key=lambda s: st[s]["ms"])
        dom = st[dominant]["roofline"]
        line = {
            "metric": METRIC, "value": st["lsq_fwd_bwd"]["value"], "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (drawn on the GPU with the workloads' distributions)",
            "config": {"workload": head["workload"], "config_index": head["config_index"],
                       "matrices": head["matrices"], "weights": head["weights"], "hessians": head["hessians"],
                       "n_calib": head["n_calib"], "searched_matrices": head["searched_matrices"], "K": head["K"],
                       "parallelism": f"replicas x{world} (every GPU its own seeded copy of the workload)",
                       "l2": head["l2"]},
            "roofline": {"kernel": dominant, **{k: dom[k] for k in ("bound", "achieved", "peak", "unit", "frac")},
                         "traffic": dom.get("traffic"), "traffic_source": dom.get("traffic_source"),
                         "traffic_unit": "bytes per step of the stage (ncu DRAM read + write)",
                         "peak_kind": dom["peak_kind"],
                         "note": "achieved = the stage's algorithmic work per step / its CUDA-event time "
                                 "(launches fanned out over side streams, joined on the launching stream)"},
            "stages": {**st, **{f"config{c}": {k: results[c][k] for k in
                                               ("workload", "ms_per_step", "stages", "clocks", "gpu_launches", "l2")}
                                for c in configs[1:]}},
            "e2e": head.get("e2e"),
            "gpu_launches": sum(results[c]["gpu_launches"] for c in configs),
            "clocks": head["clocks"],
            "input_gen_s": round(sum(results[c]["input_gen_s"] for c in configs), 1),
        }
        if "cpu_baseline" in head:
            line["cpu_baseline"] = head["cpu_baseline"]
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------ CPU oracle legs
def _oracle_step(W, G, X, alpha, hblocks: int, search_rows: int):
    """One pass of the oracle over host samples: LSQ fwd+bwd and pack over every matrix in W/G,
    the diagonal 32x32 Hessian blocks 0..hblocks-1 of X over all its rows, and the scale search of
    those groups on the first `search_rows` rows of the first matrix.  Returns per-stage
    (units, seconds) in the GPU's units (flop, groups, bytes)."""
    import oracle
    res = {}
    n = X.shape[0]
    t = time.perf_counter()
    starts = [32 * g for g in range(hblocks)]
    blocks = oracle.hessian_blocks(X, starts, starts, 32)
    res["hessian"] = (float(n) * 32 * 33 * hblocks, time.perf_counter() - t)
    Hd = np.zeros((32 * hblocks, 32 * hblocks), np.float32)
    for g in range(hblocks):
        Hd[32 * g:32 * g + 32, 32 * g:32 * g + 32] = blocks[g]
    Ws = np.ascontiguousarray(W[0][:search_rows, :32 * hblocks])
    t = time.perf_counter()
    oracle.scale_search(Ws, Hd, alpha)
    res["scale_search"] = (float(Ws.size // 32), time.perf_counter() - t)
    lsq_u = pack_u = lsq_s = pack_s = 0.0
    s_ = float(np.float32(1 / np.sqrt(224)))
    for w, g in zip(W, G):
        delta = (np.abs(w).reshape(w.shape[0], -1, 32).max(axis=2) / np.float32(7)).astype(np.float32)
        bpe = LSQ_BYTES_PER_ELT if g.dtype == np.uint16 else LSQ_BYTES_PER_ELT_F32G
        t = time.perf_counter()
        oracle.lsq_fwd(w, delta)
        oracle.lsq_bwd(w, delta, g, s_)
        lsq_s += time.perf_counter() - t
        lsq_u += bpe * w.size
        t = time.perf_counter()
        oracle.pack_w4a16(w, delta)
        pack_s += time.perf_counter() - t
        pack_u += PACK_BYTES_PER_ELT * w.size
    res["lsq_fwd_bwd"] = (lsq_u, lsq_s)
    res["pack_w4a16"] = (pack_u, pack_s)
    return res


def _rates(res):
    return {"hessian_gflops": res["hessian"][0] / res["hessian"][1] * 1e-9,
            "scale_search_groups_per_s": res["scale_search"][0] / res["scale_search"][1],
            "lsq_fwd_bwd_gbs": res["lsq_fwd_bwd"][0] / res["lsq_fwd_bwd"][1] * 1e-9,
            "pack_w4a16_gbs": res["pack_w4a16"][0] / res["pack_w4a16"][1] * 1e-9}


def _host_bits(t):
    """A device tensor as host NumPy data; bf16 as its uint16 bit patterns."""
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def cpu_baseline(p: DeviceProblem, hblocks: int = 128):
    """The oracle as it stands on the host cores, on a bounded sample of the workload the GPU
    just ran (its own tensors, copied to the host): LSQ and pack over every matrix of layer 0 (for
    the stacks; the whole layer otherwise), the first `hblocks` diagonal Hessian blocks over all
    calibration rows of the first searched matrix's input, and the search of those groups over
    all rows of that matrix."""
    import oracle
    cores = oracle.set_threads(0)
    layer0 = [e for e in p.mats if e["m"].name.startswith("L0.")] if p.cfg in (3, 4) else p.mats
    first = p.searched[0]
    order = [first] + [e for e in layer0 if e is not first]
    W = [_host_bits(e["W"]) for e in order]
    G = [_host_bits(e["G"]) for e in order]
    X = _host_bits(p.X[first["m"].x_name])
    alpha = p.alpha.cpu().numpy()
    hb = min(hblocks, X.shape[1] // 32)
    rows = W[0].shape[0]
    res = _oracle_step(W, G, X, alpha, hb, rows)
    r = _rates(res)
    return {"value": r["lsq_fwd_bwd_gbs"], "unit": "GB/s", "cores": cores, "cpu_model": cpu_model(),
            "kind": "oracle",
            "sample": (f"LSQ fwd+bwd and W4A16 pack over {'all 7 matrices of layer 0' if p.cfg in (3, 4) else 'the whole layer'} "
                       f"({sum(w.size for w in W)} weights, in full); Hessian: {hb} diagonal 32x32 blocks of "
                       f"{first['m'].x_name} over all {X.shape[0]} calibration rows (sampled); scale search: "
                       f"those {hb} groups x {rows} rows of {first['m'].name} (sampled)"),
            "seconds": round(sum(v[1] for v in res.values()), 2), "stages": r}


def run_reference(args):
    """The oracle as it stands on the host cores, on bounded samples of the headline workload:
    each step runs every stage once on a fixed sample (the first rows of every layer-0 matrix for
    LSQ and pack, diagonal Hessian blocks over a row sample of the calibration set, the search of
    those groups on a row sample).  Under several ranks, rank 0 alone runs and prints; the others
    exit without work."""
    rank, world, _ = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("gloo", timeout=timedelta(seconds=300))
        try:
            if rank == 0:
                _reference_line(args, world)
            dist.barrier()
        finally:
            dist.destroy_process_group()
        return
    _reference_line(args, world)


def _reference_line(args, world):
    import oracle
    from int4_group_wise_b200 import inputs
    cfg = 4 if args.config is None else args.config
    wl = inputs.workload(cfg)
    mats = [m for m in wl.matrices if m.name.startswith("L0.")] if cfg in (3, 4) else wl.matrices
    rows = 256 if cfg in (3, 4) else 1024
    searched = next(m for m in mats if m.name in wl.searched)
    order = [searched] + [m for m in mats if m is not searched]
    W = [wl.weight(m, rows=rows) for m in order]
    G = [wl.grad(m, rows=rows) for m in order]
    n = min(wl.n_calib, 16384)
    X = wl.activations(searched.x_name, n=n)
    alpha = wl.alpha()
    hb = 4
    cores = oracle.set_threads(0)
    for _ in range(args.warmup):
        _oracle_step(W, G, X, alpha, hb, rows)
    tot = {s: [0.0, 0.0] for s in STAGES}
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r = _oracle_step(W, G, X, alpha, hb, rows)
        for s in STAGES:
            tot[s][0] += r[s][0]
            tot[s][1] += r[s][1]
    wall = time.perf_counter() - t0
    rates = _rates({s: tuple(v) for s, v in tot.items()})
    v = rates["lsq_fwd_bwd_gbs"]
    sample = (f"per step: the first {rows} rows of every {'layer-0 ' if cfg in (3, 4) else ''}matrix "
              f"({sum(w.size for w in W)} weights) for LSQ fwd+bwd and pack; {hb} diagonal 32x32 Hessian blocks "
              f"of {searched.x_name} over its first {n} calibration rows; the scale search of those {hb} groups "
              f"x {rows} rows of {searched.name}")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"{wl.title} (CPU oracle, bounded row sample)", "config_index": cfg},
        "stages": rates,
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_per_channel(args):
    """The per-channel variant (one scale per row) on the same layer shape: fused LSQ step and
    W4A16 export, each launch timed with CUDA events after an L2 flush; one JSON line."""
    import torch

    import int4_group_wise_b200 as q4
    from int4_group_wise_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    wl = inputs.workload(1 if args.config is None else args.config)
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
    """Decode on the W4A16 export of the 8B-class stack (32 layers x {q, k, v, o, gate, up, down}):
    one step = the GEMVs of one token batch (M = 1 and M = 4) over every layer, replayed from a
    CUDA graph.  The export is laid out the way a decode engine stores it: the rows of q, k and v
    (which read the same input) stacked into one matrix, likewise gate and up, so a layer is four
    GEMVs (qkv 6144x4096, o 4096x4096, gate_up 28672x4096, down 4096x14336).  Stacking rows changes
    no value: every output row is the same dot product.  The seeded layer-0 weights, packed once,
    are copied into 32 distinct layer buffers (3.9 GB of codes and scales, 31x L2), so every step
    streams its bytes from HBM."""
    import torch

    import int4_group_wise_b200 as q4
    from int4_group_wise_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    wl = inputs.workload(4)
    layer0 = {m.name.split(".")[1]: m for m in wl.matrices if m.name.startswith("L0.")}
    n_layers = len(wl.matrices) // len(layer0) if args.layers is None else args.layers
    fused = [("qkv", ["q", "k", "v"]), ("o", ["o"]), ("gate_up", ["gate", "up"]), ("down", ["down"])]
    base = []
    for name, parts in fused:
        ps, ss = [], []
        for part in parts:
            m = layer0[part]
            W = torch.from_numpy(wl.weight(m)).to(dev)
            R, C = W.shape
            delta = (W.abs().reshape(R, C // 32, 32).amax(dim=2) / 7).contiguous()
            p_, s_ = q4.pack_w4a16(W, delta)
            ps.append(p_)
            ss.append(s_)
            del W, delta
        base.append((torch.cat(ps, 0).contiguous(), torch.cat(ss, 0).contiguous()))
    q4.sync_check()
    layers = [[(p.clone(), sc.clone()) for p, sc in base] for _ in range(n_layers)]
    del base
    torch.cuda.synchronize()
    shapes = [(lay[0].shape[0], lay[0].shape[1] * 2) for lay in layers[0]]
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
        for (name, _), (R, C), (p, sc), y in zip(fused, shapes, layers[0], ys):
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
            per_shape[name] = {"shape": [R, C], "us": us, "gbs": nbytes / us / 1e3, "frac": nbytes / us / 1e3 / hbm}
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
        "config": {"workload": f"8B-class stack, {n_layers} layers x (qkv, o, gate_up, down), {weights} weights, "
                               "group-32 export, decode batch M = 1 and 4",
                   "l2": "inputs 31x L2 (distinct layer buffers); per-shape times flush L2 before every launch"},
        "roofline": {"bound": "hbm", "achieved": r1["gbs"], "peak": hbm, "unit": "GB/s", "frac": r1["frac"],
                     "peak_kind": f"{peak_kind} copy"},
        "gpu_launches": r1["launches_per_step"] * args.steps,
        "stages": {f"M={M}": v for M, v in results.items()}}), flush=True)


def run_fq_gemm(args):
    """The fake-quant forward GEMM of a QAT step on the 1B-class up-projection (W fp32 8192x2048,
    searched-range scales) for a micro-batch of --tokens tokens: TFLOP/s of the staged call
    (quantizer into a bf16 workspace, then the persistent tcgen05 GEMM) against the bf16 tensor
    peak, each launch timed with CUDA events after an L2 flush.  Timed beside it, interleaved:
    the single fused kernel, and the same product unfused through libraries (the LSQ forward, a
    cast to bf16 and a cuBLAS bf16 GEMM)."""
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

    ws = torch.empty(q4.lib().qat4_fq_gemm_staged_workspace_bytes(R, C), dtype=torch.uint8, device=dev)
    staged = lambda: q4.fq_gemm(X, W, D, Y, workspace=ws)
    fused = lambda: q4.fq_gemm(X, W, D, Y, fused=True)

    def unfused():
        q4.lsq_fwd(W, D, Q)
        torch.matmul(X, Q.to(torch.bfloat16).t())

    for _ in range(args.warmup):
        staged()
        fused()
        unfused()
    q4.sync_check()
    # interleaved rounds so that the three paths see the same power state
    t_f, t_1, t_u = [], [], []
    with ClockSampler(0) as clk:
        for _ in range(3):
            t_f += timed(staged, max(1, args.steps // 3))
            t_1 += timed(fused, max(1, args.steps // 3))
            t_u += timed(unfused, max(1, args.steps // 3))
    t_f.sort()
    q4.sync_check()
    flop = 2.0 * T * R * C
    ms = statistics.median(t_f)
    tf = flop / ms / 1e9
    peak = float(peaks["bf16_tflops"])
    print(json.dumps({
        "metric": "fake-quant GEMM TFLOP/s (Y = X bf16(Q_Delta(W))^T)", "value": tf, "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "variant": "fq-gemm", "data": "synthetic", "dtype": "bf16 x bf16 -> f32 (quantizer f32)",
        "config": {"workload": f"1B-class up-projection W fp32 {R}x{C}, X bf16 {T}x{C} (micro-batch of {T} tokens)",
                   "l2": "flushed (512 MB read sweep) before every launch"},
        "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                     "flop_per_launch": flop, "peak_kind": f"{peak_kind} bf16 burst"},
        "ms_min_median_max": [t_f[0], ms, t_f[-1]],
        "what": "qat4_fq_gemm_staged: quantizer into a bf16 workspace, then a persistent tcgen05 GEMM",
        "fused_single_kernel_ms": statistics.median(t_1),
        "unfused_library_ms": statistics.median(t_u),
        "unfused_library": "qat4_lsq_fwd + cast to bf16 + torch.matmul (cuBLAS bf16), same product",
        "gpu_launches": 2 * len(t_f), "clocks": clk.summary()}), flush=True)


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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=None, choices=[0, 1, 2, 3, 4],
                    help="time only this workload as the headline (default: the 8B-class stack, then "
                         "configs 1 and 2 under stages)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--variant", choices=["path", "per-channel", "w4a16-decode", "fq-gemm", "hessian-split",
                                          "refine"],
                    default="path",
                    help="per-channel: time the one-scale-per-row LSQ step and export instead; "
                         "w4a16-decode: time the inference GEMV on the packed 8B-class stack; "
                         "fq-gemm: time the fake-quant forward GEMM (staged, fused and unfused); "
                         "hessian-split: the calibration Hessian with its rows split over the ranks; "
                         "refine: one sweep of the full-objective refinement")
    ap.add_argument("--tokens", type=int, default=8192, help="fq-gemm: tokens of the micro-batch")
    ap.add_argument("--layers", type=int, default=None,
                    help="w4a16-decode: number of layers of the 8B-class stack (default: all 32)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ:
        if args.gpus > 1:          # one process per GPU: start the ranks, then report their status
            sys.exit(relaunch_ranks(args.gpus, sys.argv[1:]))
    elif int(os.environ["WORLD_SIZE"]) != args.gpus:
        ap.error(f"--gpus {args.gpus} but the launcher started WORLD_SIZE={os.environ['WORLD_SIZE']} ranks")
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
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
