"""Host logic of bench.py's JSON line (CPU): the per-stage roofline arithmetic, the single-layer
references (`copy_floor`, `alone`) and the stored DRAM-traffic table's hash gate."""
import os
import types

import pytest

import bench


def _problem(K=101):
    wl = types.SimpleNamespace(calib={"x": 2048})
    return types.SimpleNamespace(
        wl=wl, K=K, searched=[object()], mats=[object()],
        units=lambda: {"hessian": 1.1e12, "scale_search": 524288.0, "lsq_fwd_bwd": 2.39e8, "pack_w4a16": 7.86e7})


PEAKS = {"hbm_gbs": 6400.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 2000.0}


def _res(with_refs: bool):
    res = {"stage_ms": {"hessian": 0.8, "scale_search": 1.3, "lsq_fwd_bwd": 0.04, "pack_w4a16": 0.016}}
    if with_refs:
        res["copy_floor"] = {"lsq_fwd_bwd": 0.038, "pack_w4a16": 0.014}
        res["alone_ms"] = {"hessian": 0.79, "scale_search": 1.25, "lsq_fwd_bwd": 0.039, "pack_w4a16": 0.0155}
    return res


def test_stage_rooflines_follow_the_work_and_the_peaks():
    p = _problem()
    out = bench.stage_lines(p, _res(False), 1, PEAKS, "measured", long_step=False, traffic={})
    h = out["hessian"]
    assert h["value"] == pytest.approx(1.1e12 / 0.8e-3 / 1e12)                    # TFLOP/s
    assert h["roofline"]["frac"] == pytest.approx(h["value"] / 1600.0)            # single layer: burst peak
    s = out["scale_search"]
    roof = 148 * 128 * 2000e6 / (bench.SEARCH_OPS_PER_CAND * 101)                  # groups/s
    assert s["roofline"]["frac"] == pytest.approx(524288.0 / 1.3e-3 / roof)
    for st, ms in (("lsq_fwd_bwd", 0.04), ("pack_w4a16", 0.016)):
        gbs = p.units()[st] / (ms * 1e-3) / 1e9
        assert out[st]["value"] == pytest.approx(gbs)
        assert out[st]["roofline"]["frac"] == pytest.approx(gbs / 6400.0)
        assert "copy_floor" not in out[st] and "alone" not in out[st]
    assert all(out[st]["roofline"]["traffic"] is None for st in bench.STAGES)


def test_long_step_compares_the_tensor_stage_with_the_sustained_peak():
    out = bench.stage_lines(_problem(), _res(False), 1, PEAKS, "measured", long_step=True, traffic={})
    h = out["hessian"]["roofline"]
    assert h["peak"] == 1400.0 and h["frac"] == pytest.approx(h["achieved"] / 1400.0)
    assert h["frac_of_burst"] == pytest.approx(h["achieved"] / 1600.0)


def test_single_layer_references():
    out = bench.stage_lines(_problem(), _res(True), 1, PEAKS, "measured", long_step=False, traffic={})
    for st in ("lsq_fwd_bwd", "pack_w4a16"):
        cf = out[st]["copy_floor"]
        ms = _res(True)["copy_floor"][st]
        assert cf["ms"] == ms
        assert cf["gbs"] == pytest.approx(_problem().units()[st] / (ms * 1e-3) / 1e9)
        assert cf["stage_over_copy"] == pytest.approx(out[st]["value"] / cf["gbs"])
    for st in bench.STAGES:
        a = out[st]["alone"]
        ms = _res(True)["alone_ms"][st]
        # the same work against the same peak: the fraction scales with the inverse time
        assert a["frac"] == pytest.approx(out[st]["roofline"]["frac"] * out[st]["ms"] / ms)


def test_stored_traffic_is_used_only_while_the_sources_match(tmp_path, monkeypatch):
    table = ("source_hash: {h}\n\n| config | kernel | bytes |\n|---|---|---|\n"
             "| 1 | hessian_pair_kernel | 1000 |\n| 1 | hessian_reduce_kernel | 24 |\n"
             "| 1 | scale_search_kernel | 7 |\n| 1 | lsq_blocks_kernel | 5 |\n| 1 | pack_w4a16_blocks_kernel | 3 |\n"
             "| 2 | lsq_blocks_kernel | 9 |\n")
    f = tmp_path / "traffic.md"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    f.write_text(table.format(h="0000000000000000"))
    assert bench.load_traffic(1) == {}                                # stale capture: nothing reported
    f.write_text(table.format(h=bench.source_hash()))
    t = bench.load_traffic(1)
    assert t["hessian"]["bytes"] == 1024                              # pair kernel + its reduction
    assert (t["scale_search"]["bytes"], t["lsq_fwd_bwd"]["bytes"], t["pack_w4a16"]["bytes"]) == (7, 5, 3)
    assert set(bench.load_traffic(2)) == {"lsq_fwd_bwd"}              # only what was captured


def test_committed_traffic_table_matches_the_current_sources():
    """The committed capture must be of the kernels as they are: its hash is the sources' hash."""
    with open(os.path.join(bench.ROOT, "profiles", "dram_traffic_path.md")) as fh:
        line = next(ln for ln in fh if ln.startswith("source_hash:"))
    assert line.split(":", 1)[1].strip() == bench.source_hash()
