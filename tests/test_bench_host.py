"""Host arithmetic of bench.py, on CPU: the roofline numerators (algorithmic
FLOPs and bytes per launch) and the summary of the SM-clock samples that
decides whether a timed run was throttled (fed with nvidia-smi CSV lines)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from mixture_experts_projections_b200.inputs import WORKLOADS  # noqa: E402


def test_block_flops_of_the_workloads():
    f = bench.block_flops(WORKLOADS["prefill_16k"])
    assert f["conv_gate"] == pytest.approx(549.76e9, rel=1e-4)  # 4 * 16384 * 2048 * 4096
    assert f["out"] == pytest.approx(274.88e9, rel=1e-4)
    assert "backward" not in f
    t2 = bench.block_flops(WORKLOADS["top2_fwd_bwd"])
    # R = 65536 routed rows: 5.154 TFLOP forward, twice that backward
    assert t2["conv_gate"] + t2["out"] == pytest.approx(5.154e12, rel=1e-3)
    assert t2["backward"] == pytest.approx(2 * 5.154e12, rel=1e-3)
    assert bench.block_flops(WORKLOADS["decode_swimba_inproj"]) == {
        "inproj": 2.0 * 64 * 4096 * 10240}


def test_inproj_bytes_of_the_decode_workload():
    wl = WORKLOADS["decode_swimba_inproj"]
    # 335.5 MB of weights (4 experts hit) + 0.5 MB x + 1.3 MB out
    assert bench.inproj_bytes(wl, 4) == 4 * 4096 * 10240 * 2 + 64 * 4096 * 2 + 64 * 10240 * 2
    assert bench.inproj_bytes(wl, 4) == pytest.approx(337.4e6, rel=1e-3)
    # only the experts that received tokens stream their weights
    assert bench.inproj_bytes(wl, 3) == bench.inproj_bytes(wl, 4) - 4096 * 10240 * 2


def _line(sm, smax, hw="Not Active", hwt="Not Active", swt="Not Active", cap="Not Active"):
    return f"0, {sm}, {smax}, 812.50, 0x0000000000000000, {hw}, {hwt}, {swt}, {cap}"


def test_clock_summary_unthrottled():
    s = bench.summarize_clocks([_line(1965, 1965), _line(1950, 1965), _line(1965, 1965)])
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3}


def test_clock_summary_reports_every_active_reason():
    s = bench.summarize_clocks([_line(1830, 1965, cap="Active"), _line(1700, 1965, cap="Active"),
                                _line(1500, 1965, hwt="Active"), _line(1965, 1965)])
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert s["sm_mhz"] == pytest.approx(1765.0)
    assert s["samples"] == 4


def test_clock_summary_skips_lines_that_do_not_parse():
    s = bench.summarize_clocks(["", "garbage", _line("[N/A]", 1965), _line(1965, 1965),
                                "0, 1965, 1965"])
    assert s["samples"] == 1 and s["sm_mhz"] == 1965.0
    empty = bench.summarize_clocks([])
    assert empty["sm_mhz"] is None and empty["sm_max_mhz"] is None and empty["samples"] == 0


def test_nvml_clock_summary_and_merge():
    """The NVML samples of the timed steps: median and lowest clock and the
    throttle reasons among their bits; with at least 3 of them their median
    and reasons replace nvidia-smi's, which may have seen only idle moments."""
    fast = bench.summarize_nvml([(1965, 0), (1800, 0x4), (1700, 0x4 | 0x1), (1965, 0)], 0.002)
    assert fast["samples"] == 4 and fast["sm_mhz"] == 1882.5 and fast["sm_mhz_min"] == 1700
    assert fast["reasons"] == ["sw_power_cap"]  # the idle bit (0x1) is not a throttle reason
    assert bench.summarize_nvml([(1965, 0x8 | 0x40)], 0.002)["reasons"] == [
        "hw_slowdown", "hw_thermal_slowdown"]
    assert bench.summarize_nvml([], 0.002) == {"samples": 0}
    smi = bench.summarize_clocks([_line(1965, 1965), _line(1965, 1965)])
    m = bench.merge_clocks(smi, fast)
    assert m["sm_mhz"] == 1882.5 and m["sm_max_mhz"] == 1965.0
    assert m["reasons"] == ["sw_power_cap"] and m["nvml"] is fast and m["samples"] == 2
    few = bench.summarize_nvml([(1500, 0), (1500, 0)], 0.002)
    assert bench.merge_clocks(smi, few) == smi
    assert bench.merge_clocks(smi, None) == smi


def test_core_roofline_counts_one_exp_per_state_update():
    wl = WORKLOADS["prefill_16k_core"]
    res = {"part_ms": {"core": 1.0}, "clocks": {"sm_max_mhz": 1965.0}}
    r = bench.core_roofline(res, wl)
    # 16384 tokens x 4096 channels x 16 states in 1 ms
    assert r["achieved"] == pytest.approx(16384 * 4096 * 16 / 1e-3 / 1e9)
    assert r["peak"] == pytest.approx(148 * 16 * 1965e6 / 1e9)
    assert r["bound"] == "alu" and 0 < r["frac"] < 1


def test_workload_config_of_every_workload():
    """The config dict each JSON line carries: the workload's name and sizes;
    the decode-sized in-projection says its weights are tile-major."""
    for name, wl in WORKLOADS.items():
        cfg = bench.workload_config(wl, 1)
        assert cfg["workload"] == name and cfg["tokens"] == wl.T and cfg["experts"] == wl.E
        assert cfg["parallelism"] == "replicas x1"
        tiled = wl.kind == "inproj" and wl.dtype == "bf16" and wl.T <= 64
        assert ("weights" in cfg) == tiled, name


def test_phase_figures():
    """The route + dispatch phase's algorithmic bytes (X read by the router,
    the T*k routed rows read and written by the dispatch) over its time, and
    a training step's forward token rate."""
    wl = WORKLOADS["prefill_16k"]
    f = bench.phase_figures(wl, {"route_dispatch": 0.05, "proj0": 0.3, "proj1": 0.2}, 6500.0, 1)
    nbytes = 16384 * 2048 * 2 * 3
    assert f["route_dispatch_hbm"]["bytes"] == nbytes
    assert abs(f["route_dispatch_hbm"]["achieved_gbs"] - nbytes / 5e-5 / 1e9) < 1e-6
    assert "forward_tokens_per_s" not in f
    wl = WORKLOADS["top2_fwd_bwd"]
    f = bench.phase_figures(wl, {"route_dispatch": 0.3, "proj0": 2.5, "proj1": 2.2,
                                 "backward": 11.0}, 6500.0, 1)
    assert f["route_dispatch_hbm"]["bytes"] == 32768 * 2560 * 2 * (1 + 2 * 2)
    assert abs(f["forward_tokens_per_s"] - 32768 / 5.0e-3) < 1e-3
    assert bench.phase_figures(WORKLOADS["decode_swimba_inproj"], {"route": 0.01}, 6500.0, 1) == {}


def test_tensor_roofline_gives_the_sustained_peak_only_under_the_power_cap():
    """The dominant GEMM's fraction is of the burst peak; when the clocks of
    its run show sw_power_cap, the fraction of the sustained peak is added."""
    wl = WORKLOADS["top2_fwd_bwd"]
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    res = {"wl": wl, "dominant_ms": 2.0, "dominant_kind": "flop", "dominant_work": 2.8e12,
           "clocks": {"reasons": ["sw_power_cap"]}}
    r = bench.roofline(res, peaks, "measured")
    assert abs(r["achieved"] - 1400.0) < 1e-9 and abs(r["frac"] - 0.875) < 1e-12
    assert abs(r["sustained"]["frac"] - 1.0) < 1e-12 and r["sustained"]["peak"] == 1400.0
    res["clocks"] = {"reasons": []}
    assert "sustained" not in bench.roofline(res, peaks, "measured")
