"""bench.py's algorithmic work counts (host logic, no GPU), against hand-worked values."""
import numpy as np
import pytest

import bench
from gen import LayerConfig


def test_backward_units_hand_worked():
    """Three chunks, two experts: counts [[1, 0], [2, 3], [0, 4]].  The weight gradients run
    per pair of chunks, (0, 1) then (2): the first pair stores dW of both experts, the
    second reads and writes expert 1's."""
    cfg = LayerConfig("u", T=3, H=64, E=2, k=2, I=32, routing="normal")
    u = bench.backward_units(cfg, np.array([[1, 0], [2, 3], [0, 4]], np.int32))
    H, I = 64, 32
    rows = 10
    assert u["flops"]["bwd_wgrad"] == 6 * rows * H * I
    # recomputed gate/up 4, SwiGLU backward 2, dX 4, weight gradients 6 (no down GEMM: d_w
    # comes from the SwiGLU-backward epilogue)
    assert sum(u["flops"].values()) == 16 * rows * H * I
    operands = rows * (2 * H + 3 * I) * 2
    dw = 12 * H * I * (3 + 1)  # 3 (pair, expert) stores or adds written, 1 of them also read
    assert u["wgrad_bytes"] == pytest.approx(operands + dw)


def test_forward_units_hand_worked():
    cfg = LayerConfig("u", T=3, H=64, E=2, k=2, I=32, routing="normal")
    u = bench.algorithmic_units(cfg, np.array([[1, 0], [2, 3]], np.int32), 2)
    assert u["gateup_flops"] == 4 * 6 * 64 * 32
    assert u["gateup_weight_bytes"] == 3 * 2 * 32 * 64 * 2
    assert u["permute_bytes"] == (3 + 6) * 64 * 2 + 6 * 4


def test_traffic_reported_only_for_the_captured_launch(monkeypatch):
    """The committed ncu traffic figure belongs to one launch: the gate/up GEMM source it
    was taken on, the Qwen3-shaped layer, num_chunks=4, fused dispatch with pair sweeps.
    Any other case, or a changed kernel source, reports no traffic."""
    import json
    with open(bench.TRAFFIC_FILE) as f:
        rec = json.load(f)
    got = bench.traffic_per_launch("qwen3", 4, "fused", True)
    if rec["gemm_src_sha256_16"] == bench.gemm_src_hash():
        assert got == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    else:  # the kernel changed after the capture: the bench reports null until retaken
        assert got is None
    monkeypatch.setattr(bench, "gemm_src_hash", lambda: rec["gemm_src_sha256_16"])
    assert bench.traffic_per_launch("qwen3", 2, "fused", True) is None
    assert bench.traffic_per_launch("qwen3", 4, "separate", True) is None
    assert bench.traffic_per_launch("qwen3", 4, "fused", False) is None
    assert bench.traffic_per_launch("mixtral", 4, "fused", True) is None
    monkeypatch.setattr(bench, "gemm_src_hash", lambda: "0" * 16)
    assert bench.traffic_per_launch("qwen3", 4, "fused", True) is None


def test_clock_summary_keeps_only_the_timed_window():
    """Samples (host time, SM MHz, max SM MHz, reasons): only those inside the timed region
    (plus one sampling period) count; the median SM clock and every reason among them are
    reported; with too few samples inside, the window widens back to the untimed steps
    just before the region, and says so."""
    s = bench.ClockSampler(0, period_s=0.05)
    s.source = "test"
    s.samples = [(0.5, 700.0, 1965.0, set()),                 # before the region
                 (1.0, 1400.0, 1965.0, {"sw_power_cap"}),
                 (1.2, 1500.0, 1965.0, set()),
                 (1.4, 1450.0, 1965.0, {"sw_power_cap"}),
                 (1.54, 1300.0, 1965.0, set()),               # within one period after it
                 (3.0, 600.0, 1965.0, {"hw_slowdown"})]
    out = s.summary(1.0, 1.5)
    assert out["sm_mhz"] == 1425.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 4
    assert out["sm_mhz_min"] == 1300.0 and out["window"] == "timed region"
    narrow = s.summary(1.19, 1.21, min_samples=3, widen_to=0.4)
    assert narrow["samples"] == 3 and narrow["window"].startswith("timed region and")
    assert s.summary(1.19, 1.21, min_samples=1)["samples"] == 1
    every = s.summary()
    assert every["samples"] == 6 and "hw_slowdown" in every["reasons"]
    assert s.summary(5.0, 6.0) is None


def test_tensor_peak_follows_the_sampled_clock():
    """The roof at clock f: the sustained figure scaled from its own clock, capped by the
    burst figure; without a sample, the burst figure."""
    peaks = {"bf16_tflops": 1679.8, "bf16_tflops_sustained": 1394.0, "hbm_gbs": 6549.4,
             "sustained_mhz": 1335.0, "burst_mhz": None}
    assert bench.tensor_peak(peaks, None) == (1679.8, 1.0)
    p, sc = bench.tensor_peak(peaks, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0})
    assert (p, sc) == (1679.8, 1.0)                       # capped by the burst figure
    p, sc = bench.tensor_peak(peaks, {"sm_mhz": 1335.0, "sm_max_mhz": 1965.0})
    assert p == pytest.approx(1394.0)                     # the sustained point itself
    p, sc = bench.tensor_peak(peaks, {"sm_mhz": 1417.0, "sm_max_mhz": 1965.0})
    assert p == pytest.approx(1394.0 * 1417 / 1335) and sc == pytest.approx(p / 1679.8)
    # no recorded sustained clock: the burst figure scaled by clock / max clock
    peaks["sustained_mhz"] = None
    p, sc = bench.tensor_peak(peaks, {"sm_mhz": 1310.0, "sm_max_mhz": 1965.0})
    assert sc == pytest.approx(2 / 3) and p == pytest.approx(1679.8 * 2 / 3)


def test_measured_peaks_clock_keys(tmp_path, monkeypatch):
    """Clock entries of MEASURED_PEAKS.json are found by name (nested or flat)."""
    import json
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({
        "hbm_gbs": 6549.4, "bf16_tflops": 1679.8, "bf16_tflops_sustained": 1394.0,
        "clocks": {"bf16_sustained_sm_mhz_median": 1335, "bf16_burst_sm_mhz": 1860,
                   "sm_max_mhz": 1965}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "measured" and peaks["sustained_mhz"] == 1335.0
    assert peaks["burst_mhz"] == 1860.0
    monkeypatch.setattr(bench, "ROOT", str(tmp_path / "none"))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks["sustained_mhz"] == bench.FALLBACK_SUSTAINED_MHZ


def test_gemm_roofline_reproduces_from_its_per_launch_figures():
    """frac = per_launch.flops / per_launch.ms / (burst x clock ratio), for a tensor-bound
    gate/up launch (two launches per step, 4 steps)."""
    cfg = LayerConfig("u", T=16384, H=2048, E=128, k=8, I=768, routing="normal")
    counts = np.full((2, 128), 512, np.int32)
    units = bench.algorithmic_units(cfg, counts, 4, "fused", True)
    peaks = {"bf16_tflops": 1679.8, "bf16_tflops_sustained": 1394.0, "hbm_gbs": 6549.4,
             "sustained_mhz": 1335.0, "burst_mhz": None}
    m = {"units": units, "steps": 4, "dispatch": "fused",
         "prof": {"gateup": {"launches": 8, "ms": 8 * 0.4}},
         "clk": {"sm_mhz": 1450.0, "sm_max_mhz": 1965.0}}
    r = bench.gemm_roofline(m, peaks, "measured")
    pl = r["per_launch"]
    assert r["bound"] == "tensor"
    assert pl["flops"] == pytest.approx(4.0 * 65536 * 2048 * 768)
    tf = pl["flops"] / (pl["ms"] / 1e3) / 1e12
    assert r["frac"] == pytest.approx(tf / (1394.0 * 1450 / 1335))
    assert r["tensor_frac_of_burst"] == pytest.approx(tf / 1679.8)
    assert r["tensor_frac_of_burst_x_clock_ratio"] == pytest.approx(tf / (1679.8 * 1450 / 1965))
