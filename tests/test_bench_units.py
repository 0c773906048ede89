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
    assert sum(u["flops"].values()) == 18 * rows * H * I
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


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_summary_keeps_only_the_timed_window():
    """nvidia-smi lines (index, sm, max sm, power, active mask, hw, hw thermal, sw thermal,
    sw power cap): only samples inside the timed region (plus 0.1 s) count; the median SM
    clock and every active reason among them are reported."""
    s = bench.ClockSampler(0)
    s.proc = _DoneProc()
    ok = "0, {}, 1965, 900, 0x4, Not Active, Not Active, Not Active, {}"
    s.lines = [(0.5, ok.format(700, "Not Active")),      # before the region
               (1.0, ok.format(1400, "Active")),
               (1.2, ok.format(1500, "Not Active")),
               (1.4, ok.format(1450, "Active")),
               (1.55, ok.format(1300, "Not Active")),    # within the 0.1 s grace
               (3.0, "0, 600, 1965, 90, 0x1, Active, Not Active, Not Active, Not Active"),
               (3.1, "garbage")]
    out = s.stop(1.0, 1.5)
    assert out == {"sm_mhz": 1425.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 4}
    s.proc = _DoneProc()
    every = s.stop()
    assert every["samples"] == 6 and "hw_slowdown" in every["reasons"]
