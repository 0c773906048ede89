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
