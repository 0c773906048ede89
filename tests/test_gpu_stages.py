"""Each kernel on its own against the oracle's stage definitions.

Inputs are drawn by the seeded generator (never taken from the CUDA path); expert row
ranges come from the oracle's metadata or are chosen by hand to hit ragged tiles."""
import numpy as np
import pytest
import torch

import oracle
from gen import CONFIGS, bf16_normal, bits, routing
from parity import assert_gemm_close, assert_unpermute_close, to_f64

pytestmark = pytest.mark.gpu


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def _expert_of_row(counts):
    return np.repeat(np.arange(len(counts), dtype=np.int32), counts)


# ---------------------------------------------------------------------------- permute

@pytest.mark.parametrize("name", ["tiny", "edge", "edge_pair01", "qwen3"])
def test_permute_bit_exact(moe, name):
    cfg = CONFIGS[name]
    idx, _ = routing(cfg)
    x = bf16_normal((cfg.T, cfg.H), 1.0, 11)
    m = oracle.metadata(idx, cfg.E, 1, 1)
    dst = torch.from_numpy(m["dst"]).cuda()
    X = moe.permute(x.cuda(), dst, cfg.k)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bits(X), oracle.permute(bits(x), m["dst"], cfg.k))


# -------------------------------------------------------------------------- unpermute

@pytest.mark.parametrize("name", ["tiny", "edge", "edge_pair01", "qwen3"])
def test_unpermute(moe, name):
    cfg = CONFIGS[name]
    idx, w = routing(cfg)
    m = oracle.metadata(idx, cfg.E, 1, 1)
    Y = bf16_normal((cfg.T * cfg.k, cfg.H), 1.0, 12)
    out = moe.unpermute(Y.cuda(), torch.from_numpy(m["dst"]).cuda(),
                        torch.from_numpy(w).cuda(), cfg.k)
    ref = oracle.unpermute(bits(Y), m["dst"], w, cfg.k)
    assert_unpermute_close(out, ref, name)


def test_unpermute_is_deterministic(moe):
    cfg = CONFIGS["edge"]
    idx, w = routing(cfg)
    m = oracle.metadata(idx, cfg.E, 1, 1)
    Y = bf16_normal((cfg.T * cfg.k, cfg.H), 1.0, 13).cuda()
    dst = torch.from_numpy(m["dst"]).cuda()
    wt = torch.from_numpy(w).cuda()
    a = moe.unpermute(Y, dst, wt, cfg.k)
    b = moe.unpermute(Y, dst, wt, cfg.k)
    assert torch.equal(a, b)


# ------------------------------------------------------------------ grouped GEMMs

GEMM_CASES = {
    # name: (H, I, counts)
    "tiny": (256, 512, None),
    "ragged": (200, 136, [0, 1, 127, 128, 129, 300]),
    "one_row_experts": (64, 64, [1] * 7 + [0]),
    "edge": (1024, 1408, None),
    "skewed": (512, 384, [0, 0, 2000, 3, 0, 640, 1, 0]),
    # an expert of 40 row tiles spans several 16-tile raster bands
    "big_expert": (256, 264, [5000, 3, 0, 700]),
}


def _gemm_case(name):
    H, I, counts = GEMM_CASES[name]
    if counts is None:
        cfg = CONFIGS[name]
        idx, _ = routing(cfg)
        counts = oracle.metadata(idx, cfg.E, 1, 1)["counts"][0]
    counts = np.asarray(counts, np.int32)
    return H, I, counts


@pytest.mark.parametrize("name", list(GEMM_CASES))
def test_grouped_gateup(moe, name):
    H, I, counts = _gemm_case(name)
    E, rows = len(counts), int(counts.sum())
    X = bf16_normal((rows, H), 1.0, 21)
    wgu = bf16_normal((E, 2 * I, H), 1.0 / np.sqrt(H), 22)
    offs = torch.from_numpy(_offsets(counts)).cuda()
    Act, status = moe.grouped_gateup(X.cuda(), offs, counts, wgu.cuda())
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    ref = oracle.gateup_rows(bits(X), _expert_of_row(counts), bits(wgu))
    assert_gemm_close(Act, ref, f"gateup/{name}")


@pytest.mark.parametrize("name", list(GEMM_CASES))
def test_grouped_down(moe, name):
    H, I, counts = _gemm_case(name)
    E, rows = len(counts), int(counts.sum())
    A = bf16_normal((rows, I), 1.0, 31)
    wd = bf16_normal((E, H, I), 1.0 / np.sqrt(I), 32)
    offs = torch.from_numpy(_offsets(counts)).cuda()
    Y, status = moe.grouped_down(A.cuda(), offs, counts, wd.cuda())
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    ref = oracle.down_rows(bits(A), _expert_of_row(counts), bits(wd))
    assert_gemm_close(Y, ref, f"down/{name}")


def test_gemm_rows_outside_the_experts_are_untouched(moe):
    """Masked epilogue: a tile's rows past its expert's end are never stored, so a
    sentinel pattern in rows beyond offsets[E] survives."""
    H, I = 128, 128
    counts = np.array([5, 0, 130], np.int32)
    rows = int(counts.sum())
    X = bf16_normal((rows + 64, H), 1.0, 41).cuda()
    wgu = bf16_normal((3, 2 * I, H), 0.1, 42).cuda()
    Act = torch.full((rows + 64, I), 7.0, dtype=torch.bfloat16, device="cuda")
    offs = torch.from_numpy(_offsets(counts)).cuda()
    moe.grouped_gateup(X[:rows], offs, counts, wgu, Act=Act[:rows])
    torch.cuda.synchronize()
    assert bool((Act[rows:] == 7.0).all())


def test_gemm_position_independence(moe):
    """A row's result does not depend on where it sits in a tile: shifting every expert's
    rows by a few positions (an extra leading expert) gives bit-identical rows."""
    H, I = 256, 256
    counts = np.array([100, 300, 7], np.int32)
    E = len(counts)
    X = bf16_normal((int(counts.sum()), H), 1.0, 51)
    wgu = bf16_normal((E, 2 * I, H), 1.0 / 16, 52).cuda()
    wd = bf16_normal((E, H, I), 1.0 / 16, 53).cuda()
    offs = torch.from_numpy(_offsets(counts)).cuda()
    a, _ = moe.grouped_gateup(X.cuda(), offs, counts, wgu)
    y, _ = moe.grouped_down(a, offs, counts, wd)
    # prepend 37 rows of a new expert 0 (weights zero-padded in front)
    pad = 37
    counts2 = np.concatenate([[pad], counts]).astype(np.int32)
    X2 = torch.cat([bf16_normal((pad, H), 1.0, 54), X])
    wgu2 = torch.cat([torch.zeros((1, 2 * I, H), dtype=torch.bfloat16, device="cuda"), wgu])
    wd2 = torch.cat([torch.zeros((1, H, I), dtype=torch.bfloat16, device="cuda"), wd])
    offs2 = torch.from_numpy(_offsets(counts2)).cuda()
    a2, _ = moe.grouped_gateup(X2.cuda(), offs2, counts2, wgu2)
    y2, _ = moe.grouped_down(a2, offs2, counts2, wd2)
    torch.cuda.synchronize()
    assert torch.equal(a2[pad:], a)
    assert torch.equal(y2[pad:], y)
