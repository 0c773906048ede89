"""GPU metadata (splits, counts, permutation) against the oracle: bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from gen import CONFIGS, routing

pytestmark = pytest.mark.gpu


def _compare(moe, idx_np, E, G, N, S=0):
    idx = torch.from_numpy(idx_np).cuda()
    got = moe.metadata(idx, E, G, N, with_permutation=True, chunk_size=S)
    ref = oracle.metadata(idx_np, E, G, N, chunk_size=S)
    np.testing.assert_array_equal(got["bounds"], ref["bounds"])
    np.testing.assert_array_equal(got["counts"], ref["counts"])
    np.testing.assert_array_equal(got["send"], ref["send"])
    np.testing.assert_array_equal(got["recv"], ref["recv"])
    np.testing.assert_array_equal(got["dst"].cpu().numpy(), ref["dst"])
    np.testing.assert_array_equal(got["src_tok"].cpu().numpy(), ref["src_tok"])
    assert int(got["send"].sum()) == idx_np.size  # splits sum to T*k
    return got


CASES = [(name, N) for name in ["tiny", "edge", "edge_pair01", "edge_varlen", "edge_varlen7",
                                "qwen3", "deepseek", "mixtral"]
         for N in CONFIGS[name].chunks]


@pytest.mark.parametrize("name,N", CASES)
def test_metadata_configs(moe, name, N):
    cfg = CONFIGS[name]
    idx, _ = routing(cfg)
    _compare(moe, idx, cfg.E, cfg.G, N)


def test_metadata_edge_structure(moe):
    """The edge layer's Zipf routing leaves exactly 20 experts without tokens; the
    variable-length case at N=8 has exactly one empty chunk."""
    cfg = CONFIGS["edge"]
    idx, _ = routing(cfg)
    got = _compare(moe, idx, cfg.E, 1, 1)
    assert int((got["counts"][0] == 0).sum()) == 20
    v = CONFIGS["edge_varlen"]
    idx, _ = routing(v)
    got = _compare(moe, idx, v.E, 1, 8)
    sizes = np.diff(got["bounds"])
    assert sizes.tolist() == [7] * 7 + [0]
    assert got["counts"][7].sum() == 0


@pytest.mark.parametrize("seed", range(6))
def test_metadata_random_shapes(moe, seed):
    rng = np.random.default_rng(100 + seed)
    for _ in range(8):
        E = int(rng.choice([1, 2, 3, 8, 64, 256, 1000, 1024]))
        k = int(rng.integers(1, min(E, 32) + 1))
        T = int(rng.integers(0, 3000))
        G = int(rng.choice([g for g in (1, 2, 4, 8, 16) if E % g == 0]))
        N = int(rng.integers(0, 12))
        if T == 0:
            continue
        idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
        _compare(moe, idx, E, G, N)


@pytest.mark.parametrize("S", [1, 7, 143, 256, 999, 1000, 5000])
def test_metadata_chunk_size(moe, S):
    """Chunks of exactly S tokens (moe_chunk_size, section 操作指南 step 3)."""
    cfg = CONFIGS["edge"]
    idx, _ = routing(cfg)
    got = _compare(moe, idx, cfg.E, 4, 0, S)
    assert got["bounds"][1] == min(S, cfg.T)


def test_metadata_many_tiles_per_chunk(moe):
    """T*k far above one tile's 2048 copies, with a skewed expert: the scan over tiles."""
    rng = np.random.default_rng(5)
    T, k, E = 40000, 4, 16
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    idx[rng.random((T, k)) < 0.5] = 3
    for N in (1, 3, 16):
        _compare(moe, idx, E, 4, N)


def test_metadata_more_tiles_than_resident_ctas(moe):
    """More tiles than one cooperative grid holds at once (at most 5 CTAs of the largest
    shared-memory size per SM, 148 SMs): the metadata kernel's CTAs each loop over several
    tiles in every phase, and a bad index in a late tile still reaches the status word."""
    rng = np.random.default_rng(11)
    T, k, E = 60000, 32, 1024  # 64 tokens per tile of 2048 copies: ~940 tiles
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    idx[rng.random((T, k)) < 0.2] = 17
    for N in (1, 5):
        _compare(moe, idx, E, 8, N)
    bad = idx.copy()
    bad[T - 1, 3] = E
    with pytest.raises(moe.MoEError) as ei:
        moe.metadata(torch.from_numpy(bad).cuda(), E, 8, 5)
    assert ei.value.status == 2
    _compare(moe, idx, E, 8, 5)


def test_metadata_bad_index(moe):
    idx = np.zeros((100, 2), np.int32)
    idx[37, 1] = 8
    with pytest.raises(moe.MoEError) as ei:
        moe.metadata(torch.from_numpy(idx).cuda(), 8, 1, 2)
    assert ei.value.status == 2
    idx[37, 1] = -1
    with pytest.raises(moe.MoEError) as ei:
        moe.metadata(torch.from_numpy(idx).cuda(), 8, 1, 2)
    assert ei.value.status == 2
    # the next good call succeeds (the status word is reset per call)
    idx[37, 1] = 7
    _compare(moe, idx, 8, 1, 2)
