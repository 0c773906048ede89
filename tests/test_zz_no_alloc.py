"""moe_metadata_noalloc: the metadata entry point for callers that cannot allocate.

Some callers must not allocate device or pinned host memory where they need the routing
metadata (a runtime that owns all device memory through its own caching allocator, a
latency-critical serving path, a plugin handed only its inputs and outputs).  The
allocation-free entry point keeps its scratch in a fixed device array; here it is called
through the C ABI and checked against moe_metadata, which uses a caller workspace, on
consecutive calls (the array keeps the previous call's contents).  The results are
integers, so the comparison is exact.

This file is collected last on purpose, so that a run stopping at its first failure has
already run every other test; it passes alone as well.
"""
import ctypes

import numpy as np
import pytest
import torch

from gen import CONFIGS, routing

pytestmark = pytest.mark.gpu

MOE_ERR_ARG, MOE_ERR_INDEX, MOE_ERR_WORKSPACE = 1, 2, 4


def _p(a):
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        return a.ctypes.data_as(ctypes.c_void_p)
    return ctypes.c_void_p(a.data_ptr())


def _noalloc(lib, idx, E, G, N):
    T, k = idx.shape
    n = max(N, 1)
    out = dict(send=np.full((n, max(G, 1)), -7, np.int32), recv=np.full((n, max(G, 1)), -7, np.int32),
               counts=np.full((n, E), -7, np.int32), bounds=np.full(n + 1, -7, np.int64),
               dst=torch.full((T * k,), -7, dtype=torch.int32, device="cuda"),
               src_tok=torch.full((T * k,), -7, dtype=torch.int32, device="cuda"))
    st = lib.moe_metadata_noalloc(_p(idx), T, k, E, G, N, _p(out["send"]), _p(out["recv"]),
                                  _p(out["counts"]), _p(out["bounds"]), _p(out["dst"]),
                                  _p(out["src_tok"]),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


def _same_as_workspace_version(moe, idx, E, G, N):
    lib = moe.load()
    st, got = _noalloc(lib, idx, E, G, N)
    assert st == 0, moe.status_string(st)
    ref = moe.metadata(idx, E, G, N, with_permutation=True)
    for key in ("send", "recv", "counts", "bounds"):
        np.testing.assert_array_equal(got[key], ref[key], err_msg=key)
    assert torch.equal(got["dst"], ref["dst"])
    assert torch.equal(got["src_tok"], ref["src_tok"])


@pytest.fixture(scope="module")
def lib(moe):
    lib = moe.load()
    lib.moe_metadata_noalloc.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                         ctypes.c_int32, ctypes.c_int32, ctypes.c_int32] + \
        [ctypes.c_void_p] * 7
    lib.moe_metadata_noalloc.restype = ctypes.c_int
    return lib


def test_noalloc_matches_workspace_metadata_on_consecutive_calls(moe, lib):
    big = CONFIGS["qwen3"]
    small = CONFIGS["edge_varlen"]
    idx_big = torch.from_numpy(routing(big)[0]).cuda()
    idx_small = torch.from_numpy(routing(small)[0]).cuda()
    # two calls in a row with different shapes, then the first shape again: each call must
    # be unaffected by what the previous one left in the shared scratch array
    _same_as_workspace_version(moe, idx_big, big.E, 4, 4)
    _same_as_workspace_version(moe, idx_small, small.E, 8, 8)
    _same_as_workspace_version(moe, idx_big, big.E, 4, 4)
    ds = CONFIGS["deepseek"]
    idx_ds = torch.from_numpy(routing(ds)[0]).cuda()
    _same_as_workspace_version(moe, idx_ds, ds.E, ds.G, 1)
    _same_as_workspace_version(moe, idx_ds, ds.E, ds.G, 4)


def test_noalloc_bad_index_then_good_call(moe, lib):
    """A flagged bad index must not leak into the next call through the shared array."""
    idx = np.zeros((300, 2), np.int32)
    idx[123, 0] = 9
    st, _ = _noalloc(lib, torch.from_numpy(idx).cuda(), 8, 1, 2)
    assert st == MOE_ERR_INDEX
    idx[123, 0] = 3
    _same_as_workspace_version(moe, torch.from_numpy(idx).cuda(), 8, 2, 2)


def test_noalloc_rejects_sizes_beyond_the_array(moe, lib):
    # E = 1024 experts over 300 chunks needs 300*1025*4 B of offsets alone (> 1 MiB)
    idx = torch.zeros((600, 2), dtype=torch.int32, device="cuda")
    st, _ = _noalloc(lib, idx, 1024, 1, 300)
    assert st == MOE_ERR_WORKSPACE
    # dst_rows is required
    n = np.zeros(8, np.int64)
    st = lib.moe_metadata_noalloc(_p(idx), 600, 2, 8, 1, 1, _p(n), _p(n), _p(n), _p(n), None,
                                  None, None)
    assert st == MOE_ERR_ARG


def test_noalloc_defaults_and_empty_input(moe, lib):
    """num_chunks=0 (no split) and ep_groups=0 (one group) resolve as moe_metadata resolves
    them, and T=0 returns zero splits, counts and chunk bounds."""
    cfg = CONFIGS["edge"]
    idx = torch.from_numpy(routing(cfg)[0]).cuda()
    _same_as_workspace_version(moe, idx, cfg.E, 0, 0)
    _same_as_workspace_version(moe, idx, cfg.E, 0, 3)
    _same_as_workspace_version(moe, idx, cfg.E, 4, 0)
    empty = torch.zeros((0, cfg.k), dtype=torch.int32, device="cuda")
    for G, N in ((0, 0), (4, 3)):
        _same_as_workspace_version(moe, empty, cfg.E, G, N)
