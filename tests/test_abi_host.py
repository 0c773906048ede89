"""The C ABI library without a GPU: it loads, exports every declared entry point, and its
host-only logic (chunk bounds, workspace sizes, argument checks) behaves as declared.

Argument checks run on the host before any CUDA call, so they are exercised here with
dummy (never dereferenced) pointers."""
import ctypes
import os
import re

import numpy as np
import pytest

import expert_router_top_b200 as moe
import oracle
from gen import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for n in ["moe_metadata", "moe_forward", "moe_workspace_bytes", "moe_status_string",
              "moe_chunk_bounds", "moe_permute", "moe_grouped_gateup", "moe_grouped_down",
              "moe_unpermute"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    L = moe.load()
    for name in declared_symbols():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_abi_version_and_status_strings():
    L = moe.load()
    assert L.moe_abi_version() == 4
    for code, name in moe.STATUS_NAMES.items():
        assert moe.status_string(code).startswith(name)
    assert "unknown" in moe.status_string(99)


def test_chunk_bounds_match_oracle():
    for T in [0, 1, 7, 49, 1000, 16384]:
        for N in [0, 1, 2, 3, 4, 7, 8]:
            assert moe.chunk_bounds(T, N).tolist() == oracle.chunk_bounds(T, N).tolist()
    with pytest.raises(moe.MoEError):
        moe.chunk_bounds(-1, 2)


def test_resolve_chunks_matches_oracle():
    """num_chunks / chunk_size precedence (Chunk MoE, section 操作指南 step 3)."""
    import warnings
    for T in (0, 1, 10, 49, 1000, 16384):
        for N in (0, 1, 3, 8):
            for S in (0, 1, 4, 143, 5000):
                ref_n, ref_tc, ref_warn = oracle.resolve_chunks(T, N, S)
                with warnings.catch_warnings(record=True) as caught:
                    warnings.simplefilter("always")
                    n, tc = moe.resolve_chunks(T, N, S)
                assert n == ref_n and tc == ref_tc, (T, N, S)
                assert (len(caught) > 0) == ref_warn, (T, N, S)
                if ref_warn:
                    assert "moe_num_chunks" in str(caught[0].message)


def test_chunk_size_workspace_and_limits():
    cfg = CONFIGS["qwen3"]
    # chunks of 4096 tokens: the same buffers as num_chunks=4
    a = moe.workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.G, 0, 4096)
    b = moe.workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.G, 4, 0)
    assert a == b
    # a chunk size above T is one chunk of T tokens
    assert moe.workspace_bytes(100, 64, 64, 8, 2, 1, 0, 10**6) == moe.workspace_bytes(
        100, 64, 64, 8, 2, 1, 1, 0)
    assert moe.workspace_bytes(100, 64, 64, 8, 2, 1, 0, -5) == 0
    with pytest.raises(moe.MoEError):
        moe.resolve_chunks(10, 0, -1)
    with pytest.raises(moe.MoEError):  # more than MOE_MAX_CHUNKS chunks
        moe.resolve_chunks(10**9, 0, 1)


def _ws(cfg, N):
    return moe.workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.G, N)


def _expert_buffer_bytes(cfg, N):
    """Expert workspace the pair double buffer needs by construction: min(N,2) buffers
    of ceil(T/N)*k rows of (H + I) bf16."""
    n = max(N, 1)
    tc = -(-cfg.T // n)
    return min(n, 2) * tc * cfg.k * (cfg.H + cfg.I) * 2


@pytest.mark.parametrize("name", ["mixtral", "qwen3", "deepseek", "tiny", "edge"])
def test_workspace_follows_pair_double_buffer(name):
    """W_pair = O(2 * T_chunk) (Chunk MoE, section 一组关键公式): N=2 keeps the unsplit
    size, N=4 halves it; the query adds only small metadata arrays on top."""
    cfg = CONFIGS[name]
    for N in (1, 2, 4, 8):
        ws = _ws(cfg, N)
        buf = _expert_buffer_bytes(cfg, N)
        assert buf <= ws <= buf + 64 * 1024 + 8 * cfg.T * cfg.k + 16 * N * (cfg.E + 8) + 4096
    if cfg.T % 4 == 0:
        assert _expert_buffer_bytes(cfg, 4) * 2 == _expert_buffer_bytes(cfg, 1)
        assert _ws(cfg, 4) <= 0.6 * _ws(cfg, 1)  # at least the 40 % cut the method targets


def _bwd_row_buffer_bytes(cfg, N):
    """Backward rows by construction: the units are the pairs of chunks, ceil(N/2) of them,
    each of at most 2*ceil(T/N) tokens, whose rows padded per expert to 64 fit in
    tokens*k + 63*E rows; the permuted rows X (H wide, bf16) and their routing weights (fp32)
    in min(units, 2) unit buffers, and one unit set of [g u] (2I), w h (I), dX (H) and dY (H),
    all bf16, with two fp32 partials of d_w per 256 columns of I."""
    n = max(N, 1)
    tu = min(2 * -(-cfg.T // n), cfg.T)
    units = -(-n // 2)
    rows = tu * cfg.k + 63 * cfg.E
    per_row = (min(units, 2) * (2 * cfg.H + 4) + 2 * (3 * cfg.I + 2 * cfg.H)
               + 4 * 2 * -(-cfg.I // 256))
    return per_row * rows, units, tu


@pytest.mark.parametrize("name", ["mixtral", "qwen3", "deepseek", "tiny", "edge", "edge_varlen"])
def test_backward_workspace_follows_pair_units(name):
    """The backward's workspace is its row buffers plus metadata arrays (three int32 per
    routed copy, per-unit offsets and histograms): N=2 is one pair, the size of N=1, and
    N=4 holds a pair in flight and the next one's permuted rows."""
    cfg = CONFIGS[name]
    ws = {}
    for N in (1, 2, 3, 4, 8):
        ws[N] = moe.backward_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.G, N)
        buf, units, tu = _bwd_row_buffer_bytes(cfg, N)
        meta = (12 * cfg.T * cfg.k + 4 * cfg.E * units * (tu * cfg.k // 2048 + 2)
                + 8 * (units + 2) * (cfg.E + 8) + 20 * 256)
        assert buf <= ws[N] <= buf + meta, (N, ws[N] - buf, meta)
    assert ws[2] == ws[1]
    if cfg.T >= 4096:
        assert ws[8] < ws[4] < ws[1]
    if name == "qwen3":
        assert ws[4] < 0.7 * ws[1]  # 1.55 vs 2.35 GB


def test_workspace_rejects_bad_shapes():
    assert moe.workspace_bytes(16, 12, 16, 4, 2) == 0       # H % 8
    assert moe.workspace_bytes(16, 16, 16, 4, 5) == 0       # k > E
    assert moe.workspace_bytes(16, 16, 16, 6, 2, 4) == 0    # E % G
    assert moe.workspace_bytes(16, 16, 16, 4, 2, 1, -1) == 0
    assert moe.workspace_bytes(16, 16, 16, 2048, 2) == 0    # E beyond the kernel limit
    assert moe.workspace_bytes(0, 16, 16, 4, 2) > 0
    assert moe.metadata_workspace_bytes(100, 2, 8, 2, 4) > 0
    assert moe.metadata_workspace_bytes(100, 9, 8, 1, 1) == 0


FAKE = 0x10000  # a 64 KB-aligned address that is never dereferenced


def _fwd(shape, ptrs=None, ws_bytes=1 << 40):
    L = moe.load()
    p = dict(hidden=FAKE, idx=FAKE, w=FAKE, wgu=FAKE, wd=FAKE, out=FAKE, ws=FAKE)
    p.update(ptrs or {})
    v = ctypes.c_void_p
    return L.moe_forward(ctypes.byref(shape) if shape is not None else None, v(p["hidden"]),
                         v(p["idx"]), v(p["w"]), v(p["wgu"]), v(p["wd"]), v(p["out"]),
                         v(p["ws"]), ws_bytes, None)


def test_forward_argument_checks_run_on_host():
    good = moe.shape(64, 64, 64, 8, 2, 2, 4)
    assert _fwd(None) == 1                                            # MOE_ERR_ARG
    assert _fwd(moe.shape(64, 60, 64, 8, 2)) == 1                     # H % 8
    assert _fwd(moe.shape(64, 64, 64, 8, 9)) == 1                     # k > E
    assert _fwd(moe.shape(64, 64, 64, 8, 2, 3)) == 1                  # E % G
    assert _fwd(moe.shape(64, 64, 64, 8, 2, 1, -2)) == 1              # N < 0
    assert _fwd(moe.shape(64, 64, 64, 4096, 2)) == 7                  # MOE_ERR_UNSUPPORTED
    assert _fwd(moe.shape(64, 64, 64, 64, 33)) == 7                   # k > MOE_MAX_TOPK
    assert _fwd(good, dict(hidden=0)) == 1                            # null pointer
    assert _fwd(good, dict(out=FAKE + 8)) == 3                        # MOE_ERR_ALIGN
    assert _fwd(good, dict(wgu=FAKE + 4)) == 3
    assert _fwd(good, dict(ws=FAKE + 16)) == 3                        # workspace 256 B
    assert _fwd(good, ws_bytes=1024) == 4                             # MOE_ERR_WORKSPACE
    assert _fwd(moe.shape(0, 64, 64, 8, 2)) == 0                      # T = 0: no work


def test_host_workspace_adds_staging():
    for name in ("qwen3", "tiny"):
        cfg = CONFIGS[name]
        for N in (1, 2, 4):
            dev = moe.workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.G, N)
            host = moe.workspace_bytes_host(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.G, N)
            tc = -(-cfg.T // N)
            staging = 8 * cfg.T * cfg.k + min(N, 2) * 2 * tc * cfg.H * 2
            assert dev + staging <= host <= dev + staging + 8 * 256


def test_forward_ex_rejects_unknown_flags():
    L = moe.load()
    v = ctypes.c_void_p
    good = moe.shape(64, 64, 64, 8, 2, 2, 4)
    for flags in (8, 3):  # an unknown bit; both dispatch flags at once
        assert L.moe_forward_ex(ctypes.byref(good), v(FAKE), v(FAKE), v(FAKE), v(FAKE), v(FAKE),
                                v(FAKE), v(FAKE), 1 << 40, flags, None) == 1


def test_stage_argument_checks_run_on_host():
    L = moe.load()
    v = ctypes.c_void_p
    assert L.moe_permute(v(FAKE), v(FAKE), 4, 12, 2, v(FAKE), None) == 1       # H % 8
    assert L.moe_permute(v(FAKE + 2), v(FAKE), 4, 16, 2, v(FAKE), None) == 3   # align
    assert L.moe_permute(v(0), v(FAKE), 0, 16, 2, v(FAKE), None) == 0          # Tc = 0
    assert L.moe_unpermute(v(FAKE), v(FAKE), v(FAKE), 4, 16, 40, v(FAKE), None) == 1
    counts = np.array([3, 1], np.int32)
    cptr = counts.ctypes.data_as(ctypes.c_void_p)
    # counts that do not sum to rows
    assert L.moe_grouped_gateup(v(FAKE), 5, 16, 16, 2, v(FAKE), cptr, v(FAKE), v(FAKE),
                                v(FAKE), None) == 1
    assert L.moe_grouped_down(v(FAKE), 4, 16, 16, 2, v(FAKE), cptr, v(FAKE), v(FAKE + 8),
                              v(FAKE), None) == 3


def test_metadata_argument_checks_run_on_host():
    L = moe.load()
    v = ctypes.c_void_p
    host = np.zeros(64, np.int64)
    hp = host.ctypes.data_as(ctypes.c_void_p)
    # k > E, E % G, null host outputs, unaligned workspace
    assert L.moe_metadata(v(FAKE), 4, 5, 4, 1, 1, hp, hp, hp, hp, None, None, v(FAKE), 1 << 30,
                          None) == 1
    assert L.moe_metadata(v(FAKE), 4, 2, 6, 4, 1, hp, hp, hp, hp, None, None, v(FAKE), 1 << 30,
                          None) == 1
    assert L.moe_metadata(v(FAKE), 4, 2, 4, 1, 1, None, hp, hp, hp, None, None, v(FAKE), 1 << 30,
                          None) == 1
    assert L.moe_metadata(v(FAKE), 4, 2, 4, 1, 1, hp, hp, hp, hp, None, None, v(FAKE + 64),
                          1 << 30, None) == 3
    assert L.moe_metadata(v(FAKE), 4, 2, 4, 1, 1, hp, hp, hp, hp, None, None, v(FAKE), 16,
                          None) == 4
    # T = 0: bounds and zero splits, no device work
    send = np.full((2, 2), 7, np.int32)
    cnt = np.full((2, 4), 7, np.int32)
    b = np.full(3, 7, np.int64)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    assert L.moe_metadata(None, 0, 2, 4, 2, 2, p(send), p(send), p(cnt), p(b), None, None,
                          None, 0, None) == 0
    assert b.tolist() == [0, 0, 0] and not send.any() and not cnt.any()


def test_profile_api_without_launches():
    moe.profile_enable(True)
    prof = moe.profile_read()
    assert prof["kernels"] == 0 and all(prof[k]["launches"] == 0 for k in moe.KERNEL_KINDS)
    moe.profile_enable(False)


def test_forward_dispatch_choice():
    """moe_forward_dispatch (host logic): flags force a dispatch; flags = 0 gathers in the
    gate/up GEMM (fused) at every shape and chunk count."""
    import expert_router_top_b200 as moe
    q, m, d = CONFIGS["qwen3"], CONFIGS["mixtral"], CONFIGS["deepseek"]
    for N in (1, 2, 4, 8):
        assert moe.forward_dispatch(q.T, q.H, q.I, q.E, q.k, num_chunks=N) == "fused"
        assert moe.forward_dispatch(m.T, m.H, m.I, m.E, m.k, num_chunks=N) == "fused"
        assert moe.forward_dispatch(d.T, d.H, d.I, d.E, d.k, ep_groups=d.G, num_chunks=N) == "fused"
    assert moe.forward_dispatch(95, 64, 96, 8, 2) == "fused"
    assert moe.forward_dispatch(q.T, q.H, q.I, q.E, q.k, "separate", num_chunks=4) == "separate"
    assert moe.forward_dispatch(m.T, m.H, m.I, m.E, m.k, "separate") == "separate"
    assert moe.forward_dispatch(m.T, m.H, m.I, m.E, m.k, "fused") == "fused"
    L = moe.load()
    s = moe.shape(16, 64, 64, 4, 2, 1, 1, 0)
    assert L.moe_forward_dispatch(ctypes.byref(s), 3) == -1
    assert L.moe_forward_dispatch(ctypes.byref(s), 8) == -1
    assert L.moe_forward_dispatch(ctypes.byref(s), 4) == 1  # a valid flag; auto: fused


def test_selftest_argument_checks_run_on_host():
    L = moe.load()
    v = ctypes.c_void_p
    assert L.moe_selftest_wait_timeout(None, 1000, None) == 1          # null status
    assert L.moe_selftest_wait_timeout(v(FAKE), 0, None) == 1          # limit 0
    assert L.moe_selftest_wait_timeout(v(FAKE), 2000000, None) == 1    # limit above 1 s
    assert L.moe_selftest_wait_timeout(v(FAKE + 2), 1000, None) == 3   # misaligned


def test_checks_api_in_the_regular_build():
    L = moe.load()
    assert L.moe_checks_enabled() == 0
    assert L.moe_checks_read(None) == 1  # null flags


def test_profile_timeline_argument_checks_and_empty_list():
    """With nothing timed the timeline call touches no device: it returns zero records;
    a null count, a negative capacity or a null array with room are MOE_ERR_ARG."""
    L = moe.load()
    moe.profile_enable(True)
    n = ctypes.c_int32(-1)
    recs = (moe.LaunchRecord * 4)()
    assert L.moe_profile_timeline(recs, 4, ctypes.byref(n)) == 0 and n.value == 0
    assert L.moe_profile_timeline(None, 0, ctypes.byref(n)) == 0 and n.value == 0
    assert L.moe_profile_timeline(recs, 4, None) == 1
    assert L.moe_profile_timeline(recs, -1, ctypes.byref(n)) == 1
    assert L.moe_profile_timeline(None, 4, ctypes.byref(n)) == 1
    assert moe.profile_timeline() == []
    moe.profile_enable(False)
    assert ctypes.sizeof(moe.LaunchRecord) == 40
