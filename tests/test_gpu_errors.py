"""Error paths on the GPU: every one is a returned status, none faults or hangs."""
import numpy as np
import pytest
import torch

from gen import CONFIGS, layer_inputs

pytestmark = pytest.mark.gpu


def test_forward_bad_index_returns_status(moe):
    cfg = CONFIGS["tiny"]
    gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
    bad = gpu["idx"].clone()
    bad[100, 1] = cfg.E  # out of range
    with pytest.raises(moe.MoEError) as ei:
        moe.forward(gpu["hidden"], bad, gpu["w"], gpu["wgu"], gpu["wd"], num_chunks=2)
    assert ei.value.status == 2
    # the library stays usable
    out = moe.forward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"], gpu["wd"], num_chunks=2)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out.float()).all())


@pytest.mark.parametrize("dispatch,pair_gemms", [("fused", True), ("fused", False),
                                                 ("separate", False)])
@pytest.mark.parametrize("N", [1, 3, 4])
def test_forward_bad_index_leaves_output_untouched(moe, dispatch, pair_gemms, N):
    """The pipeline is enqueued before the host sees the metadata: every kernel after it
    must do nothing when an index is out of range (no row of `out` written), and the call
    still returns the index status."""
    cfg = CONFIGS["tiny"]
    gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
    bad = gpu["idx"].clone()
    bad[cfg.T - 1, 0] = -1
    out = torch.full((cfg.T, cfg.H), 7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as ei:
        moe.forward(gpu["hidden"], bad, gpu["w"], gpu["wgu"], gpu["wd"], num_chunks=N, out=out,
                    dispatch=dispatch, pair_gemms=pair_gemms)
    assert ei.value.status == 2
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())


def test_forward_workspace_too_small(moe):
    cfg = CONFIGS["tiny"]
    gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
    ws = moe.alloc_workspace(1024)
    with pytest.raises(moe.MoEError) as ei:
        moe.forward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"], gpu["wd"], workspace=ws)
    assert ei.value.status == 4


def test_forward_zero_tokens(moe):
    cfg = CONFIGS["tiny"]
    gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
    out = moe.forward(gpu["hidden"][:0], gpu["idx"][:0], gpu["w"][:0], gpu["wgu"], gpu["wd"],
                      num_chunks=4)
    assert out.shape == (0, cfg.H)


def test_device_status_clean_after_forward(moe):
    cfg = CONFIGS["tiny"]
    gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, 1, 2))
    moe.forward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"], gpu["wd"], num_chunks=2,
                workspace=ws)
    moe.check_device_status(ws)  # raises on a recorded timeout or bad index


def test_all_tokens_to_one_expert(moe):
    """Maximal skew: every copy goes to expert 5; the other experts are idle."""
    cfg = CONFIGS["tiny"]
    gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
    idx = torch.full_like(gpu["idx"], 5)
    a = moe.forward(gpu["hidden"], idx, gpu["w"], gpu["wgu"], gpu["wd"], num_chunks=1)
    b = moe.forward(gpu["hidden"], idx, gpu["w"], gpu["wgu"], gpu["wd"], num_chunks=3)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert bool(torch.isfinite(a.float()).all())


def test_bounded_wait_gives_up_and_reports_timeout(moe):
    """Failure detection on the device: a bounded mbarrier wait that nothing completes gives
    up after its limit (20 ms here), reports MOE_ERR_TIMEOUT through the status word and
    returns; the context stays usable (a forward right after it matches one before it)."""
    import time
    cfg = CONFIGS["tiny"]
    gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
    before = moe.forward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"], gpu["wd"], num_chunks=2)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert moe.selftest_wait_timeout(20000) == 6  # MOE_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    after = moe.forward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"], gpu["wd"], num_chunks=2)
    torch.cuda.synchronize()
    assert torch.equal(before, after)
