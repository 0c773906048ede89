"""Expert parallelism on the GPU through the C ABI.

One GPU stands in for W ranks in two ways, neither with a kernel that waits for another:
  - in one process (expert_router_top_b200.ep.forward_emulated): W receive buffers on the
    device, dispatches of every source, then every rank's GEMMs, then every combine;
  - in two processes on the same GPU, each mapping the other's receive buffer with CUDA
    IPC (the peer pointers of the NVLink path), the phases ordered by gloo barriers.
Both must give, bit for bit, moe_forward over all ranks' tokens with all experts (each row
meets the same GEMM and the same ascending-j sum), which is itself checked against the
oracle within the layer's tolerance."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from gen import CONFIGS, LayerConfig, bits, layer_inputs
from parity import assert_layer_close

pytestmark = pytest.mark.gpu


def _split(cpu, W):
    parts = np.array_split(np.arange(cpu["hidden"].shape[0]), W)
    return parts, [{k: cpu[k][torch.from_numpy(p)].contiguous().cuda()
                    for k in ("hidden", "idx", "w")} for p in parts]


@pytest.mark.parametrize("name,W,N", [("tiny", 2, 1), ("tiny", 4, 3), ("edge", 8, 2),
                                      ("edge_pair01", 2, 2), ("edge_varlen", 4, 8)])
def test_ep_emulated_equals_single_gpu(moe, name, W, N):
    from expert_router_top_b200 import ep
    cfg = CONFIGS[name]
    cpu = layer_inputs(cfg)
    gpu = {k: v.cuda() for k, v in cpu.items()}
    ref = moe.forward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"], gpu["wd"], num_chunks=N)
    parts, ranks = _split(cpu, W)
    outs = ep.forward_emulated([r["hidden"] for r in ranks], [r["idx"] for r in ranks],
                               [r["w"] for r in ranks], gpu["wgu"], gpu["wd"], num_chunks=N)
    torch.cuda.synchronize()
    for p, o in zip(parts, outs):
        assert torch.equal(o, ref[torch.from_numpy(p).cuda()]), f"{name} W={W} N={N}"
    if cfg.T * cfg.k <= 8192:
        full = oracle.forward(bits(cpu["hidden"]), cpu["idx"].numpy(), cpu["w"].numpy(),
                              bits(cpu["wgu"]), bits(cpu["wd"]))
        assert_layer_close(torch.cat(outs)[torch.from_numpy(np.argsort(np.concatenate(parts)))
                                           .cuda()], full, f"EP {name} W={W}")


def test_ep_abi_checks(moe):
    L = moe.load()
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    i = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    t = torch.zeros(2, dtype=torch.int64, device="cuda")
    # E % W != 0, W beyond the limit, misaligned hidden: nothing launched
    assert L.moe_ep_dispatch(x.data_ptr(), i.data_ptr(), i.data_ptr(), i.data_ptr(),
                             t.data_ptr(), 4, 64, 2, 6, 4, 8, None) == 1
    assert L.moe_ep_dispatch(x.data_ptr(), i.data_ptr(), i.data_ptr(), i.data_ptr(),
                             t.data_ptr(), 4, 64, 2, 128, 128, 8, None) == 7
    assert L.moe_ep_dispatch(x.data_ptr() + 2, i.data_ptr(), i.data_ptr(), i.data_ptr(),
                             t.data_ptr(), 4, 64, 2, 8, 2, 8, None) == 3
    assert L.moe_ep_combine(t.data_ptr(), i.data_ptr(), i.data_ptr(), i.data_ptr(), None,
                            4, 64, 2, 8, 2, 8, x.data_ptr(), None) == 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_rank(rank, world, port, name, N, results):
    import datetime

    import torch.distributed as dist

    import expert_router_top_b200 as moe
    from expert_router_top_b200.ep import EPGroup
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    torch.cuda.set_device(0)
    try:
        cfg = CONFIGS[name]
        cpu = layer_inputs(cfg)
        parts = np.array_split(np.arange(cfg.T), world)
        mine = torch.from_numpy(parts[rank])
        El = cfg.E // world
        tc = max(-(-len(p) // N) for p in parts)
        grp = EPGroup(dist, world * tc * cfg.k, cfg.H, cfg.I, torch.device("cuda", 0))
        out = grp.forward(cpu["hidden"][mine].cuda(), cpu["idx"][mine].cuda(),
                          cpu["w"][mine].cuda(), cpu["wgu"][rank * El:(rank + 1) * El].cuda(),
                          cpu["wd"][rank * El:(rank + 1) * El].cuda(), cfg.E, num_chunks=N)
        torch.cuda.synchronize()
        results[rank] = out.view(torch.int16).cpu().numpy().tobytes()
        grp.close()
        del grp
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,N", [("tiny", 2), ("edge", 3)])
def test_ep_two_processes_with_ipc_peer_buffers(moe, name, N):
    """Two ranks as two processes on one GPU: dispatch stores into, and combine loads from,
    the other process's receive buffer through its CUDA IPC mapping."""
    cfg = CONFIGS[name]
    cpu = layer_inputs(cfg)
    gpu = {k: v.cuda() for k, v in cpu.items()}
    ref = moe.forward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"], gpu["wd"], num_chunks=N)
    torch.cuda.synchronize()
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_ipc_rank, args=(world, _free_port(), name, N, results),
                           nprocs=world, join=True, start_method="spawn")
        res = dict(results)
    parts = np.array_split(np.arange(cfg.T), world)
    for r in range(world):
        got = torch.from_numpy(np.frombuffer(res[r], np.int16).copy()).view(torch.bfloat16)
        want = ref[torch.from_numpy(parts[r]).cuda()].cpu().reshape(-1)
        assert torch.equal(got, want), f"rank {r}"
