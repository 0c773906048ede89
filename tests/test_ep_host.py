"""Expert parallelism without a GPU: the row plan (moe_ep_plan, host arithmetic) against a
hand-worked example, and, across two gloo ranks on the CPU, against the properties that fix
the receive layout: every destination's rows are filled exactly once, each local expert's
rows are contiguous, and inside an expert the source ranks come in ascending order with
each source's copies in its own stable (t, j) order."""
import json
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import expert_router_top_b200 as moe
import oracle
from gen import CONFIGS, routing

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ep_plan_small.json")


def test_plan_hand_worked():
    g = json.load(open(GOLDEN))
    counts = np.array(g["counts_all"], np.int32)
    for r in range(g["W"]):
        delta, offs = moe.ep_plan(counts, r)
        assert delta.tolist() == g["send_delta"][r]
        assert offs.tolist() == g["recv_offsets"][r]


def test_plan_argument_checks():
    with pytest.raises(moe.MoEError):
        moe.ep_plan(np.zeros((2, 3), np.int32), 0)      # E % W != 0
    with pytest.raises(moe.MoEError):
        moe.ep_plan(np.zeros((2, 4), np.int32), 2)      # rank outside [0, W)
    with pytest.raises(moe.MoEError):
        moe.ep_plan(-np.ones((2, 4), np.int32), 0)      # negative count


def _check_layout(counts_all, per_source, E):
    """per_source[s] = (idx [Tc,k], dst [Tc*k]) of source s for one chunk."""
    W = counts_all.shape[0]
    El = E // W
    plans = [moe.ep_plan(counts_all, r) for r in range(W)]
    filled = [dict() for _ in range(W)]
    for s, (idx, dst) in enumerate(per_source):
        delta = plans[s][0]
        e = idx.reshape(-1)
        rank = e // El
        row = dst.reshape(-1) + delta[e]
        for n in range(e.size):
            d = int(rank[n])
            assert int(row[n]) not in filled[d], "two copies land on one receive row"
            filled[d][int(row[n])] = (int(e[n]), s, n)
    for d in range(W):
        offs = plans[d][1]
        assert sorted(filled[d]) == list(range(int(offs[-1]))), "receive rows not a bijection"
        seq = [filled[d][r] for r in range(int(offs[-1]))]
        for el in range(El):
            block = seq[offs[el]:offs[el + 1]]
            assert all(x[0] == d * El + el for x in block), "expert rows not contiguous"
            assert block == sorted(block, key=lambda x: (x[1], x[2])), \
                "sources ascending, each in (t, j) order"


@pytest.mark.parametrize("W,name,N", [(2, "tiny", 1), (4, "tiny", 3), (8, "edge", 2),
                                      (2, "edge_pair01", 2)])
def test_plan_layout_properties(W, name, N):
    """W sources, each with its own tokens (a slice of the configuration's routing), the
    oracle's chunk-local expert-major rows, one plan per chunk."""
    cfg = CONFIGS[name]
    idx_all = routing(cfg)[0]
    parts = np.array_split(np.arange(cfg.T), W)
    metas = [oracle.metadata(idx_all[p], cfg.E, W, N) for p in parts]
    bounds = [oracle.chunk_bounds(len(p), N) for p in parts]
    for c in range(N):
        counts_all = np.stack([m["counts"][c] for m in metas]).astype(np.int32)
        per_source = []
        for s, p in enumerate(parts):
            b0, b1 = bounds[s][c], bounds[s][c + 1]
            per_source.append((idx_all[p][b0:b1], metas[s]["dst"][b0 * cfg.k:b1 * cfg.k]))
        _check_layout(counts_all, per_source, cfg.E)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cfg = CONFIGS["edge"]
        idx_all = routing(cfg)[0]
        mine = np.array_split(np.arange(cfg.T), world)[rank]
        meta = oracle.metadata(idx_all[mine], cfg.E, world, 2)
        b = oracle.chunk_bounds(len(mine), 2)
        out = []
        for c in range(2):
            rows = [None] * world
            dist.all_gather_object(rows, meta["counts"][c].astype(np.int32).tolist())
            counts_all = np.asarray(rows, np.int32)
            delta, offs = moe.ep_plan(counts_all, rank)
            out.append((counts_all.tolist(), delta.tolist(), offs.tolist(),
                        idx_all[mine][b[c]:b[c + 1]].tolist(),
                        meta["dst"][b[c] * cfg.k:b[c + 1] * cfg.k].tolist()))
        results[rank] = out
    finally:
        dist.destroy_process_group()


def test_plan_across_gloo_ranks():
    """Two processes, each with its own tokens: the counts all-gather and each rank's own
    plan give a receive layout that is consistent across the ranks."""
    world = 2
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), results), nprocs=world, join=True)
        res = dict(results)
    cfg = CONFIGS["edge"]
    for c in range(2):
        counts = [np.asarray(res[r][c][0], np.int32) for r in range(world)]
        assert all(np.array_equal(counts[0], x) for x in counts), "ranks disagree on counts"
        per_source = [(np.asarray(res[r][c][3], np.int32), np.asarray(res[r][c][4], np.int32))
                      for r in range(world)]
        _check_layout(counts[0], per_source, cfg.E)
        for r in range(world):
            d, o = moe.ep_plan(counts[0], r)
            assert d.tolist() == res[r][c][1] and o.tolist() == res[r][c][2]
