"""Expert parallelism over several GPUs, with the exchange fused into the row kernels.

Chunk MoE article ("昇腾MindSpeed分块专家计算Chunk MoE"), sections 一张专业时序图 (per chunk:
All-to-All dispatch, expert computation, All-to-All combine) and 操作指南
(expert_parallel_size).  W ranks, one process per GPU: rank d holds the weights of experts
[d E/W, (d+1) E/W) and routes its own tokens.  Per chunk:

  1. the chunk's expert counts of every rank are all-gathered (W x E integers);
  2. moe_ep_plan gives each rank the row offset of its copies in every receive buffer;
  3. moe_ep_dispatch stores each token copy straight into its row of the owning rank's
     receive buffer (peer stores over NVLink, CUDA IPC mappings);
  4. every rank runs its grouped GEMMs (gate/up + SwiGLU, down) on the rows it received,
     writing the expert outputs over them;
  5. moe_ep_combine loads each token's k expert outputs back from their ranks (peer loads)
     and forms the weighted sum in fp32, ascending j.

The results equal moe_forward over all ranks' tokens with all experts, bit for bit.  The
phases are ordered across ranks by host barriers (device synchronize + a process-group
barrier).  This module only orchestrates: every row and every GEMM runs in libmoe.so.
"""
import numpy as np
import torch

from . import (_ptr_table, ep_combine, ep_dispatch, ep_plan, grouped_down,
               grouped_gateup, ipc_close, ipc_handle, ipc_open, metadata)


def _chunk_meta(idx, E, W, num_chunks):
    meta = metadata(idx, E, W, num_chunks, with_permutation=True)
    return meta


def _check_capacity(counts_all, cap):
    """Every rank's received rows of this chunk fit its receive buffer (checked on every
    rank from the all-gathered counts, before anything is stored into a peer)."""
    W, E = counts_all.shape
    per_dest = counts_all.reshape(W, W, E // W).sum(axis=(0, 2))
    if int(per_dest.max(initial=0)) > cap:
        raise ValueError(f"a rank receives {int(per_dest.max())} rows of this chunk, more than "
                         f"its receive buffer's {cap}")


def _experts(recv, act, offs, W_gate_up_local, W_down_local, stream=None):
    """Grouped GEMMs of one rank on its received rows; Y overwrites the rows in place."""
    rows = int(offs[-1])
    if rows == 0:
        return
    counts = np.diff(offs).astype(np.int32)
    offs_dev = torch.from_numpy(np.ascontiguousarray(offs, dtype=np.int32)).to(recv.device)
    grouped_gateup(recv[:rows], offs_dev, counts, W_gate_up_local, Act=act[:rows], stream=stream)
    grouped_down(act[:rows], offs_dev, counts, W_down_local, Y=recv[:rows], stream=stream)


def forward_emulated(hiddens, idxs, weights, W_gate_up, W_down, num_chunks=1):
    """All W ranks in one process on one GPU (receive buffers are plain local tensors, every
    launch on the current stream, so no kernel waits for another).  hiddens / idxs /
    weights: per-rank lists; W_gate_up / W_down: all E experts (rank d uses its slice).
    Returns the per-rank outputs."""
    W = len(hiddens)
    E, twoI, H = W_gate_up.shape
    I = twoI // 2
    El = E // W
    k = idxs[0].shape[1]
    dev = hiddens[0].device
    metas = [_chunk_meta(idxs[r], E, W, num_chunks) for r in range(W)]
    n = metas[0]["counts"].shape[0]
    t_chunk = max(int(np.diff(m["bounds"]).max()) if m["bounds"].size > 1 else 0 for m in metas)
    cap = max(1, W * t_chunk * k)
    recv = [torch.empty((cap, H), dtype=torch.bfloat16, device=dev) for _ in range(W)]
    act = [torch.empty((cap, I), dtype=torch.bfloat16, device=dev) for _ in range(W)]
    table = _ptr_table([x.data_ptr() for x in recv], dev)
    outs = [torch.empty_like(h) for h in hiddens]
    for c in range(n):
        counts_all = np.stack([m["counts"][c] for m in metas])
        _check_capacity(counts_all, cap)
        plans = [ep_plan(counts_all, r) for r in range(W)]
        deltas = [torch.from_numpy(p[0]).to(dev) for p in plans]
        for s in range(W):
            b0, b1 = int(metas[s]["bounds"][c]), int(metas[s]["bounds"][c + 1])
            if b1 > b0:
                ep_dispatch(hiddens[s][b0:b1], idxs[s][b0:b1], metas[s]["dst"][b0 * k:b1 * k],
                            deltas[s], table, E, W, cap)
        for d in range(W):
            _experts(recv[d], act[d], plans[d][1], W_gate_up[d * El:(d + 1) * El],
                     W_down[d * El:(d + 1) * El])
        for s in range(W):
            b0, b1 = int(metas[s]["bounds"][c]), int(metas[s]["bounds"][c + 1])
            if b1 > b0:
                ep_combine(table, idxs[s][b0:b1], metas[s]["dst"][b0 * k:b1 * k], deltas[s],
                           weights[s][b0:b1], H, E, W, cap, out=outs[s][b0:b1])
    return outs


class EPGroup:
    """One rank of an expert-parallel layer.  `dist` is an initialised torch.distributed
    (any backend: the collectives here are an all-gather of small host integer arrays,
    an all-gather of IPC handles and barriers).  The receive buffers hold rows_cap rows
    (at most W * T_chunk * k per chunk)."""

    def __init__(self, dist, rows_cap: int, H: int, I: int, device):
        self.dist = dist
        self.rank, self.W = dist.get_rank(), dist.get_world_size()
        self.cap, self.H, self.I, self.device = int(rows_cap), H, I, device
        self.recv = torch.empty((self.cap, H), dtype=torch.bfloat16, device=device)
        self.act = torch.empty((self.cap, I), dtype=torch.bfloat16, device=device)
        torch.cuda.synchronize(device)
        handles = [None] * self.W
        dist.all_gather_object(handles, ipc_handle(self.recv))
        self.peers = {}
        ptrs = []
        for r, (h, off) in enumerate(handles):
            if r == self.rank:
                ptrs.append(self.recv.data_ptr())
            else:
                p = ipc_open(h, off)
                self.peers[r] = (p, off)
                ptrs.append(p)
        self.table = _ptr_table(ptrs, device)

    def _barrier(self):
        torch.cuda.synchronize(self.device)
        self.dist.barrier()

    def _all_counts(self, counts):
        rows = [None] * self.W
        self.dist.all_gather_object(rows, np.asarray(counts, np.int32).tolist())
        return np.asarray(rows, np.int32)

    def forward(self, hidden, idx, w, W_gate_up_local, W_down_local, E: int, num_chunks=1):
        """This rank's tokens through the layer; W_*_local hold this rank's E/W experts."""
        k = idx.shape[1]
        meta = _chunk_meta(idx, E, self.W, num_chunks)
        out = torch.empty_like(hidden)
        for c in range(meta["counts"].shape[0]):
            counts_all = self._all_counts(meta["counts"][c])
            _check_capacity(counts_all, self.cap)
            delta, offs = ep_plan(counts_all, self.rank)
            delta_dev = torch.from_numpy(delta).to(self.device)
            b0, b1 = int(meta["bounds"][c]), int(meta["bounds"][c + 1])
            if b1 > b0:
                ep_dispatch(hidden[b0:b1], idx[b0:b1], meta["dst"][b0 * k:b1 * k], delta_dev,
                            self.table, E, self.W, self.cap)
            self._barrier()  # every rank's rows have arrived
            _experts(self.recv, self.act, offs, W_gate_up_local, W_down_local)
            self._barrier()  # every rank's expert outputs are written
            if b1 > b0:
                ep_combine(self.table, idx[b0:b1], meta["dst"][b0 * k:b1 * k], delta_dev,
                           w[b0:b1], self.H, E, self.W, self.cap, out=out[b0:b1])
            self._barrier()  # the receive buffers may be reused
        return out

    def close(self):
        """Unmap the peers' buffers (every rank, before any rank frees its own)."""
        for p, off in self.peers.values():
            ipc_close(p, off)
        self.peers = {}
        self._barrier()


def chunk_plan_rows(counts_all, rank: int, dst_rows, idx, E: int):
    """Host restatement for tests: the receive (rank, row) of every copy of one chunk from
    the plan, as two int arrays."""
    W = counts_all.shape[0]
    delta, _ = ep_plan(counts_all, rank)
    e = np.asarray(idx).reshape(-1)
    return e // (E // W), np.asarray(dst_rows).reshape(-1) + delta[e]


__all__ = ["forward_emulated", "EPGroup", "chunk_plan_rows"]
