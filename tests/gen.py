"""Seeded synthetic inputs for the MoE layer tests and the benchmark.

This module only draws inputs: hidden states, expert weights and a router's output
(top_k_index, top_k_weights).  It holds none of the MoE layer's own arithmetic, and both
the CUDA path and the CPU oracle receive exactly the tensors it returns.

Recipes (all seeded; every tensor gets its own derived seed):
  hidden            bf16 N(0, 1)
  W_gate_up [E,2I,H] bf16 N(0, std = 1/sqrt(H));  W_down [E,H,I] bf16 N(0, std = 1/sqrt(I))
                    (drawn expert by expert, so one expert can be redrawn alone)
  routing "normal"  logits fp32 N(0,1)
          "bias"    logits N(0,1) + a per-expert bias N(0, std=0.5)
          "zipf"    logits[t,e] = -s*ln(rank_e) + Gumbel(0,1), rank = seeded permutation
                    of 1..E; optionally the n_masked least popular experts set to -inf
                    (top-k of Gumbel-perturbed log-probabilities samples k experts without
                    replacement with probability proportional to rank^-s)
          "pair01"  every slot drawn uniformly from {0, 1} (duplicates in a row on purpose),
                    weights a softmax of N(0,1) scores over the k slots
  top_k_index = the k largest logits per row (ties to the lower expert id);
  top_k_weights = softmax of the row's logits restricted to those k, in fp32 (the
  softmax over all experts renormalised over the chosen k).
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np
import torch


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    routing: str
    G: int = 1
    chunks: Tuple[int, ...] = (1,)
    zipf_s: float = 0.0
    n_masked: int = 0
    bias_std: float = 0.0
    note: str = ""


CONFIGS = {
    "tiny": LayerConfig("tiny", 512, 256, 8, 2, 512, "normal", chunks=(1, 2),
                        note="tiny MoE layer"),
    "edge": LayerConfig("edge", 1000, 1024, 64, 6, 1408, "zipf", chunks=(8, 7, 3),
                        zipf_s=1.5, n_masked=20,
                        note="edge-case layer, Zipf(1.5) with 20 experts never chosen"),
    "edge_pair01": LayerConfig("edge_pair01", 1000, 1024, 64, 6, 1408, "pair01", chunks=(8,),
                               note="every slot routed to expert 0 or 1"),
    "edge_varlen": LayerConfig("edge_varlen", 49, 1024, 64, 6, 1408, "normal", chunks=(8,),
                               note="T=49 at N=8: seven chunks of 7 and one empty chunk"),
    "edge_varlen7": LayerConfig("edge_varlen7", 7, 1024, 64, 6, 1408, "normal", chunks=(8,),
                                note="T=7 at N=8: one chunk of 1 token per chunk, one empty"),
    "mixtral": LayerConfig("mixtral", 4096, 4096, 8, 2, 14336, "normal", chunks=(1, 2, 4),
                           note="Mixtral-8x7B-shaped layer"),
    "qwen3": LayerConfig("qwen3", 16384, 2048, 128, 8, 768, "bias", chunks=(1, 2, 4),
                         bias_std=0.5,
                         note="Qwen3-30B-A3B-shaped layer over one 16k packed sequence"),
    "deepseek": LayerConfig("deepseek", 8192, 7168, 256, 8, 2048, "zipf", G=16, chunks=(1, 4),
                            zipf_s=1.1, note="DeepSeek-V3-shaped routed-expert layer, 16 groups"),
}

_TAG = {"hidden": 1, "wgu": 2, "wd": 3, "route": 4, "bias": 5, "rank": 6}


def _seed(seed: int, tag: str, sub: int = 0) -> int:
    return (int(seed) * 1_000_003 + _TAG[tag] * 65_537 + int(sub)) % (2**63 - 1)


def bf16_normal(shape, std: float, seed: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def hidden(T: int, H: int, seed: int = 0) -> torch.Tensor:
    return bf16_normal((T, H), 1.0, _seed(seed, "hidden"))


def expert_gate_up(e: int, H: int, I: int, seed: int = 0) -> torch.Tensor:
    return bf16_normal((2 * I, H), 1.0 / np.sqrt(H), _seed(seed, "wgu", e))


def expert_down(e: int, H: int, I: int, seed: int = 0) -> torch.Tensor:
    return bf16_normal((H, I), 1.0 / np.sqrt(I), _seed(seed, "wd", e))


def expert_weights(E: int, H: int, I: int, seed: int = 0, experts=None, device=None):
    """(W_gate_up [E,2I,H], W_down [E,H,I]) bf16; `experts` limits which are drawn
    (the others stay zero); `device` places the full tensors there, expert by expert."""
    wgu = torch.zeros((E, 2 * I, H), dtype=torch.bfloat16, device=device)
    wd = torch.zeros((E, H, I), dtype=torch.bfloat16, device=device)
    for e in (range(E) if experts is None else experts):
        wgu[e].copy_(expert_gate_up(e, H, I, seed))
        wd[e].copy_(expert_down(e, H, I, seed))
    return wgu, wd


def _topk_softmax(logits: np.ndarray, k: int):
    order = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(logits, order, axis=1).astype(np.float64)
    sel = sel - sel.max(axis=1, keepdims=True)
    p = np.exp(sel)
    p /= p.sum(axis=1, keepdims=True)
    return order.astype(np.int32), p.astype(np.float32)


def routing(cfg: LayerConfig, seed: int = 0, T: Optional[int] = None):
    """(top_k_index int32 [T,k], top_k_weights fp32 [T,k]) as numpy arrays."""
    T = cfg.T if T is None else T
    E, k = cfg.E, cfg.k
    rng = np.random.default_rng(_seed(seed, "route"))
    if cfg.routing == "pair01":
        idx = rng.integers(0, 2, size=(T, k), dtype=np.int64).astype(np.int32)
        scores = rng.standard_normal((T, k)).astype(np.float32)
        _, w = _topk_softmax(scores, k)  # softmax over the k slot scores
        return idx, w
    logits = rng.standard_normal((T, E), dtype=np.float32)
    if cfg.routing == "bias":
        b = np.random.default_rng(_seed(seed, "bias")).standard_normal(E).astype(np.float32)
        logits = logits + np.float32(cfg.bias_std) * b[None, :]
    elif cfg.routing == "zipf":
        rank = np.random.default_rng(_seed(seed, "rank")).permutation(E) + 1
        gumbel = -np.log(-np.log(rng.uniform(1e-12, 1.0, size=(T, E))))
        logits = (-cfg.zipf_s * np.log(rank)[None, :] + gumbel).astype(np.float32)
        if cfg.n_masked:
            logits[:, rank > E - cfg.n_masked] = -np.inf
    elif cfg.routing != "normal":
        raise ValueError(cfg.routing)
    return _topk_softmax(logits, k)


def layer_inputs(cfg: LayerConfig, seed: int = 0, device=None, weights: bool = True):
    """Everything one forward call needs, as torch tensors on `device` (CPU if None)."""
    idx, w = routing(cfg, seed)
    x = hidden(cfg.T, cfg.H, seed)
    out = dict(hidden=x.to(device), idx=torch.from_numpy(idx).to(device),
               w=torch.from_numpy(w).to(device))
    if weights:
        out["wgu"], out["wd"] = expert_weights(cfg.E, cfg.H, cfg.I, seed, device=device)
    return out


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 view of a bf16 tensor's bits (CPU numpy), the oracle's bf16 format."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
