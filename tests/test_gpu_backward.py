"""Backward pass (expert computation recomputed per chunk) against the fp64 oracle.

Tolerances: d_hidden is a bf16 output built from bf16 intermediates (the layer's bar:
relative Frobenius <= 1e-2, |err| <= 3e-2 + 2e-2 |ref|).  d_weights, dW_gate_up and dW_down
are fp32 sums of products of bf16-rounded intermediates: each term carries a relative error
of ~2^-8, and the terms of the weight gradients are heavy-tailed (dg = dh u silu'(g) is a
product of three roughly Gaussian factors), so an entry whose few terms cancel keeps an
absolute error of a few per cent of the gradient's RMS.  Bar: relative Frobenius <= 1e-2
and |err| <= 2e-2 |ref| + 1e-1 rms(ref)."""
import numpy as np
import pytest
import torch

import oracle
from gen import (CONFIGS, LayerConfig, bf16_normal, bits, expert_down, expert_gate_up,
                 expert_weights, hidden, layer_inputs, routing)
from parity import assert_layer_close, rel_frobenius, to_f64

pytestmark = pytest.mark.gpu


def assert_grad_close(got, ref, what):
    got = got if isinstance(got, np.ndarray) else to_f64(got)
    fro = rel_frobenius(got, ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    worst = float((np.abs(got - ref) / (2e-2 * np.abs(ref) + 1e-1 * rms + 1e-30)).max())
    assert fro <= 1e-2, f"{what}: relative Frobenius {fro:.3e}"
    assert worst <= 1.0, f"{what}: elementwise bound exceeded ({worst:.3f})"
    return fro


MID = LayerConfig("mid", 300, 512, 16, 4, 384, "normal", chunks=(1, 3))


def _run(moe, cfg, N=1, S=0):
    cpu = layer_inputs(cfg)
    dout = bf16_normal((cfg.T, cfg.H), 1.0, 99)
    gpu = {k: v.cuda() for k, v in cpu.items()}
    res = moe.backward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"], gpu["wd"], dout.cuda(),
                       num_chunks=N, ep_groups=cfg.G, chunk_size=S)
    torch.cuda.synchronize()
    return cpu, dout, res


@pytest.mark.parametrize("cfg", [CONFIGS["tiny"], MID, CONFIGS["edge_varlen"]],
                         ids=["tiny", "mid", "edge_varlen"])
def test_backward_matches_oracle(moe, cfg):
    cpu, dout, (dx, dw, dwgu, dwd) = _run(moe, cfg, N=cfg.chunks[-1])
    rx, rw, rgu, rd = oracle.backward(bits(cpu["hidden"]), cpu["idx"].numpy(), cpu["w"].numpy(),
                                      bits(cpu["wgu"]), bits(cpu["wd"]), bits(dout))
    stats = dict(d_hidden=assert_layer_close(dx, rx, f"{cfg.name} d_hidden")["rel_fro"],
                 d_weights=assert_grad_close(dw, rw, f"{cfg.name} d_weights"),
                 dW_gate_up=assert_grad_close(dwgu, rgu, f"{cfg.name} dW_gate_up"),
                 dW_down=assert_grad_close(dwd, rd, f"{cfg.name} dW_down"))
    print(cfg.name, {k: f"{v:.2e}" for k, v in stats.items()})


def test_backward_chunk_invariance(moe):
    cfg = MID
    _, _, base = _run(moe, cfg, N=1)
    for N, S in ((2, 0), (3, 0), (7, 0), (0, 64)):
        _, _, got = _run(moe, cfg, N=N, S=S)
        assert torch.equal(got[0], base[0]), f"d_hidden differs at N={N} S={S}"
        assert torch.equal(got[1], base[1]), f"d_weights differs at N={N} S={S}"
        for a, b, name in ((got[2], base[2], "dW_gate_up"), (got[3], base[3], "dW_down")):
            assert rel_frobenius(to_f64(a), to_f64(b)) < 1e-5, f"{name} at N={N} S={S}"


def test_backward_zero_tokens(moe):
    cfg = CONFIGS["tiny"]
    gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
    d = torch.zeros((0, cfg.H), dtype=torch.bfloat16, device="cuda")
    dx, dw, dwgu, dwd = moe.backward(gpu["hidden"][:0], gpu["idx"][:0], gpu["w"][:0], gpu["wgu"],
                                     gpu["wd"], d)
    torch.cuda.synchronize()
    assert dx.shape == (0, cfg.H) and not dwgu.any() and not dwd.any()


def test_backward_full_size_sampled(moe):
    """The Qwen3-shaped 16k layer at num_chunks=4, as the benchmark runs it: the weight
    gradients of two experts (the least-routed one with rows and one of median load), and
    d_hidden and d_weights of every token routed to them, against the oracle run on exactly
    those tokens (all k experts of each token included, so every compared value is whole)."""
    cfg = CONFIGS["qwen3"]
    idx, w = routing(cfg)
    x = hidden(cfg.T, cfg.H)
    dout = bf16_normal((cfg.T, cfg.H), 1.0, 99)
    wgu, wd = expert_weights(cfg.E, cfg.H, cfg.I, device="cuda")
    dx, dw, dwgu, dwd = moe.backward(x.cuda(), torch.from_numpy(idx).cuda(),
                                     torch.from_numpy(w).cuda(), wgu, wd, dout.cuda(),
                                     num_chunks=4)
    torch.cuda.synchronize()
    counts = np.bincount(idx.reshape(-1), minlength=cfg.E)
    live = np.flatnonzero(counts)
    e_small = int(live[np.argmin(counts[live])])
    e_mid = int(live[np.argsort(counts[live])[len(live) // 2]])
    toks = np.flatnonzero(((idx == e_small) | (idx == e_mid)).any(1))
    used = sorted(set(idx[toks].reshape(-1).tolist()))
    remap = {e: i for i, e in enumerate(used)}
    sub_idx = np.vectorize(remap.get)(idx[toks]).astype(np.int32)
    sub_wgu = np.stack([bits(expert_gate_up(e, cfg.H, cfg.I)) for e in used])
    sub_wd = np.stack([bits(expert_down(e, cfg.H, cfg.I)) for e in used])
    rx, rw, rgu, rd = oracle.backward(bits(x[torch.from_numpy(toks)]), sub_idx, w[toks], sub_wgu,
                                      sub_wd, bits(dout[torch.from_numpy(toks)]))
    t_d = torch.from_numpy(toks).cuda()
    assert_layer_close(dx[t_d], rx, "qwen3 N=4 d_hidden (sampled tokens)")
    assert_grad_close(dw[t_d], rw, "qwen3 N=4 d_weights (sampled tokens)")
    for e in (e_small, e_mid):
        assert_grad_close(dwgu[e], rgu[remap[e]], f"qwen3 N=4 dW_gate_up[{e}]")
        assert_grad_close(dwd[e], rd[remap[e]], f"qwen3 N=4 dW_down[{e}]")
    assert bool(torch.isfinite(dwgu).all()) and bool(torch.isfinite(dwd).all())
    assert bool(torch.isfinite(dx.float()).all())


@pytest.mark.parametrize("E,k,T,H,I", [(1024, 8, 1536, 128, 128),   # MOE_MAX_EXPERTS
                                       (64, 32, 600, 256, 192),     # MOE_MAX_TOPK
                                       (1, 1, 300, 64, 64),         # one expert, top-1
                                       (16, 4, 257, 192, 96)])      # I not a multiple of 64
def test_backward_limits_and_odd_shapes(moe, E, k, T, H, I):
    """The backward at the ABI's limits (the most experts, the largest top-k), with a single
    expert, and with widths that are not multiples of the 128/256 tile widths: every
    gradient against the oracle at three chunk counts (odd counts leave a pair with one
    chunk), d_hidden and d_weights bit-identical across them."""
    cfg = LayerConfig("bwd_limits", T, H, E, k, I, "normal")
    cpu = layer_inputs(cfg)
    dout = bf16_normal((T, H), 1.0, 99)
    gpu = {kk: v.cuda() for kk, v in cpu.items()}
    rx, rw, rgu, rd = oracle.backward(bits(cpu["hidden"]), cpu["idx"].numpy(), cpu["w"].numpy(),
                                      bits(cpu["wgu"]), bits(cpu["wd"]), bits(dout))
    base = None
    for N in (1, 3, 4):
        dx, dw, dwgu, dwd = moe.backward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"],
                                         gpu["wd"], dout.cuda(), num_chunks=N)
        torch.cuda.synchronize()
        tag = f"E={E} k={k} H={H} I={I} N={N}"
        assert_layer_close(dx, rx, f"{tag} d_hidden")
        assert_grad_close(dw, rw, f"{tag} d_weights")
        assert_grad_close(dwgu, rgu, f"{tag} dW_gate_up")
        assert_grad_close(dwd, rd, f"{tag} dW_down")
        if base is None:
            base = (dx, dw)
        else:
            assert torch.equal(dx, base[0]) and torch.equal(dw, base[1]), tag
