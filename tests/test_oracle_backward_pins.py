"""Pins of the oracle's backward pass (no GPU).

The oracle's gradients are checked against: fp64 reverse-mode autodiff of the forward
definition in torch on the CPU (an independent derivation of all four gradients), exact
finite differences in the routing weights (the output is linear in them), and the closed
form of identity-like experts."""
import numpy as np
import pytest
import torch

import oracle
from test_oracle_pins import _bf16_round, _bits


def _case(seed, T=7, H=16, I=24, E=3, k=2):
    rng = np.random.default_rng(seed)
    x = _bf16_round(rng.standard_normal((T, H)))
    wgu = _bf16_round(rng.standard_normal((E, 2 * I, H)) / 3)
    wd = _bf16_round(rng.standard_normal((E, H, I)) / 4)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    idx[0, :] = 1  # a duplicated expert in one row
    w = rng.uniform(0.1, 1.0, size=(T, k)).astype(np.float32)
    dout = _bf16_round(rng.standard_normal((T, H)))
    return x, wgu, wd, idx, w, dout


def _torch_grads(x, wgu, wd, idx, w, dout):
    """Reverse-mode autodiff of sum(out * dout) through the plain forward definition."""
    X = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    Wgu = torch.tensor(wgu, dtype=torch.float64, requires_grad=True)
    Wd = torch.tensor(wd, dtype=torch.float64, requires_grad=True)
    Wt = torch.tensor(w, dtype=torch.float64, requires_grad=True)
    T, k = idx.shape
    I = wgu.shape[1] // 2
    rows = []
    for t in range(T):
        acc = 0
        for j in range(k):
            e = int(idx[t, j])
            g = Wgu[e, :I] @ X[t]
            u = Wgu[e, I:] @ X[t]
            acc = acc + Wt[t, j] * (Wd[e] @ (torch.nn.functional.silu(g) * u))
        rows.append(acc)
    out = torch.stack(rows)
    (out * torch.tensor(dout, dtype=torch.float64)).sum().backward()
    return X.grad.numpy(), Wt.grad.numpy(), Wgu.grad.numpy(), Wd.grad.numpy()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_backward_matches_fp64_autodiff(seed):
    x, wgu, wd, idx, w, dout = _case(seed)
    dx, dw, dwgu, dwd = oracle.backward(_bits(x), idx, w, _bits(wgu), _bits(wd), _bits(dout))
    rx, rw, rgu, rd = _torch_grads(x, wgu, wd, idx, w, dout)
    np.testing.assert_allclose(dx, rx, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dw, rw, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dwgu, rgu, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dwd, rd, rtol=1e-11, atol=1e-12)


def test_weight_gradient_is_the_exact_derivative():
    """out is linear in top_k_weights: d/dw sum(out*dout) = <dout, FFN_e(x)> exactly, and a
    central difference of the oracle's own forward reproduces it."""
    x, wgu, wd, idx, w, dout = _case(5)
    _, dw, _, _ = oracle.backward(_bits(x), idx, w, _bits(wgu), _bits(wd), _bits(dout))
    for t, j in [(0, 0), (0, 1), (3, 1), (6, 0)]:
        h = np.float32(2.0 ** -4)
        wp, wm = w.copy(), w.copy()
        wp[t, j] += h
        wm[t, j] -= h
        fp = oracle.forward(_bits(x), idx, wp, _bits(wgu), _bits(wd))
        fm = oracle.forward(_bits(x), idx, wm, _bits(wgu), _bits(wd))
        step = float(wp[t, j]) - float(wm[t, j])  # the fp32 perturbation actually applied
        fd = ((fp - fm) * dout).sum() / step
        assert dw[t, j] == pytest.approx(fd, rel=1e-12, abs=1e-12)


def test_identity_like_experts_input_gradient_closed_form():
    """W_gate = a [I_H; 0], W_up = b [I_H; 0], W_down = al [I_H 0] give
    out = sum_j w_j al b x silu(a x), hence
    d_x = dout * sum_j w_j al b (silu(a x) + a x silu'(a x)),
    silu'(z) = sig(z) (1 + z (1 - sig(z)))."""
    rng = np.random.default_rng(8)
    T, H, I, E, k = 10, 8, 16, 3, 2
    a = np.array([1.0, 2.0, 0.5])
    b = np.array([0.5, 1.0, 2.0])
    al = np.array([1.0, 0.25, 0.5])
    eye = np.eye(H, dtype=np.float32)
    pad = np.zeros((I - H, H), np.float32)
    wgu = np.stack([np.concatenate([a[e] * eye, pad, b[e] * eye, pad]) for e in range(E)])
    wd = np.stack([np.concatenate([al[e] * eye, np.zeros((H, I - H), np.float32)], axis=1)
                   for e in range(E)])
    x = _bf16_round(rng.standard_normal((T, H)))
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    w = rng.uniform(0.2, 1.0, size=(T, k)).astype(np.float32)
    dout = _bf16_round(rng.standard_normal((T, H)))
    dx, _, _, _ = oracle.backward(_bits(x), idx, w, _bits(wgu.astype(np.float32)),
                                  _bits(wd.astype(np.float32)), _bits(dout))
    xd = x.astype(np.float64)
    ref = np.zeros_like(xd)
    for j in range(k):
        e = idx[:, j]
        z = a[e][:, None] * xd
        sig = 1 / (1 + np.exp(-z))
        d = z * sig + z * sig * (1 + z * (1 - sig))  # silu(z) + z silu'(z)
        ref += (w[:, j].astype(np.float64) * al[e] * b[e])[:, None] * d
    np.testing.assert_allclose(dx, ref * dout, rtol=1e-12, atol=1e-14)
