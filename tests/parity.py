"""Comparison helpers for the GPU parity tests.

Tolerances:
  * end-to-end forward (bf16 output vs the fp64 oracle on the same bf16 inputs):
    relative Frobenius error <= 1e-2 and, per element, |err| <= 3e-2 + 2e-2 * |ref|
    (the layer's stated bar);
  * a single GEMM stage (bf16 output of an fp32-accumulated product vs fp64): the output
    rounding alone is <= 2^-9 |ref|; fp32 accumulation over K <= 8192 terms adds well
    under 1e-4 of the row scale.  Bar: |err| <= 2^-7 |ref| + 1e-3 * rms(ref), and
    relative Frobenius <= 4e-3;
  * unpermute (fp32 sum of k bf16 rows, one bf16 rounding): |err| <= 2^-8 |ref| +
    1e-5 * rms(ref).
"""
import numpy as np
import torch


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_frobenius(got: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def assert_layer_close(got, ref, what=""):
    got = got if isinstance(got, np.ndarray) else to_f64(got)
    err = np.abs(got - ref)
    bound = 3e-2 + 2e-2 * np.abs(ref)
    worst = float((err / bound).max()) if err.size else 0.0
    fro = rel_frobenius(got, ref)
    assert fro <= 1e-2, f"{what}: relative Frobenius error {fro:.3e} > 1e-2"
    assert worst <= 1.0, f"{what}: elementwise bound exceeded (worst err/bound = {worst:.3f})"
    return dict(rel_fro=fro, worst_frac_of_bound=worst)


def assert_gemm_close(got, ref, what=""):
    got = got if isinstance(got, np.ndarray) else to_f64(got)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    err = np.abs(got - ref)
    bound = 2.0 ** -7 * np.abs(ref) + 1e-3 * rms
    worst = float((err / np.maximum(bound, 1e-30)).max()) if err.size else 0.0
    fro = rel_frobenius(got, ref)
    assert fro <= 4e-3, f"{what}: relative Frobenius error {fro:.3e} > 4e-3"
    assert worst <= 1.0, f"{what}: elementwise GEMM bound exceeded (worst {worst:.3f})"
    return dict(rel_fro=fro, worst_frac_of_bound=worst)


def assert_unpermute_close(got, ref, what=""):
    got = got if isinstance(got, np.ndarray) else to_f64(got)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * rms
    worst = float((err / np.maximum(bound, 1e-30)).max()) if err.size else 0.0
    assert worst <= 1.0, f"{what}: unpermute bound exceeded (worst {worst:.3f})"
    return dict(worst_frac_of_bound=worst)
