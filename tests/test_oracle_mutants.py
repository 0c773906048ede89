"""The pins must catch plausible mistakes in the oracle.

Each case copies oracle.c, plants one mistake (a textual replacement), builds the copy
with gcc into a temporary library, points the oracle wrappers at it and runs the pin
tests of test_oracle_pins.py: at least one pin must fail for every planted mistake.
Nothing here touches the CUDA library or a GPU."""
import os
import subprocess
import tempfile

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.abspath(oracle.__file__)), "oracle.c")

# (name, text in oracle.c, replacement)
MUTANTS = [
    ("silu sign", "return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    ("silu without z", "return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));"),
    ("gate and up swapped",
     "const uint16_t* wg = wgu_e + (int64_t)i * H;\n    const uint16_t* wu = wgu_e + (int64_t)(I + i) * H;",
     "const uint16_t* wu = wgu_e + (int64_t)i * H;\n    const uint16_t* wg = wgu_e + (int64_t)(I + i) * H;"),
    ("up projection dropped", "h[i] = silu(g) * u;", "h[i] = silu(g);"),
    ("down operand transposed", "const uint16_t* w = wd_e + (int64_t)o * I;\n    double acc = 0.0;\n    for (int32_t i = 0; i < I; ++i) acc += bf16_to_f64(w[i]) * h[i];",
     "double acc = 0.0;\n    for (int32_t i = 0; i < I; ++i) acc += bf16_to_f64(wd_e[(int64_t)i * H + o]) * h[i];"),
    ("routing weight dropped", "for (int32_t c = 0; c < H; ++c) acc[c] += wt * y[c];",
     "for (int32_t c = 0; c < H; ++c) acc[c] += y[c];"),
    ("only the first choice",
     "for (int32_t j = 0; j < k; ++j) {\n      int32_t e = idx[t * k + j];\n      if (e < 0 || e >= E) {",
     "for (int32_t j = 0; j < 1; ++j) {\n      int32_t e = idx[t * k + j];\n      if (e < 0 || e >= E) {"),
    ("chunk size floor(T/N)", "int64_t t_chunk = (T + n - 1) / n;", "int64_t t_chunk = T / n + (T % n > 1);"),
    ("resolved chunk size floor(T/N)", "*t_chunk_out = (T + num_chunks - 1) / num_chunks;",
     "*t_chunk_out = T / num_chunks + (T % num_chunks > 1);"),
    ("chunk size wins over chunk count", "  if (num_chunks > 0) {\n    *n_out = num_chunks;",
     "  if (num_chunks > 0 && chunk_size == 0) {\n    *n_out = num_chunks;"),
    ("chunk size split evenly", "*t_chunk_out = chunk_size;\n    return 0;",
     "*t_chunk_out = (T + *n_out - 1) / *n_out;\n    return 0;"),
    ("N=0 read as 0 chunks", "return num_chunks <= 0 ? 1 : num_chunks;", "return num_chunks < 0 ? 1 : (num_chunks ? num_chunks : 2);"),
    ("copies of an expert in reverse order", "for (int64_t t = t0; t < t1; ++t) {\n        for (int32_t j = 0; j < k; ++j) {\n          if (idx[t * k + j] != e) continue;",
     "for (int64_t t = t1 - 1; t >= t0; --t) {\n        for (int32_t j = 0; j < k; ++j) {\n          if (idx[t * k + j] != e) continue;"),
    ("experts in descending order", "for (int32_t e = 0; e < E; ++e) {\n      int32_t start = row;",
     "for (int32_t e = E - 1; e >= 0; --e) {\n      int32_t start = row;"),
    ("group of an expert by modulo", "if (idx[t * k + j] / per_group == g) ++rows_g;", "if (idx[t * k + j] % G == g) ++rows_g;"),
    ("unpermute weight dropped", "double wt = (double)w[t * k + j];\n      for (int32_t c = 0; c < H; ++c) o[c] += wt * bf16_to_f64(y[c]);",
     "double wt = 1.0;\n      for (int32_t c = 0; c < H; ++c) o[c] += wt * bf16_to_f64(y[c]);"),
]

BACKWARD_MUTANTS = [
    ("dW_gate: sigmoid derivative sign", "double dg = dh[i] * u[i] * (sig + g[i] * sig * (1.0 - sig));",
     "double dg = dh[i] * u[i] * (sig - g[i] * sig * (1.0 - sig));"),
    ("dW_up: silu dropped", "double du = dh[i] * g[i] * sig;", "double du = dh[i] * sig;"),
    ("dW_down: routing weight dropped",
     "for (int32_t o = 0; o < H; ++o) dy[o] = wt * bf16_to_f64(dout[t * H + o]);\n        for (int32_t i = 0; i < I; ++i) {\n          double a = 0.0;",
     "for (int32_t o = 0; o < H; ++o) dy[o] = bf16_to_f64(dout[t * H + o]);\n        for (int32_t i = 0; i < I; ++i) {\n          double a = 0.0;"),
    ("d_x: up path dropped", "out[c] += bf16_to_f64(wg[(int64_t)i * H + c]) * dg + bf16_to_f64(wu[(int64_t)i * H + c]) * du;",
     "out[c] += bf16_to_f64(wg[(int64_t)i * H + c]) * dg;"),
    ("d_w: dot with dy", "for (int32_t o = 0; o < H; ++o) dot += bf16_to_f64(dout[t * H + o]) * y[o];",
     "for (int32_t o = 0; o < H; ++o) dot += bf16_to_f64(dout[t * H + o]) * y[o] * w[t * k + j];"),
]

PIN_TESTS = [
    pins.test_chunk_bounds_golden,
    pins.test_chunk_settings_golden,
    pins.test_metadata_golden,
    lambda: pins.test_metadata_bruteforce(3, 2, 3),
    lambda: pins.test_metadata_bruteforce(2, 2, 4),
    pins.test_metadata_larger_random,
    pins.test_silu_textbook_values_through_identity_expert,
    pins.test_identity_like_experts_closed_form,
    pins.test_ffn_matches_numpy_matmul,
    pins.test_equal_experts_return_the_dense_ffn,
    pins.test_combine_is_linear_in_weights,
    pins.test_worked_example_by_hand,
    pins.test_permute_then_unpermute_restores_tokens,
    pins.test_stage_gemms_match_numpy,
]


def _build(text, where):
    path = os.path.join(where, "oracle_mutant.c")
    with open(path, "w") as f:
        f.write(text)
    lib = os.path.join(where, "liboracle_mutant.so")
    subprocess.run(["gcc", "-std=c11", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", lib, path,
                    "-lm"], check=True)
    return lib


def test_unmutated_copy_passes_every_pin():
    with tempfile.TemporaryDirectory() as d:
        oracle.use_library(_build(open(SRC).read(), d))
        try:
            for t in PIN_TESTS:
                t()
        finally:
            oracle.use_library(None)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for '{name}' not found exactly once"
    with tempfile.TemporaryDirectory() as d:
        oracle.use_library(_build(text.replace(old, new), d))
        caught = []
        try:
            for t in PIN_TESTS:
                try:
                    t()
                except (AssertionError, ValueError) as e:  # a pin failed
                    caught.append(e)
                    break
        finally:
            oracle.use_library(None)
    assert caught, f"no pin caught the planted mistake '{name}'"


@pytest.mark.parametrize("name,old,new", BACKWARD_MUTANTS, ids=[m[0] for m in BACKWARD_MUTANTS])
def test_backward_pins_catch_planted_mistake(name, old, new):
    import test_oracle_backward_pins as bpins
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for '{name}' not found exactly once"
    with tempfile.TemporaryDirectory() as d:
        oracle.use_library(_build(text.replace(old, new), d))
        caught = False
        try:
            for t in (lambda: bpins.test_backward_matches_fp64_autodiff(0),
                      bpins.test_weight_gradient_is_the_exact_derivative,
                      bpins.test_identity_like_experts_input_gradient_closed_form):
                try:
                    t()
                except AssertionError:
                    caught = True
                    break
        finally:
            oracle.use_library(None)
    assert caught, f"no backward pin caught the planted mistake '{name}'"
