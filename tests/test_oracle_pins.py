"""Pins of the CPU oracle to facts outside itself (no GPU needed).

Each test ties the oracle to something it does not compute itself: hand-worked values
from the Chunk MoE article's definitions (tests/golden/), properties that determine the
permutation uniquely, exhaustive brute force on tiny inputs, closed forms of special
expert weights, textbook values of the logistic function, and numpy's matrix product.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------------
# chunk partition: T_chunk = ceil(T/N)  (Chunk MoE article, section 一组关键公式)

def test_chunk_bounds_golden():
    for case in _load("chunk_bounds.json")["cases"]:
        b = oracle.chunk_bounds(case["T"], case["N"])
        assert b.tolist() == case["bounds"], case
        if case["T"] > 0:
            assert b[1] - b[0] == case["T_chunk"]


def test_chunk_settings_golden():
    """moe_num_chunks / moe_chunk_size precedence (section 操作指南 step 3)."""
    for case in _load("chunk_settings.json")["cases"]:
        n, tc, warn = oracle.resolve_chunks(case["T"], case["num_chunks"], case["chunk_size"])
        assert (n, tc, warn) == (case["n"], case["t_chunk"], case["warn"]), case
        b = oracle.chunk_bounds_sized(case["T"], case["num_chunks"], case["chunk_size"])
        assert b.tolist() == case["bounds"], case
    with pytest.raises(ValueError):
        oracle.resolve_chunks(10, 0, -1)


def test_chunk_size_metadata_properties():
    """Metadata with a chunk size obeys the same unique-permutation properties per chunk."""
    rng = np.random.default_rng(4)
    idx = rng.integers(0, 16, size=(1000, 4)).astype(np.int32)
    for S in (1, 7, 143, 999, 1000, 5000):
        m = oracle.metadata(idx, 16, 4, 0, chunk_size=S)
        b = m["bounds"]
        assert b[0] == 0 and b[-1] == 1000 and (np.diff(b)[:-1] == min(S, 1000)).all()
        flat = idx.reshape(-1)
        for c in range(len(b) - 1):
            e_c = flat[b[c] * 4:b[c + 1] * 4]
            assert m["counts"][c].tolist() == np.bincount(e_c, minlength=16).tolist()
            d = m["dst"][b[c] * 4:b[c + 1] * 4]
            assert sorted(d.tolist()) == list(range(len(e_c)))


@pytest.mark.parametrize("T", [0, 1, 2, 7, 49, 100, 1000, 4097])
@pytest.mark.parametrize("N", [0, 1, 2, 3, 4, 7, 8, 16])
def test_chunk_bounds_properties(T, N):
    b = oracle.chunk_bounds(T, N)
    n = max(N, 1)
    sizes = np.diff(b)
    assert len(b) == n + 1 and b[0] == 0 and b[-1] == T
    assert (sizes >= 0).all() and sizes.sum() == T
    # every chunk but the trailing ones holds exactly T_chunk tokens, none holds more
    tc = -(-T // n)
    assert (sizes <= tc).all()
    if T > 0:
        assert len(sizes[sizes == tc]) == T // tc
    assert (np.diff(sizes) <= 0).all()


# ---------------------------------------------------------------------------------
# metadata and permutation (section 一张专业时序图: batched_pre_dispatch_metadata;
# section 核心原理: permute groups token copies by expert)

def test_metadata_golden():
    g = _load("metadata_small.json")
    m = oracle.metadata(np.array(g["top_k_index"]), g["E"], g["G"], g["N"])
    assert m["bounds"].tolist() == g["bounds"]
    assert m["counts"].tolist() == g["counts"]
    assert m["offsets"].tolist() == g["offsets"]
    assert m["send"].tolist() == g["send_splits"]
    assert m["recv"].tolist() == g["recv_splits"]
    assert m["dst"].tolist() == g["dst"]
    assert m["src_tok"].tolist() == g["src_tok"]


def check_metadata(idx, E, G, N, m):
    """Properties that together determine the permutation uniquely.  Raises AssertionError."""
    T, k = idx.shape
    G = max(G, 1)
    b = oracle.chunk_bounds(T, N)
    n = len(b) - 1
    assert m["bounds"].tolist() == b.tolist()
    flat = idx.reshape(-1)
    for c in range(n):
        s0, s1 = b[c] * k, b[c + 1] * k
        e_c = flat[s0:s1]
        cnt = np.bincount(e_c, minlength=E) if len(e_c) else np.zeros(E, np.int64)
        assert m["counts"][c].tolist() == cnt.tolist()
        assert m["offsets"][c].tolist() == [0] + np.cumsum(cnt).tolist()
        grp = np.bincount(e_c // (E // G), minlength=G) if len(e_c) else np.zeros(G, np.int64)
        assert m["send"][c].tolist() == grp.tolist()
        assert m["recv"][c].tolist() == m["send"][c].tolist()
        d = m["dst"][s0:s1]
        # a bijection onto the chunk's rows
        assert sorted(d.tolist()) == list(range(s1 - s0))
        # expert-contiguous, experts ascending
        lo = m["offsets"][c][e_c]
        hi = m["offsets"][c][e_c + 1]
        assert ((d >= lo) & (d < hi)).all()
        # stable: inside one expert the row grows with the flat index t*k+j
        for e in range(E):
            de = d[e_c == e]
            assert (np.diff(de) > 0).all()
        # src_tok inverts dst
        toks = np.arange(s0, s1) // k
        assert (m["src_tok"][s0 + d] == toks).all()
    assert sum(int(m["send"][c].sum()) for c in range(n)) == T * k


def _all_index_tensors(T, k, E):
    for vals in itertools.product(range(E), repeat=T * k):
        yield np.array(vals, dtype=np.int32).reshape(T, k)


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (1, 2, 3), (2, 2, 2), (3, 1, 4), (3, 2, 2),
                                   (2, 2, 4), (3, 2, 3)])
def test_metadata_bruteforce(T, k, E):
    groups = [g for g in (1, 2, 4) if E % g == 0]
    for idx in _all_index_tensors(T, k, E):
        for N in range(0, 5):
            for G in groups:
                check_metadata(idx, E, G, N, oracle.metadata(idx, E, G, N))


def test_metadata_checker_rejects_planted_mistakes():
    """The property check must catch each plausible metadata mistake planted in the
    oracle's output: an unstable order, a swapped expert order, a wrong count."""
    idx = np.array([[2, 0], [0, 2], [3, 2], [0, 0]], np.int32)
    m = oracle.metadata(idx, 4, 2, 1)
    check_metadata(idx, 4, 2, 1, m)
    # 1) unstable: swap the two rows of expert 0 from tokens 0 and 1
    bad = {k_: v.copy() for k_, v in m.items()}
    a, b_ = 1, 2  # flat slots (0,1) and (1,0), both expert 0
    bad["dst"][a], bad["dst"][b_] = bad["dst"][b_], bad["dst"][a]
    with pytest.raises(AssertionError):
        check_metadata(idx, 4, 2, 1, bad)
    # 2) experts in descending order
    bad = {k_: v.copy() for k_, v in m.items()}
    bad["dst"] = (idx.size - 1 - bad["dst"]).astype(np.int32)
    with pytest.raises(AssertionError):
        check_metadata(idx, 4, 2, 1, bad)
    # 3) a count off by one
    bad = {k_: v.copy() for k_, v in m.items()}
    bad["counts"][0, 0] += 1
    with pytest.raises(AssertionError):
        check_metadata(idx, 4, 2, 1, bad)


def test_metadata_rejects_bad_index():
    with pytest.raises(ValueError):
        oracle.metadata(np.array([[0, 4]], np.int32), 4, 1, 1)
    with pytest.raises(ValueError):
        oracle.metadata(np.array([[-1, 0]], np.int32), 4, 1, 1)


def test_metadata_larger_random():
    rng = np.random.default_rng(3)
    for T, k, E, G, N in [(1000, 6, 64, 8, 8), (49, 6, 64, 4, 8), (513, 2, 8, 2, 3)]:
        idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
        check_metadata(idx, E, G, N, oracle.metadata(idx, E, G, N))


# ---------------------------------------------------------------------------------
# expert FFN (SwiGLU) and the weighted combine


def _bits(a):
    """fp32 values that are exact in bf16 -> their bf16 bit patterns."""
    a = np.asarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    assert (u & 0xFFFF == 0).all(), "value not exact in bf16"
    return (u >> 16).astype(np.uint16)


def _bf16_round(a):
    """Round fp32 values to bf16 (round to nearest even) -> fp32 values."""
    u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def sigmoid_textbook(z):
    return 1.0 / (1.0 + math.exp(-z))


def test_silu_textbook_values_through_identity_expert():
    """One expert with W_gate = W_up = [I_H; 0] and W_down = [I_H 0] maps x to x*silu(x)
    elementwise; compare with textbook values of the logistic function."""
    H, I = 8, 8
    x = np.array([0.0, 1.0, -1.0, 2.0, -2.0, 0.5, 4.0, -8.0], np.float32)
    eye = np.eye(H, dtype=np.float32)
    wgu = _bits(np.concatenate([eye, eye])[None])
    wd = _bits(eye[None])
    out = oracle.forward(_bits(x[None]), np.zeros((1, 1), np.int32), np.ones((1, 1), np.float32),
                         wgu, wd)[0]
    # silu(z) = z * sigmoid(z); sigmoid(1) = 0.7310585786300049, sigmoid(2) = 0.8807970779778823
    expect = {0.0: 0.0, 1.0: 0.7310585786300049, -1.0: -0.2689414213699951,
              2.0: 2 * 0.8807970779778823, -2.0: -2 * 0.11920292202211755}
    for xi, oi in zip(x, out):
        z = float(xi)
        ref = z * z * sigmoid_textbook(z)  # y = x * silu(x) = x^2 sigmoid(x)
        assert oi == pytest.approx(ref, rel=1e-14, abs=1e-300)
        if z in expect:
            assert oi == pytest.approx(z * expect[z], rel=1e-12, abs=1e-300)


def test_identity_like_experts_closed_form():
    """Experts with W_gate[e] = a_e [I_H; 0], W_up[e] = b_e [I_H; 0] and
    W_down[e] = al_e [I_H 0] (all powers of two, exact in bf16).  Then
        out[t] = sum_j w[t,j] * al_e * b_e * x * silu(a_e x)   (e = idx[t,j]),
    which pins routing, the weighting, which half of W_gate_up is the gate, and SwiGLU."""
    rng = np.random.default_rng(7)
    T, H, I, E, k = 24, 16, 32, 4, 3
    a = np.array([1.0, 2.0, 0.5, 1.0])
    b = np.array([1.0, 0.25, 2.0, 4.0])
    al = np.array([1.0, 0.5, 0.25, 0.125])
    pad = np.zeros((I - H, H), np.float32)
    eye = np.eye(H, dtype=np.float32)
    wgu = np.stack([np.concatenate([a[e] * eye, pad, b[e] * eye, pad]) for e in range(E)])
    wd = np.stack([np.concatenate([al[e] * eye, np.zeros((H, I - H), np.float32)], axis=1)
                   for e in range(E)])
    x = _bf16_round(rng.standard_normal((T, H)).astype(np.float32))
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)  # duplicates allowed (reading R6)
    w = rng.uniform(0.1, 1.0, size=(T, k)).astype(np.float32)
    out = oracle.forward(_bits(x), idx, w, _bits(wgu), _bits(wd))
    for t in range(T):
        ref = np.zeros(H)
        for j in range(k):
            e = idx[t, j]
            xe = x[t].astype(np.float64)
            ref += float(w[t, j]) * al[e] * b[e] * xe * (a[e] * xe) / (1 + np.exp(-a[e] * xe))
        np.testing.assert_allclose(out[t], ref, rtol=1e-13, atol=1e-300)


def _numpy_ffn(xe, wgu_e, wd_e):
    I = wgu_e.shape[0] // 2
    g = wgu_e[:I] @ xe
    u = wgu_e[I:] @ xe
    h = g / (1 + np.exp(-g)) * u
    return wd_e @ h


def test_ffn_matches_numpy_matmul():
    """Random small experts (H != I so a transposed operand cannot pass)."""
    rng = np.random.default_rng(11)
    T, H, I, E, k = 9, 16, 40, 3, 2
    x = _bf16_round(rng.standard_normal((T, H)))
    wgu = _bf16_round(rng.standard_normal((E, 2 * I, H)) / 4)
    wd = _bf16_round(rng.standard_normal((E, H, I)) / 6)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    w = rng.uniform(0, 1, size=(T, k)).astype(np.float32)
    out = oracle.forward(_bits(x), idx, w, _bits(wgu), _bits(wd))
    for t in range(T):
        ref = sum(float(w[t, j]) * _numpy_ffn(x[t].astype(np.float64),
                                              wgu[idx[t, j]].astype(np.float64),
                                              wd[idx[t, j]].astype(np.float64))
                  for j in range(k))
        np.testing.assert_allclose(out[t], ref, rtol=1e-12, atol=1e-12)
    # a token subset returns the same rows
    sub = oracle.forward(_bits(x), idx, w, _bits(wgu), _bits(wd), tokens=[8, 0, 3])
    np.testing.assert_array_equal(sub, out[[8, 0, 3]])


def test_equal_experts_return_the_dense_ffn():
    """All experts equal and weights summing to 1: the layer is the one dense FFN."""
    rng = np.random.default_rng(5)
    T, H, I, E, k = 12, 16, 24, 5, 3
    x = _bf16_round(rng.standard_normal((T, H)))
    w0 = _bf16_round(rng.standard_normal((2 * I, H)) / 4)
    d0 = _bf16_round(rng.standard_normal((H, I)) / 4)
    wgu = np.stack([w0] * E)
    wd = np.stack([d0] * E)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    w = rng.uniform(0.1, 1, size=(T, k))
    w = (w / w.sum(1, keepdims=True)).astype(np.float32)
    out = oracle.forward(_bits(x), idx, w, _bits(wgu), _bits(wd))
    dense = oracle.forward(_bits(x), np.zeros((T, 1), np.int32), np.ones((T, 1), np.float32),
                           _bits(w0[None]), _bits(d0[None]))
    wsum = w.astype(np.float64).sum(1, keepdims=True)  # 1 up to fp32 rounding of w
    np.testing.assert_allclose(out, dense * wsum, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(out, dense, rtol=1e-6, atol=1e-7)


def test_combine_is_linear_in_weights():
    rng = np.random.default_rng(9)
    T, H, I, E, k = 6, 8, 16, 3, 2
    x = _bf16_round(rng.standard_normal((T, H)))
    wgu = _bf16_round(rng.standard_normal((E, 2 * I, H)) / 3)
    wd = _bf16_round(rng.standard_normal((E, H, I)) / 3)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    w1 = np.zeros((T, k), np.float32); w1[:, 0] = 1
    w2 = np.zeros((T, k), np.float32); w2[:, 1] = 1
    o1 = oracle.forward(_bits(x), idx, w1, _bits(wgu), _bits(wd))
    o2 = oracle.forward(_bits(x), idx, w2, _bits(wgu), _bits(wd))
    o12 = oracle.forward(_bits(x), idx, w1 + w2, _bits(wgu), _bits(wd))
    np.testing.assert_allclose(o12, o1 + o2, rtol=1e-13, atol=1e-15)
    # each one-hot weight picks exactly one expert's FFN
    for t in range(T):
        ref = _numpy_ffn(x[t].astype(np.float64), wgu[idx[t, 1]].astype(np.float64),
                         wd[idx[t, 1]].astype(np.float64))
        np.testing.assert_allclose(o2[t], ref, rtol=1e-12, atol=1e-13)


def test_worked_example_by_hand():
    """H=I=2, one expert: W_gate = I_2, W_up = diag(2, 1), W_down = [[1, 1], [0, 1]],
    x = (1, -1).  g = (1, -1), u = (2, -1), h = (2 silu(1), -silu(-1)),
    silu(1) = sigmoid(1) = 0.7310585786300049, silu(-1) = -0.2689414213699951, so
    h = (1.4621171572600098, 0.2689414213699951) and y = (h0 + h1, h1)."""
    wgu = _bits(np.array([[[1, 0], [0, 1], [2, 0], [0, 1]]], np.float32))
    wd = _bits(np.array([[[1, 1], [0, 1]]], np.float32))
    x = _bits(np.array([[1, -1]], np.float32))
    out = oracle.forward(x, np.array([[0, 0]], np.int32),
                         np.array([[0.75, 0.25]], np.float32), wgu, wd)[0]
    np.testing.assert_allclose(out, [1.7310585786300049, 0.2689414213699951], rtol=1e-14)


# ---------------------------------------------------------------------------------
# stage oracles: permute, grouped gate/up, grouped down, unpermute

def test_permute_then_unpermute_restores_tokens():
    rng = np.random.default_rng(1)
    T, H, E, k = 37, 24, 6, 3
    x = _bf16_round(rng.standard_normal((T, H)))
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    m = oracle.metadata(idx, E, 1, 1)
    X = oracle.permute(_bits(x), m["dst"], k)
    # every permuted row is its source token, bit for bit
    np.testing.assert_array_equal(X, _bits(x)[m["src_tok"]])
    w = rng.uniform(0, 1, size=(T, k)).astype(np.float32)
    back = oracle.unpermute(X, m["dst"], w, k)
    np.testing.assert_allclose(back, x * w.astype(np.float64).sum(1, keepdims=True),
                               rtol=1e-15, atol=0)


def test_stage_gemms_match_numpy():
    rng = np.random.default_rng(2)
    rows, H, I, E = 50, 16, 24, 4
    X = _bf16_round(rng.standard_normal((rows, H)))
    wgu = _bf16_round(rng.standard_normal((E, 2 * I, H)) / 4)
    wd = _bf16_round(rng.standard_normal((E, H, I)) / 5)
    eor = np.sort(rng.integers(0, E, size=rows)).astype(np.int32)
    act = oracle.gateup_rows(_bits(X), eor, _bits(wgu))
    A = _bf16_round(rng.standard_normal((rows, I)))
    y = oracle.down_rows(_bits(A), eor, _bits(wd))
    for r in range(rows):
        e = eor[r]
        g = wgu[e, :I].astype(np.float64) @ X[r]
        u = wgu[e, I:].astype(np.float64) @ X[r]
        np.testing.assert_allclose(act[r], g / (1 + np.exp(-g)) * u, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(y[r], wd[e].astype(np.float64) @ A[r], rtol=1e-12,
                                   atol=1e-14)


def test_forward_is_gateup_then_down():
    """The token-by-token forward equals the stage functions chained (with the
    intermediate kept in fp64 by forward), on a case where Act is exact in bf16."""
    H, I = 8, 8
    eye = np.eye(H, dtype=np.float32)
    wgu = _bits(np.concatenate([eye, eye])[None])
    wd = _bits(eye[None])
    x = np.array([[0.0, 1.0, -1.0, 2.0, 0.0, 0.0, 0.0, 0.0]], np.float32)
    act = oracle.gateup_rows(_bits(x), np.zeros(1, np.int32), wgu)
    np.testing.assert_allclose(act[0], x[0] * x[0] / (1 + np.exp(-x[0].astype(np.float64))),
                               rtol=1e-14)
