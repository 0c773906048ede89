"""CPU oracle of the chunked MoE forward pass -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package.  The CUDA library never calls it, and nothing here calls the CUDA
library: the two share no code.  Every function is a thin ctypes wrapper around
``oracle.c`` (plain C, fp64), which cites the passage of the Chunk MoE article that each
definition follows.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def use_library(path=None):
    """Point the wrappers at another build of oracle.c (None: the default build).  The
    tests use it to run the pins against deliberately broken copies of the oracle."""
    global _lib
    _lib = None if path is None else _bind(ctypes.CDLL(path))


def lib():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(_build.build()))
    return _lib


def _bind(L):
    """Declare the argument and return types of the oracle's C functions on L."""
    i32, i64, p, d = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    L.oracle_effective_chunks.argtypes = [i32]
    L.oracle_effective_chunks.restype = ctypes.c_int
    L.oracle_chunk_bounds.argtypes = [i64, i32, p]
    L.oracle_chunk_bounds.restype = None
    L.oracle_metadata.argtypes = [p, i64, i32, i32, i32, i32, p, p, p, p, p, p]
    L.oracle_metadata.restype = i64
    L.oracle_metadata_sized.argtypes = [p, i64, i32, i32, i32, i32, i64, p, p, p, p, p, p]
    L.oracle_metadata_sized.restype = i64
    L.oracle_resolve_chunks.argtypes = [i64, i32, i32, p, p]
    L.oracle_resolve_chunks.restype = ctypes.c_int
    L.oracle_chunk_bounds_sized.argtypes = [i64, i32, i64, p]
    L.oracle_chunk_bounds_sized.restype = None
    L.oracle_forward.argtypes = [p, p, p, p, p, i64, i32, i32, i32, i32, p, i64, p, d]
    L.oracle_forward.restype = i64
    L.oracle_permute.argtypes = [p, p, i64, i32, i32, p]
    L.oracle_permute.restype = None
    L.oracle_gateup_rows.argtypes = [p, p, i64, p, i32, i32, p, d]
    L.oracle_gateup_rows.restype = None
    L.oracle_down_rows.argtypes = [p, p, i64, p, i32, i32, p, d]
    L.oracle_down_rows.restype = None
    L.oracle_unpermute.argtypes = [p, p, p, i64, i32, i32, p]
    L.oracle_unpermute.restype = None
    L.oracle_backward.argtypes = [p, p, p, p, p, p, i64, i32, i32, i32, i32, p, p, p, p, d]
    L.oracle_backward.restype = i64
    L.oracle_max_threads.argtypes = []
    L.oracle_max_threads.restype = ctypes.c_int
    return L


def _c(a, dtype):
    """C-contiguous numpy array of `dtype` (bf16 tensors travel as uint16 bits)."""
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def effective_chunks(num_chunks: int) -> int:
    return int(lib().oracle_effective_chunks(num_chunks))


def chunk_bounds(T: int, num_chunks: int) -> np.ndarray:
    n = effective_chunks(num_chunks)
    b = np.zeros(n + 1, dtype=np.int64)
    lib().oracle_chunk_bounds(T, num_chunks, _ptr(b))
    return b


def resolve_chunks(T: int, num_chunks: int, chunk_size: int = 0):
    """(n_chunks, t_chunk, warned) from the two chunk settings."""
    n = ctypes.c_int32(0)
    tc = ctypes.c_int64(0)
    r = lib().oracle_resolve_chunks(T, num_chunks, chunk_size, ctypes.byref(n), ctypes.byref(tc))
    if r < 0:
        raise ValueError("negative chunk setting")
    return int(n.value), int(tc.value), bool(r)


def chunk_bounds_sized(T: int, num_chunks: int, chunk_size: int = 0) -> np.ndarray:
    n, tc, _ = resolve_chunks(T, num_chunks, chunk_size)
    b = np.zeros(n + 1, dtype=np.int64)
    lib().oracle_chunk_bounds_sized(T, n, tc, _ptr(b))
    return b


def metadata(idx, E: int, G: int, num_chunks: int, chunk_size: int = 0):
    """Per-chunk counts/offsets/splits and the permutation of every (t, j) copy.

    Returns a dict with counts [N,E], offsets [N,E+1], send [N,G], recv [N,G],
    dst [T*k], src_tok [T*k], bounds [N+1]; raises ValueError on an out-of-range index.
    """
    idx = _c(idx, np.int32)
    T, k = idx.shape
    G = max(int(G), 1)
    n, tc, _ = resolve_chunks(T, num_chunks, chunk_size)
    out = dict(
        counts=np.zeros((n, E), np.int32), offsets=np.zeros((n, E + 1), np.int32),
        send=np.zeros((n, G), np.int32), recv=np.zeros((n, G), np.int32),
        dst=np.full(T * k, -1, np.int32), src_tok=np.full(T * k, -1, np.int32))
    bad = lib().oracle_metadata_sized(_ptr(idx), T, k, E, G, n, tc, _ptr(out["counts"]),
                                      _ptr(out["offsets"]), _ptr(out["send"]), _ptr(out["recv"]),
                                      _ptr(out["dst"]), _ptr(out["src_tok"]))
    if bad:
        raise ValueError(f"{bad} top_k_index entries outside [0, {E})")
    out["bounds"] = chunk_bounds_sized(T, num_chunks, chunk_size)
    return out


def forward(hidden_bits, idx, w, wgu_bits, wd_bits, tokens=None, nthreads: int = 0):
    """fp64 MoE forward rows out[n] for token tokens[n] (all tokens when None).

    hidden_bits [T,H] uint16 (bf16 bits); idx [T,k] int32; w [T,k] float32;
    wgu_bits [E,2I,H] uint16; wd_bits [E,H,I] uint16.
    """
    hidden_bits = _c(hidden_bits, np.uint16)
    idx = _c(idx, np.int32)
    w = _c(w, np.float32)
    wgu_bits = _c(wgu_bits, np.uint16)
    wd_bits = _c(wd_bits, np.uint16)
    T, H = hidden_bits.shape
    E, twoI, H2 = wgu_bits.shape
    I = twoI // 2
    k = idx.shape[1]
    assert H2 == H and wd_bits.shape == (E, H, I) and idx.shape == (T, k) == w.shape
    toks = None if tokens is None else _c(tokens, np.int64)
    n = T if toks is None else len(toks)
    out = np.zeros((n, H), np.float64)
    bad = lib().oracle_forward(_ptr(hidden_bits), _ptr(idx), _ptr(w), _ptr(wgu_bits),
                               _ptr(wd_bits), T, H, I, E, k, _ptr(toks), n, _ptr(out), nthreads)
    if bad:
        raise ValueError(f"{bad} top_k_index entries outside [0, {E})")
    return out


def permute(hidden_bits, dst, k: int):
    hidden_bits = _c(hidden_bits, np.uint16)
    dst = _c(dst, np.int32)
    Tc, H = hidden_bits.shape
    X = np.zeros((Tc * k, H), np.uint16)
    lib().oracle_permute(_ptr(hidden_bits), _ptr(dst), Tc, H, k, _ptr(X))
    return X


def gateup_rows(X_bits, expert_of_row, wgu_bits, nthreads: int = 0):
    X_bits = _c(X_bits, np.uint16)
    eor = _c(expert_of_row, np.int32)
    wgu_bits = _c(wgu_bits, np.uint16)
    rows, H = X_bits.shape
    I = wgu_bits.shape[1] // 2
    act = np.zeros((rows, I), np.float64)
    lib().oracle_gateup_rows(_ptr(X_bits), _ptr(eor), rows, _ptr(wgu_bits), H, I, _ptr(act),
                             nthreads)
    return act


def down_rows(act_bits, expert_of_row, wd_bits, nthreads: int = 0):
    act_bits = _c(act_bits, np.uint16)
    eor = _c(expert_of_row, np.int32)
    wd_bits = _c(wd_bits, np.uint16)
    rows, I = act_bits.shape
    H = wd_bits.shape[1]
    y = np.zeros((rows, H), np.float64)
    lib().oracle_down_rows(_ptr(act_bits), _ptr(eor), rows, _ptr(wd_bits), H, I, _ptr(y),
                           nthreads)
    return y


def unpermute(Y_bits, dst, w, k: int):
    Y_bits = _c(Y_bits, np.uint16)
    dst = _c(dst, np.int32)
    w = _c(w, np.float32).reshape(-1)
    Tc = dst.size // k
    H = Y_bits.shape[1]
    out = np.zeros((Tc, H), np.float64)
    lib().oracle_unpermute(_ptr(Y_bits), _ptr(dst), _ptr(w), Tc, H, k, _ptr(out))
    return out


def backward(hidden_bits, idx, w, wgu_bits, wd_bits, dout_bits, nthreads: int = 0):
    """fp64 gradients of sum(out * dout): returns (d_hidden [T,H], d_weights [T,k],
    dW_gate_up [E,2I,H], dW_down [E,H,I])."""
    hidden_bits = _c(hidden_bits, np.uint16)
    idx = _c(idx, np.int32)
    w = _c(w, np.float32)
    wgu_bits = _c(wgu_bits, np.uint16)
    wd_bits = _c(wd_bits, np.uint16)
    dout_bits = _c(dout_bits, np.uint16)
    T, H = hidden_bits.shape
    E, twoI, _ = wgu_bits.shape
    I = twoI // 2
    k = idx.shape[1]
    dx = np.zeros((T, H), np.float64)
    dw = np.zeros((T, k), np.float64)
    dwgu = np.zeros((E, 2 * I, H), np.float64)
    dwd = np.zeros((E, H, I), np.float64)
    bad = lib().oracle_backward(_ptr(hidden_bits), _ptr(idx), _ptr(w), _ptr(wgu_bits),
                                _ptr(wd_bits), _ptr(dout_bits), T, H, I, E, k, _ptr(dx), _ptr(dw),
                                _ptr(dwgu), _ptr(dwd), nthreads)
    if bad:
        raise ValueError("top_k_index entries outside [0, E)")
    return dx, dw, dwgu, dwd
