"""Chunked MoE forward on one NVIDIA B200 -- thin Python binding of libmoe.so.

Every function here only marshals arguments (tensor pointers, sizes, the current CUDA
stream) into the C ABI declared in include/moe.h; all the work runs in the library's
CUDA kernels.  There is no fallback: if libmoe.so is missing or fails to load, every
call raises.  PyTorch is used for device memory and streams only.

The method is Chunk MoE from the MindSpeed article "昇腾MindSpeed分块专家计算Chunk MoE":
the layer's tokens are split into N chunks of ceil(T/N) tokens (section 一组关键公式),
adjacent chunks run as a pair over a double-buffered workspace (section 一张专业时序图),
and the split/count metadata of all chunks comes back to the host in one copy.
"""
import ctypes
import os
import warnings

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_LIBRARY=checks selects the range-checked build (libmoe_checks.so), used by its tests.
LIB_PATH = os.path.join(_PKG, "libmoe_checks.so" if os.environ.get("MOE_LIBRARY") == "checks"
                        else "libmoe.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_ARG", 2: "MOE_ERR_INDEX", 3: "MOE_ERR_ALIGN",
                4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_CUDA", 6: "MOE_ERR_TIMEOUT",
                7: "MOE_ERR_UNSUPPORTED"}
KERNEL_KINDS = ("metadata", "permute", "gateup", "down", "unpermute", "bwd_gateup", "bwd_dswiglu",
                "bwd_dx", "bwd_wgrad", "bwd_rows")
_NK = len(KERNEL_KINDS)  # MOE_KERNEL_KINDS


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class Shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("ep_groups", ctypes.c_int32),
                ("num_chunks", ctypes.c_int32), ("chunk_size", ctypes.c_int32)]


class LaunchRecord(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("stream", ctypes.c_int32), ("call", ctypes.c_int64),
                ("rows", ctypes.c_int64), ("start_ms", ctypes.c_double),
                ("end_ms", ctypes.c_double)]


STREAM_NAMES = ("caller", "side", "copy_in", "copy_out")


class Profile(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int64 * _NK), ("ms", ctypes.c_double * _NK),
                ("rows", ctypes.c_int64 * _NK), ("active_experts", ctypes.c_int64 * _NK),
                ("kernels", ctypes.c_int64)]


_lib = None


def load():
    """Load libmoe.so (built in-tree by build.py); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          f"`python -m expert_router_top_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    p, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    st = ctypes.c_int
    L.moe_status_string.argtypes = [st]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_abi_version.argtypes = []
    L.moe_abi_version.restype = i32
    L.moe_chunk_bounds.argtypes = [i64, i32, p]
    L.moe_chunk_bounds.restype = st
    L.moe_resolve_chunks.argtypes = [ctypes.POINTER(Shape), p, p]
    L.moe_resolve_chunks.restype = st
    L.moe_last_warning.argtypes = []
    L.moe_last_warning.restype = ctypes.c_char_p
    L.moe_metadata_shape.argtypes = [ctypes.POINTER(Shape), p, p, p, p, p, p, p, p, sz, p]
    L.moe_metadata_shape.restype = st
    L.moe_metadata_workspace_bytes.argtypes = [i64, i32, i32, i32, i32]
    L.moe_metadata_workspace_bytes.restype = sz
    L.moe_workspace_bytes.argtypes = [ctypes.POINTER(Shape)]
    L.moe_workspace_bytes.restype = sz
    L.moe_metadata.argtypes = [p, i64, i32, i32, i32, i32, p, p, p, p, p, p, p, sz, p]
    L.moe_metadata.restype = st
    L.moe_forward.argtypes = [ctypes.POINTER(Shape), p, p, p, p, p, p, p, sz, p]
    L.moe_forward.restype = st
    L.moe_forward_ex.argtypes = [ctypes.POINTER(Shape), p, p, p, p, p, p, p, sz, ctypes.c_uint32,
                                 p]
    L.moe_forward_ex.restype = st
    L.moe_checks_enabled.argtypes = []
    L.moe_checks_enabled.restype = i32
    L.moe_checks_read.argtypes = [p]
    L.moe_checks_read.restype = st
    L.moe_selftest_wait_timeout.argtypes = [p, ctypes.c_uint32, p]
    L.moe_selftest_wait_timeout.restype = st
    L.moe_forward_dispatch.argtypes = [ctypes.POINTER(Shape), ctypes.c_uint32]
    L.moe_forward_dispatch.restype = i32
    L.moe_workspace_bytes_host.argtypes = [ctypes.POINTER(Shape)]
    L.moe_workspace_bytes_host.restype = sz
    L.moe_forward_host.argtypes = [ctypes.POINTER(Shape), p, p, p, p, p, p, p, sz, p]
    L.moe_forward_host.restype = st
    L.moe_backward_workspace_bytes.argtypes = [ctypes.POINTER(Shape)]
    L.moe_backward_workspace_bytes.restype = sz
    L.moe_backward.argtypes = [ctypes.POINTER(Shape), p, p, p, p, p, p, p, p, p, p, p, sz, p]
    L.moe_backward.restype = st
    L.moe_check_device_status.argtypes = [p, sz, p]
    L.moe_check_device_status.restype = st
    L.moe_permute.argtypes = [p, p, i64, i32, i32, p, p]
    L.moe_permute.restype = st
    L.moe_grouped_gateup.argtypes = [p, i64, i32, i32, i32, p, p, p, p, p, p]
    L.moe_grouped_gateup.restype = st
    L.moe_grouped_down.argtypes = [p, i64, i32, i32, i32, p, p, p, p, p, p]
    L.moe_grouped_down.restype = st
    L.moe_unpermute.argtypes = [p, p, p, i64, i32, i32, p, p]
    L.moe_unpermute.restype = st
    L.moe_profile_enable.argtypes = [i32]
    L.moe_profile_enable.restype = st
    L.moe_profile_read.argtypes = [ctypes.POINTER(Profile)]
    L.moe_profile_read.restype = st
    L.moe_profile_timeline.argtypes = [ctypes.POINTER(LaunchRecord), i32, ctypes.POINTER(i32)]
    L.moe_profile_timeline.restype = st
    L.moe_ep_plan.argtypes = [p, i32, i32, i32, p, p]
    L.moe_ep_plan.restype = st
    L.moe_ep_dispatch.argtypes = [p, p, p, p, p, i64, i32, i32, i32, i32, i64, p]
    L.moe_ep_dispatch.restype = st
    L.moe_ep_combine.argtypes = [p, p, p, p, p, i64, i32, i32, i32, i32, i64, p, p]
    L.moe_ep_combine.restype = st
    L.moe_ipc_handle.argtypes = [p, p, ctypes.POINTER(i64)]
    L.moe_ipc_handle.restype = st
    L.moe_ipc_open.argtypes = [p, i64, ctypes.POINTER(p)]
    L.moe_ipc_open.restype = st
    L.moe_ipc_close.argtypes = [p, i64]
    L.moe_ipc_close.restype = st
    _lib = L
    return L


def status_string(status: int) -> str:
    return load().moe_status_string(status).decode()


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoEError(status, what)
    msg = load().moe_last_warning()
    if msg:
        warnings.warn(f"{what}: {msg.decode()}", stacklevel=3)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data_as(ctypes.c_void_p)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name, device=True):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def shape(T, H, I, E, k, ep_groups=1, num_chunks=1, chunk_size=0) -> Shape:
    return Shape(T, H, I, E, k, ep_groups, num_chunks, chunk_size)


def resolve_chunks(T: int, num_chunks: int = 0, chunk_size: int = 0):
    """(chunk count, tokens per chunk) under the num_chunks / chunk_size precedence rule."""
    n = ctypes.c_int32(0)
    tc = ctypes.c_int64(0)
    s = shape(T, 8, 8, 1, 1, 1, num_chunks, chunk_size)
    _check(load().moe_resolve_chunks(ctypes.byref(s), ctypes.byref(n), ctypes.byref(tc)),
           "moe_resolve_chunks")
    return int(n.value), int(tc.value)


def chunk_bounds(T: int, num_chunks: int) -> np.ndarray:
    b = np.zeros(max(num_chunks, 1) + 1, np.int64)
    _check(load().moe_chunk_bounds(T, num_chunks, _ptr(b)), "moe_chunk_bounds")
    return b


def workspace_bytes(T, H, I, E, k, ep_groups=1, num_chunks=1, chunk_size=0) -> int:
    s = shape(T, H, I, E, k, ep_groups, num_chunks, chunk_size)
    return int(load().moe_workspace_bytes(ctypes.byref(s)))


def metadata_workspace_bytes(T, k, E, ep_groups=1, num_chunks=1) -> int:
    return int(load().moe_metadata_workspace_bytes(T, k, E, ep_groups, num_chunks))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A caller-owned device workspace (uint8, 256-byte aligned by the allocator)."""
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device or "cuda")


def metadata(top_k_index: torch.Tensor, E: int, ep_groups: int = 1, num_chunks: int = 1,
             with_permutation: bool = False, workspace: torch.Tensor = None, stream=None,
             chunk_size: int = 0):
    """Batched metadata for every chunk (one device pass, one host copy).

    Returns a dict of numpy arrays: send/recv [N,G], counts [N,E], bounds [N+1]; with
    with_permutation also torch int32 dst [T*k] and src_tok [T*k] on the device."""
    _need(top_k_index, torch.int32, "top_k_index")
    T, k = top_k_index.shape
    n = resolve_chunks(T, num_chunks, chunk_size)[0] if chunk_size > 0 else max(num_chunks, 1)
    G = max(ep_groups, 1)
    send = np.zeros((n, G), np.int32)
    recv = np.zeros((n, G), np.int32)
    counts = np.zeros((n, E), np.int32)
    bounds = np.zeros(n + 1, np.int64)
    dst = src = None
    if with_permutation:
        dst = torch.empty(T * k, dtype=torch.int32, device=top_k_index.device)
        src = torch.empty(T * k, dtype=torch.int32, device=top_k_index.device)
    if chunk_size > 0:
        s = shape(T, 8, 8, E, k, ep_groups, num_chunks, chunk_size)
        if workspace is None:
            workspace = alloc_workspace(load().moe_workspace_bytes(ctypes.byref(s)),
                                        top_k_index.device)
        _check(load().moe_metadata_shape(ctypes.byref(s), _ptr(top_k_index), _ptr(send),
                                         _ptr(recv), _ptr(counts), _ptr(bounds), _ptr(dst),
                                         _ptr(src), _ptr(workspace), workspace.numel(),
                                         _stream(stream)), "moe_metadata_shape")
    else:
        if workspace is None:
            workspace = alloc_workspace(metadata_workspace_bytes(T, k, E, ep_groups, num_chunks),
                                        top_k_index.device)
        _check(load().moe_metadata(_ptr(top_k_index), T, k, E, ep_groups, num_chunks, _ptr(send),
                                   _ptr(recv), _ptr(counts), _ptr(bounds), _ptr(dst), _ptr(src),
                                   _ptr(workspace), workspace.numel(), _stream(stream)),
               "moe_metadata")
    out = dict(send=send, recv=recv, counts=counts, bounds=bounds)
    if with_permutation:
        out["dst"], out["src_tok"] = dst, src
    return out


FWD_FUSED_DISPATCH = 1
FWD_SEPARATE_DISPATCH = 2
_DISPATCH = {"auto": 0, "fused": FWD_FUSED_DISPATCH, "separate": FWD_SEPARATE_DISPATCH}


def _dispatch_flags(dispatch):
    if dispatch not in _DISPATCH:
        raise ValueError(f"dispatch must be one of {sorted(_DISPATCH)}, not {dispatch!r}")
    return _DISPATCH[dispatch]


def forward_dispatch(T, H, I, E, k, dispatch="auto", ep_groups=1, num_chunks=1) -> str:
    """The dispatch ("fused" or "separate") that forward() takes for this shape."""
    s = shape(T, H, I, E, k, ep_groups, num_chunks, 0)
    r = int(load().moe_forward_dispatch(ctypes.byref(s), _dispatch_flags(dispatch)))
    if r < 0:
        raise ValueError("invalid dispatch flags")
    return "fused" if r == 1 else "separate"


FWD_PER_CHUNK_GEMMS = 4


def forward(hidden, top_k_index, top_k_weights, W_gate_up, W_down, num_chunks: int = 1,
            ep_groups: int = 1, out=None, workspace=None, stream=None,
            dispatch: str = "auto", chunk_size: int = 0, pair_gemms: bool = True):
    """One MoE layer forward, chunked as Chunk MoE.  Returns out [T,H] bf16.

    hidden [T,H] bf16, top_k_index [T,k] int32, top_k_weights [T,k] fp32,
    W_gate_up [E,2I,H] bf16 (gate rows then up rows), W_down [E,H,I] bf16; all on the
    same CUDA device.  Asynchronous after its single metadata copy.
    dispatch="separate": a permute kernel writes the permuted rows first; "fused": the
    gate/up GEMM gathers its rows from `hidden`; "auto": the library's choice for the
    shape (forward_dispatch).  pair_gemms=False: with the fused dispatch, one GEMM sweep per
    chunk instead of one per pair of chunks.  All give identical bits."""
    _dispatch_flags(dispatch)
    _need(hidden, torch.bfloat16, "hidden")
    _need(top_k_index, torch.int32, "top_k_index")
    _need(top_k_weights, torch.float32, "top_k_weights")
    _need(W_gate_up, torch.bfloat16, "W_gate_up")
    _need(W_down, torch.bfloat16, "W_down")
    T, H = hidden.shape
    E, twoI, H2 = W_gate_up.shape
    I = twoI // 2
    k = top_k_index.shape[1]
    if H2 != H or tuple(W_down.shape) != (E, H, I) or tuple(top_k_index.shape) != (T, k) \
            or tuple(top_k_weights.shape) != (T, k):
        raise ValueError("inconsistent shapes")
    s = shape(T, H, I, E, k, ep_groups, num_chunks, chunk_size)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=hidden.device)
    if workspace is None:
        workspace = alloc_workspace(load().moe_workspace_bytes(ctypes.byref(s)), hidden.device)
    flags = _dispatch_flags(dispatch) | (0 if pair_gemms else FWD_PER_CHUNK_GEMMS)
    _check(load().moe_forward_ex(ctypes.byref(s), _ptr(hidden), _ptr(top_k_index),
                                 _ptr(top_k_weights), _ptr(W_gate_up), _ptr(W_down), _ptr(out),
                                 _ptr(workspace), workspace.numel(), flags, _stream(stream)),
           "moe_forward_ex")
    return out


def workspace_bytes_host(T, H, I, E, k, ep_groups=1, num_chunks=1, chunk_size=0) -> int:
    s = shape(T, H, I, E, k, ep_groups, num_chunks, chunk_size)
    return int(load().moe_workspace_bytes_host(ctypes.byref(s)))


def forward_host(hidden, top_k_index, top_k_weights, W_gate_up, W_down, num_chunks: int = 1,
                 ep_groups: int = 1, out=None, workspace=None, stream=None, chunk_size: int = 0):
    """moe_forward_host: activations in host memory (CPU tensors; pinned ones let the
    per-chunk copies overlap the kernels), weights on the device.  Returns out [T,H] bf16
    on the host, complete when the call returns."""
    _need(hidden, torch.bfloat16, "hidden", device=False)
    _need(top_k_index, torch.int32, "top_k_index", device=False)
    _need(top_k_weights, torch.float32, "top_k_weights", device=False)
    _need(W_gate_up, torch.bfloat16, "W_gate_up")
    _need(W_down, torch.bfloat16, "W_down")
    if hidden.is_cuda or top_k_index.is_cuda or top_k_weights.is_cuda:
        raise ValueError("forward_host takes host (CPU) activations")
    T, H = hidden.shape
    E, twoI, _ = W_gate_up.shape
    k = top_k_index.shape[1]
    s = shape(T, H, twoI // 2, E, k, ep_groups, num_chunks, chunk_size)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, pin_memory=hidden.is_pinned())
    if workspace is None:
        workspace = alloc_workspace(load().moe_workspace_bytes_host(ctypes.byref(s)),
                                    W_gate_up.device)
    _check(load().moe_forward_host(ctypes.byref(s), _ptr(hidden), _ptr(top_k_index),
                                   _ptr(top_k_weights), _ptr(W_gate_up), _ptr(W_down), _ptr(out),
                                   _ptr(workspace), workspace.numel(), _stream(stream)),
           "moe_forward_host")
    return out


def backward_workspace_bytes(T, H, I, E, k, ep_groups=1, num_chunks=1, chunk_size=0) -> int:
    s = shape(T, H, I, E, k, ep_groups, num_chunks, chunk_size)
    return int(load().moe_backward_workspace_bytes(ctypes.byref(s)))


def backward_buffers(T, H, I, E, k, device):
    """Output tensors of backward(): (d_hidden, d_weights, dW_gate_up, dW_down)."""
    return (torch.empty((T, H), dtype=torch.bfloat16, device=device),
            torch.empty((T, k), dtype=torch.float32, device=device),
            torch.empty((E, 2 * I, H), dtype=torch.float32, device=device),
            torch.empty((E, H, I), dtype=torch.float32, device=device))


def backward(hidden, top_k_index, top_k_weights, W_gate_up, W_down, d_out, num_chunks: int = 1,
             ep_groups: int = 1, chunk_size: int = 0, workspace=None, stream=None, out=None):
    """Backward of forward() for the loss sum(out * d_out), with the expert computation
    recomputed chunk by chunk.  Returns (d_hidden bf16 [T,H], d_weights fp32 [T,k],
    dW_gate_up fp32 [E,2I,H], dW_down fp32 [E,H,I]), written into `out` when given."""
    for t, dt, name in ((hidden, torch.bfloat16, "hidden"), (top_k_index, torch.int32, "top_k_index"),
                        (top_k_weights, torch.float32, "top_k_weights"),
                        (W_gate_up, torch.bfloat16, "W_gate_up"), (W_down, torch.bfloat16, "W_down"),
                        (d_out, torch.bfloat16, "d_out")):
        _need(t, dt, name)
    T, H = hidden.shape
    E, twoI, _ = W_gate_up.shape
    I = twoI // 2
    k = top_k_index.shape[1]
    s = shape(T, H, I, E, k, ep_groups, num_chunks, chunk_size)
    dev = hidden.device
    if out is None:
        out = backward_buffers(T, H, I, E, k, dev)
    d_hidden, d_weights, dW_gate_up, dW_down = out
    for t, dt, shp, name in ((d_hidden, torch.bfloat16, (T, H), "d_hidden"),
                             (d_weights, torch.float32, (T, k), "d_weights"),
                             (dW_gate_up, torch.float32, (E, 2 * I, H), "dW_gate_up"),
                             (dW_down, torch.float32, (E, H, I), "dW_down")):
        _need(t, dt, name)
        if tuple(t.shape) != shp:
            raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {shp}")
    if workspace is None:
        workspace = alloc_workspace(load().moe_backward_workspace_bytes(ctypes.byref(s)), dev)
    _check(load().moe_backward(ctypes.byref(s), _ptr(hidden), _ptr(top_k_index),
                               _ptr(top_k_weights), _ptr(W_gate_up), _ptr(W_down), _ptr(d_out),
                               _ptr(d_hidden), _ptr(d_weights), _ptr(dW_gate_up), _ptr(dW_down),
                               _ptr(workspace), workspace.numel(), _stream(stream)),
           "moe_backward")
    return d_hidden, d_weights, dW_gate_up, dW_down


def check_device_status(workspace, stream=None):
    _check(load().moe_check_device_status(_ptr(workspace), workspace.numel(), _stream(stream)),
           "moe_check_device_status")


def permute(hidden, dst_rows, k: int, X=None, stream=None):
    _need(hidden, torch.bfloat16, "hidden")
    _need(dst_rows, torch.int32, "dst_rows")
    Tc, H = hidden.shape
    if X is None:
        X = torch.empty((Tc * k, H), dtype=torch.bfloat16, device=hidden.device)
    _check(load().moe_permute(_ptr(hidden), _ptr(dst_rows), Tc, H, k, _ptr(X), _stream(stream)),
           "moe_permute")
    return X


def _grouped(fn, A, offsets_dev, counts_host, W, out, status, stream, H, I, what):
    _need(A, torch.bfloat16, "A")
    _need(offsets_dev, torch.int32, "expert_offsets")
    _need(W, torch.bfloat16, "W")
    counts_host = np.ascontiguousarray(counts_host, dtype=np.int32)
    rows = A.shape[0]
    E = counts_host.shape[0]
    own_status = status is None
    if own_status:
        status = torch.zeros(4, dtype=torch.int32, device=A.device)
    _check(fn(_ptr(A), rows, H, I, E, _ptr(offsets_dev), _ptr(counts_host), _ptr(W), _ptr(out),
              _ptr(status), _stream(stream)), what)
    return out, status


def grouped_gateup(X, expert_offsets, expert_counts, W_gate_up, Act=None, status=None,
                   stream=None):
    """Act[r] = bf16(silu(X[r] W_gate[e]^T) * (X[r] W_up[e]^T)) for the rows of each expert."""
    E, twoI, H = W_gate_up.shape
    I = twoI // 2
    if Act is None:
        Act = torch.empty((X.shape[0], I), dtype=torch.bfloat16, device=X.device)
    return _grouped(load().moe_grouped_gateup, X, expert_offsets, expert_counts, W_gate_up, Act,
                    status, stream, H, I, "moe_grouped_gateup")


def grouped_down(Act, expert_offsets, expert_counts, W_down, Y=None, status=None, stream=None):
    """Y[r] = bf16(Act[r] W_down[e]^T) for the rows of each expert."""
    E, H, I = W_down.shape
    if Y is None:
        Y = torch.empty((Act.shape[0], H), dtype=torch.bfloat16, device=Act.device)
    return _grouped(load().moe_grouped_down, Act, expert_offsets, expert_counts, W_down, Y, status,
                    stream, H, I, "moe_grouped_down")


def unpermute(Y, dst_rows, top_k_weights, k: int, out=None, stream=None):
    _need(Y, torch.bfloat16, "Y")
    _need(dst_rows, torch.int32, "dst_rows")
    _need(top_k_weights, torch.float32, "top_k_weights")
    H = Y.shape[1]
    Tc = dst_rows.numel() // k
    if out is None:
        out = torch.empty((Tc, H), dtype=torch.bfloat16, device=Y.device)
    _check(load().moe_unpermute(_ptr(Y), _ptr(dst_rows), _ptr(top_k_weights), Tc, H, k, _ptr(out),
                                _stream(stream)), "moe_unpermute")
    return out


def checks_enabled() -> bool:
    """True when the loaded library is the range-checked build."""
    return bool(load().moe_checks_enabled())


def checks_read() -> int:
    """Range-violation flags raised since the last read (0: every row index was in range);
    clears them.  Always 0 with the regular build."""
    flags = ctypes.c_uint32(0)
    _check(load().moe_checks_read(ctypes.byref(flags)), "moe_checks_read")
    return int(flags.value)


def selftest_wait_timeout(limit_us: int = 20000, stream=None):
    """Run the failure-detection self-test: a device wait that nothing completes must give
    up after limit_us and report a timeout.  Returns the status code (MOE_ERR_TIMEOUT = 6
    is the expected outcome); never raises for it."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    return int(load().moe_selftest_wait_timeout(_ptr(status), limit_us, _stream(stream)))


def profile_enable(on: bool = True):
    _check(load().moe_profile_enable(1 if on else 0), "moe_profile_enable")


def profile_read() -> dict:
    p = Profile()
    _check(load().moe_profile_read(ctypes.byref(p)), "moe_profile_read")
    return {kind: dict(launches=int(p.launches[i]), ms=float(p.ms[i]), rows=int(p.rows[i]),
                       active_experts=int(p.active_experts[i]))
            for i, kind in enumerate(KERNEL_KINDS)} | {"kernels": int(p.kernels)}


def profile_timeline(capacity: int = 65536) -> list:
    """The timed launches since profile_enable, in enqueue order: kind, stream, call index,
    rows and start/end times in ms (CUDA events on the launching stream)."""
    recs = (LaunchRecord * capacity)()
    n = ctypes.c_int32(0)
    _check(load().moe_profile_timeline(recs, capacity, ctypes.byref(n)), "moe_profile_timeline")
    return [dict(kind=KERNEL_KINDS[r.kind], stream=STREAM_NAMES[r.stream], call=int(r.call),
                 rows=int(r.rows), start_ms=float(r.start_ms), end_ms=float(r.end_ms))
            for r in recs[:min(n.value, capacity)]]


# ---- expert parallelism over several GPUs (see expert_router_top_b200.ep) -------------------

def ep_plan(counts_all, rank: int):
    """counts_all [W][E] int (one chunk's expert counts of every rank) -> (send_delta [E],
    recv_offsets [E/W + 1]) as int32 numpy arrays (moe_ep_plan, host arithmetic)."""
    c = np.ascontiguousarray(counts_all, dtype=np.int32)
    W, E = c.shape
    delta = np.zeros(E, np.int32)
    offs = np.zeros(E // max(W, 1) + 1, np.int32)
    _check(load().moe_ep_plan(_ptr(c), W, rank, E, _ptr(delta), _ptr(offs)), "moe_ep_plan")
    return delta, offs


def _ptr_table(ptrs, device):
    """Device array of W raw device pointers (int64) for the EP kernels."""
    return torch.tensor([int(x) for x in ptrs], dtype=torch.int64, device=device)


def ep_dispatch(hidden, top_k_index, dst_rows, send_delta, recv_table, E: int, W: int,
                rows_cap: int, stream=None):
    """recv[rank(e)][dst + delta[e]] = hidden[t] for every copy of the chunk (moe_ep_dispatch).
    recv_table: int64 device tensor of W receive-buffer pointers."""
    _need(hidden, torch.bfloat16, "hidden")
    Tc, H = hidden.shape
    k = top_k_index.shape[1]
    _check(load().moe_ep_dispatch(_ptr(hidden), _ptr(top_k_index), _ptr(dst_rows),
                                  _ptr(send_delta), _ptr(recv_table), Tc, H, k, E, W, rows_cap,
                                  _stream(stream)), "moe_ep_dispatch")


def ep_combine(expert_table, top_k_index, dst_rows, send_delta, top_k_weights, H: int, E: int,
               W: int, rows_cap: int, out=None, stream=None):
    """out[t] = sum_j w[t,j] Y[rank(e)][dst + delta[e]], fp32 in ascending j (moe_ep_combine)."""
    Tc, k = top_k_index.shape
    if out is None:
        out = torch.empty((Tc, H), dtype=torch.bfloat16, device=top_k_index.device)
    _check(load().moe_ep_combine(_ptr(expert_table), _ptr(top_k_index), _ptr(dst_rows),
                                 _ptr(send_delta), _ptr(top_k_weights), Tc, H, k, E, W, rows_cap,
                                 _ptr(out), _stream(stream)), "moe_ep_combine")
    return out


def ipc_handle(t: torch.Tensor):
    """(handle bytes, offset) of a device tensor's allocation, for ipc_open in another process."""
    h = ctypes.create_string_buffer(64)
    off = ctypes.c_int64(0)
    _check(load().moe_ipc_handle(_ptr(t), h, ctypes.byref(off)), "moe_ipc_handle")
    return h.raw, off.value


def ipc_open(handle: bytes, offset: int) -> int:
    """Device address of another process's buffer (moe_ipc_open)."""
    out = ctypes.c_void_p(0)
    _check(load().moe_ipc_open(handle, offset, ctypes.byref(out)), "moe_ipc_open")
    return out.value


def ipc_close(ptr: int, offset: int):
    _check(load().moe_ipc_close(ctypes.c_void_p(ptr), offset), "moe_ipc_close")
