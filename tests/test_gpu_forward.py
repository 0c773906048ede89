"""End-to-end chunked forward through the C ABI against the oracle.

Small configurations compare every output element; the full-size layers compare a
seeded sample of tokens (the oracle computes them one by one), and every configuration
checks that the chunked output is bit-identical to the unchunked one."""
import numpy as np
import pytest
import torch

import oracle
from gen import CONFIGS, LayerConfig, bits, expert_weights, hidden, layer_inputs, routing
from parity import assert_layer_close, to_f64

pytestmark = pytest.mark.gpu


def _run(moe, inp, N, G=1, dispatch="separate", pair_gemms=True):
    out = moe.forward(inp["hidden"], inp["idx"], inp["w"], inp["wgu"], inp["wd"], num_chunks=N,
                      ep_groups=G, dispatch=dispatch, pair_gemms=pair_gemms)
    torch.cuda.synchronize()
    return out


def _oracle(inp_cpu, tokens=None):
    return oracle.forward(bits(inp_cpu["hidden"]), inp_cpu["idx"].numpy(), inp_cpu["w"].numpy(),
                          bits(inp_cpu["wgu"]), bits(inp_cpu["wd"]), tokens=tokens)


@pytest.mark.parametrize("dispatch", ["fused", "separate"])
@pytest.mark.parametrize("name", ["tiny", "edge", "edge_pair01", "edge_varlen", "edge_varlen7"])
def test_forward_small_configs_all_tokens(moe, name, dispatch):
    cfg = CONFIGS[name]
    cpu = layer_inputs(cfg)
    gpu = {k: v.cuda() for k, v in cpu.items()}
    ref = _oracle(cpu)
    outs = []
    for N in cfg.chunks:
        out = _run(moe, gpu, N, cfg.G, dispatch)
        assert_layer_close(out, ref, f"{name} N={N} {dispatch}")
        outs.append(out)
    base = _run(moe, gpu, 1, cfg.G, dispatch)
    assert_layer_close(base, ref, f"{name} N=1 {dispatch}")
    for N, o in zip(cfg.chunks, outs):
        assert torch.equal(o, base), f"{name}: N={N} output differs from N=1 ({dispatch})"


@pytest.mark.parametrize("name", ["tiny", "edge", "edge_pair01", "edge_varlen"])
def test_fused_and_separate_dispatch_are_bit_identical(moe, name):
    """Gathering the gate/up GEMM's rows from `hidden` reads the same bf16 values as the
    permute kernel writes, so the two dispatch modes must agree bit for bit."""
    cfg = CONFIGS[name]
    gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
    for N in (1,) + tuple(cfg.chunks):
        assert torch.equal(_run(moe, gpu, N, cfg.G, "fused"), _run(moe, gpu, N, cfg.G, "separate"))


@pytest.mark.parametrize("name", ["tiny", "edge", "edge_pair01", "edge_varlen", "edge_varlen7"])
def test_pair_gemms_match_per_chunk_gemms(moe, name):
    """With the fused dispatch, both chunks of a pair share one tile sweep per GEMM; each
    row's arithmetic is unchanged, so the output equals the per-chunk sweeps bit for bit,
    for even and odd chunk counts (the last chunk of an odd count is alone)."""
    cfg = CONFIGS[name]
    gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
    base = _run(moe, gpu, 1, cfg.G, "separate")
    for N in (2, 3, 4, 5, 8) + tuple(cfg.chunks):
        a = _run(moe, gpu, N, cfg.G, "fused", pair_gemms=True)
        b = _run(moe, gpu, N, cfg.G, "fused", pair_gemms=False)
        assert torch.equal(a, b), f"{name} N={N}: pair sweep differs from per-chunk sweeps"
        assert torch.equal(a, base), f"{name} N={N}: differs from N=1"


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("name", ["tiny", "edge", "edge_varlen", "edge_varlen7"])
def test_forward_host_buffers_match_device_forward(moe, name, pinned):
    """moe_forward_host (activations in host memory, copies pipelined per chunk) gives the
    same bits as moe_forward on device-resident inputs, for every chunking."""
    cfg = CONFIGS[name]
    cpu = layer_inputs(cfg)
    gpu = {k: v.cuda() for k, v in cpu.items()}
    h = cpu["hidden"].pin_memory() if pinned else cpu["hidden"]
    i = cpu["idx"].pin_memory() if pinned else cpu["idx"]
    w = cpu["w"].pin_memory() if pinned else cpu["w"]
    for N in (1, 2, 3) + tuple(cfg.chunks):
        ref = _run(moe, gpu, N, cfg.G)
        got = moe.forward_host(h, i, w, gpu["wgu"], gpu["wd"], num_chunks=N, ep_groups=cfg.G)
        assert not got.is_cuda
        assert torch.equal(got, ref.cpu()), f"{name} N={N} pinned={pinned}"


@pytest.mark.parametrize("pinned", [True, False])
def test_forward_host_fused_gather_from_staged_chunks(moe, pinned):
    """With few expert columns (E*I small against 4*T_chunk*k) moe_forward_host gathers the
    gate/up rows straight from each chunk's staged input, through chunk-relative token
    indices: the same bits as moe_forward for even and odd chunk counts, a ragged last
    chunk and an empty trailing one, and within the layer's bar of the oracle."""
    cfg = LayerConfig("host_fused", 601, 256, 3, 2, 32, "normal")  # fused iff T_chunk >= 12
    cpu = layer_inputs(cfg)
    gpu = {k: v.cuda() for k, v in cpu.items()}
    h, i, w = ((t.pin_memory() if pinned else t) for t in (cpu["hidden"], cpu["idx"], cpu["w"]))
    ref1 = _run(moe, gpu, 1)
    assert_layer_close(ref1, _oracle(cpu), "host_fused N=1 (device)")
    # N=35: chunks of 18 tokens, the 34th holds 7 and the 35th none; N=51: 12 tokens, 1 last
    for N in (1, 2, 3, 5, 35, 51):
        got = moe.forward_host(h, i, w, gpu["wgu"], gpu["wd"], num_chunks=N)
        assert torch.equal(got, ref1.cpu()), f"host_fused N={N} pinned={pinned}"


def test_forward_host_full_size(moe):
    """The Qwen3-shaped 16k layer through moe_forward_host at num_chunks=4 (the fused
    per-chunk path the benchmark's end-to-end number takes) and 8 (the separate one): the
    same bits as moe_forward on device-resident inputs."""
    cfg = CONFIGS["qwen3"]
    idx, w = routing(cfg)
    x = hidden(cfg.T, cfg.H)
    wgu, wd = expert_weights(cfg.E, cfg.H, cfg.I, device="cuda")
    gpu = dict(hidden=x.cuda(), idx=torch.from_numpy(idx).cuda(), w=torch.from_numpy(w).cuda(),
               wgu=wgu, wd=wd)
    for N in (4, 8):
        ref = _run(moe, gpu, N, cfg.G, "auto")
        got = moe.forward_host(x.pin_memory(), torch.from_numpy(idx).pin_memory(),
                               torch.from_numpy(w).pin_memory(), wgu, wd, num_chunks=N)
        assert torch.equal(got, ref.cpu()), f"qwen3 host N={N}"


@pytest.mark.parametrize("S", [1, 143, 333, 1000])
def test_forward_chunk_size(moe, S):
    """moe_chunk_size: chunks of exactly S tokens give the unsplit bits; with both
    settings > 0 the chunk count wins and a warning is raised."""
    cfg = CONFIGS["edge"]
    cpu = layer_inputs(cfg)
    gpu = {k: v.cuda() for k, v in cpu.items()}
    base = _run(moe, gpu, 1)
    out = moe.forward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"], gpu["wd"], num_chunks=0,
                      chunk_size=S)
    torch.cuda.synchronize()
    assert torch.equal(out, base)
    with pytest.warns(UserWarning, match="moe_num_chunks"):
        out2 = moe.forward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"], gpu["wd"],
                           num_chunks=3, chunk_size=S)
    torch.cuda.synchronize()
    assert torch.equal(out2, base)
    host = moe.forward_host(cpu["hidden"].pin_memory(), cpu["idx"].pin_memory(),
                            cpu["w"].pin_memory(), gpu["wgu"], gpu["wd"], num_chunks=0,
                            chunk_size=S)
    assert torch.equal(host, base.cpu())
    if S == 333:
        assert_layer_close(out, _oracle(cpu), "chunk_size=333")


def test_forward_chunk_invariance_many_N(moe):
    cfg = CONFIGS["edge"]
    gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
    base = _run(moe, gpu, 0)  # 0 = unsplit
    for N in (1, 2, 3, 5, 7, 8, 16, 64, 999, 1000, 1001, 4096):
        assert torch.equal(_run(moe, gpu, N), base), f"N={N}"


def test_forward_repeatable(moe):
    cfg = CONFIGS["tiny"]
    gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
    a = _run(moe, gpu, 2)
    b = _run(moe, gpu, 2)
    assert torch.equal(a, b)


def test_forward_identity_like_experts_closed_form(moe):
    """W_gate[e] = W_up[e] = [I_H; 0], W_down[e] = 2^-e [I_H 0]:
    out[t] = bf16( sum_j w[t,j] 2^-idx[t,j] * x * silu(x) )  (tiny layer shape, I >= H)."""
    cfg = CONFIGS["tiny"]
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    idx, w = routing(cfg)
    x = hidden(T, H)
    eye = torch.eye(H)
    wgu = torch.zeros((E, 2 * I, H))
    wd = torch.zeros((E, H, I))
    for e in range(E):
        wgu[e, :H] = eye
        wgu[e, I:I + H] = eye
        wd[e, :, :H] = eye * 2.0 ** -e
    gpu = dict(hidden=x.cuda(), idx=torch.from_numpy(idx).cuda(), w=torch.from_numpy(w).cuda(),
               wgu=wgu.to(torch.bfloat16).cuda(), wd=wd.to(torch.bfloat16).cuda())
    xd = x.double().numpy()
    scale = (w.astype(np.float64) * 2.0 ** -idx.astype(np.float64)).sum(1, keepdims=True)
    ref = scale * xd * xd / (1 + np.exp(-xd))
    for N in (1, 2):
        assert_layer_close(_run(moe, gpu, N), ref, f"identity-like N={N}")


def test_forward_equal_experts_is_dense_ffn(moe):
    """All experts equal and weights summing to 1: the layer equals the dense FFN."""
    cfg = CONFIGS["tiny"]
    cpu = layer_inputs(cfg)
    cpu["wgu"] = cpu["wgu"][:1].repeat(cfg.E, 1, 1).contiguous()
    cpu["wd"] = cpu["wd"][:1].repeat(cfg.E, 1, 1).contiguous()
    gpu = {k: v.cuda() for k, v in cpu.items()}
    dense = oracle.forward(bits(cpu["hidden"]), np.zeros((cfg.T, 1), np.int32),
                           np.ones((cfg.T, 1), np.float32), bits(cpu["wgu"][:1]),
                           bits(cpu["wd"][:1]))
    for N in (1, 2):
        assert_layer_close(_run(moe, gpu, N), dense, f"equal experts N={N}")


def _sampled_tokens(T, n, seed=0):
    rng = np.random.default_rng(seed)
    toks = rng.choice(T, size=min(n, T), replace=False)
    toks[:2] = [0, T - 1]  # first and last token always
    return np.sort(toks)


def _boundary_tokens(idx, chunk_counts, tile=128):
    """Tokens at the seams the chunking introduces: the first and last token of every chunk
    and of every pair of chunks (2m, 2m+1) for each chunk count, and, per pair of the
    largest chunk count, tokens whose rows land in the last (partial) 128-row tile of the
    most- and the least-loaded expert of that pair.  Rows of one expert inside a pair are
    in flat (t, j) order, so the r-th copy of expert e in the pair's range is row r."""
    T, k = idx.shape
    out = set()
    for N in chunk_counts:
        b = oracle.chunk_bounds(T, N)
        for c in range(N):
            if b[c + 1] > b[c]:
                out.update((int(b[c]), int(b[c + 1]) - 1))
        for m in range(0, N, 2):
            lo, hi = int(b[m]), int(b[min(m + 2, N)])
            if hi > lo:
                out.update((lo, hi - 1))
    N = max(chunk_counts)
    b = oracle.chunk_bounds(T, N)
    for m in range(0, N, 2):
        lo, hi = int(b[m]), int(b[min(m + 2, N)])
        flat = idx[lo:hi].reshape(-1)
        counts = np.bincount(flat, minlength=int(idx.max()) + 1)
        live = np.nonzero(counts)[0]
        if live.size == 0:
            continue
        for e in (live[np.argmax(counts[live])], live[np.argmin(counts[live])]):
            pos = np.nonzero(flat == e)[0]
            last = pos[((len(pos) - 1) // tile) * tile:]  # rows of the expert's last tile
            out.update((lo + int(last[0]) // k, lo + int(last[-1]) // k))
    return out


@pytest.mark.parametrize("name,n_tok", [("qwen3", 48), ("mixtral", 64), ("deepseek", 12)])
def test_forward_full_size_sampled(moe, name, n_tok):
    """Full-size layers, every chunk count of the configuration and both dispatches: a
    seeded token sample plus the tokens at every chunk and pair boundary and in the partial
    last row tiles of the most- and least-loaded experts are compared with the oracle one
    by one; the whole output is bit-identical across chunk counts and dispatches."""
    cfg = CONFIGS[name]
    idx, w = routing(cfg)
    x = hidden(cfg.T, cfg.H)
    toks = np.array(sorted(set(_sampled_tokens(cfg.T, n_tok).tolist())
                           | _boundary_tokens(idx, cfg.chunks)), np.int64)
    used = sorted(set(idx[toks].reshape(-1).tolist()))
@pytest.mark.parametrize("E,k,T,H,I", [(1024, 8, 1536, 128, 128),   # MOE_MAX_EXPERTS
                                       (64, 32, 600, 256, 192),     # MOE_MAX_TOPK
                                       (1, 1, 300, 64, 64),         # one expert, top-1
                                       (16, 4, 257, 136, 200),      # H, I not multiples of 64
                                       (16, 4, 300, 776, 200)])     # 3 down column tiles,
                                                                    # the last one partial
def test_forward_limits_and_odd_shapes(moe, E, k, T, H, I):
    """The kernels' table and tile limits: the most experts and the largest top-k the ABI
    takes, a single expert, and widths that are multiples of 8 but not of the 64-wide K
    block or the 128-wide column tiles (the K tail reads zeros, the column tail is never
    written), every dispatch, several chunk counts; every element against the oracle."""
    cfg = LayerConfig("limits", T, H, E, k, I, "normal")
    cpu = layer_inputs(cfg)
    gpu = {kk: v.cuda() for kk, v in cpu.items()}
    ref = _oracle(cpu)
    base = None
    for N in (1, 3, 4):
        for dispatch in ("separate", "fused"):
            out = _run(moe, gpu, N, 1, dispatch)
            assert_layer_close(out, ref, f"E={E} k={k} H={H} I={I} N={N} {dispatch}")
            if base is None:
                base = out
            assert torch.equal(out, base), f"N={N} {dispatch} differs"
