"""Benchmark of the chunked MoE layer on B200.

One step = one moe_forward call over one batch of synthetic input: metadata for all
chunks + the single device-to-host copy, then the chunks' dispatch (a permute kernel, or
row gathers inside the gate/up GEMM), gate/up GEMM with SwiGLU, down GEMM and weighted
unpermute, as the two-stream pair pipeline (with the fused dispatch one GEMM sweep per
pair of chunks).  `--pass backward` times moe_backward instead, `--pass train` a forward
and a backward per step.

Prints ONE JSON line (rank 0).  `value` is tokens/s of the whole job with inputs resident
in HBM; `e2e` is the same metric through the public call with the step's inputs copied
from pinned host memory and its output copied back inside the timed region.
`--impl reference` times the CPU oracle on the same workload instead (a bounded token
sample per step).  Multi-GPU runs are independent replicas (the path has no exchange).
"""
import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
for p in (ROOT, os.path.join(ROOT, "tests")):
    if p not in sys.path:
        sys.path.insert(0, p)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from gen import CONFIGS, expert_weights, hidden as gen_hidden, routing  # noqa: E402

METRIC = "MoE fwd tokens/s; grouped-GEMM TFLOP/s and permute GB/s vs B200 peak"
METRIC_BWD = "MoE bwd tokens/s (expert computation recomputed per chunk)"
METRIC_TRAIN = "MoE fwd+bwd tokens/s (expert computation recomputed per chunk)"
DEFAULT_CONFIG = "qwen3"
DEFAULT_CHUNKS = 4
GEMM_SRC = os.path.join(ROOT, "expert_router_top_b200", "csrc", "gemm.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gateup_traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def workload_name(cfg):
    name = {"qwen3": "qwen3-30b-a3b-shaped layer, one 16k packed sequence",
            "mixtral": "mixtral-8x7b-shaped layer", "deepseek": "deepseek-v3-shaped routed layer",
            "tiny": "tiny layer", "edge": "edge-case layer"}.get(cfg.name, cfg.name)
    if cfg.name in CONFIGS and cfg.T != CONFIGS[cfg.name].T:
        name += f" (token count overridden: {cfg.T})"
    return name


# The profiling recipe's fallback: sustained bf16 settles near 1.4 PFLOP/s at about 1.3 GHz
# under the power cap; the burst figure's clock is taken as the maximum SM clock.
FALLBACK_SUSTAINED_MHZ = 1300.0


def _clock_keys(d, prefix=""):
    """(dotted key, value) of every numeric entry of a nested dict whose key names a clock."""
    out = []
    for k, v in d.items():
        key = f"{prefix}{k}"
        if isinstance(v, dict):
            out += _clock_keys(v, key + ".")
        elif isinstance(v, (int, float)) and ("mhz" in k.lower() or "clock" in k.lower()):
            out.append((key, float(v)))
    return out


def load_peaks():
    """The roofline denominators: MEASURED_PEAKS.json (driver-written) or the recipe's
    fallback, plus the SM clock each bf16 figure was measured at when the file records it
    ("sustained_mhz" / "burst_mhz" below; None = unknown)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        peaks = {k: float(d[k]) for k in FALLBACK_PEAKS}
        clocks = _clock_keys(d)
        sus = [v for k, v in clocks if "sustain" in k.lower() and "max" not in k.lower()]
        bur = [v for k, v in clocks if "sustain" not in k.lower() and "max" not in k.lower()
               and ("burst" in k.lower() or "bf16" in k.lower())]
        peaks["sustained_mhz"] = sus[0] if sus else None
        peaks["burst_mhz"] = bur[0] if bur else None
        peaks["clock_keys"] = [k for k, _ in clocks]
        return peaks, "measured"
    peaks = dict(FALLBACK_PEAKS, sustained_mhz=FALLBACK_SUSTAINED_MHZ, burst_mhz=None,
                 clock_keys=[])
    return peaks, "fallback"


def max_over_ranks(ms, dist_mod=None, device="cpu"):
    """The slowest rank's time: every multi-GPU number is the max over ranks."""
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if dist_mod is not None:
        dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, tokens_per_rank, steps, ms_max):
    """Whole-job throughput: the tokens all replicas processed / the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms_max / 1e3)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, read through NVML every 5 ms by a
    background thread (nvidia-smi every 50 ms if NVML is unavailable), each sample stamped
    with its host time so that a summary covers exactly one timed region.  Read-only: it
    changes no setting of the GPU."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, gpu_index, period_s=0.005):
        self.gpu = gpu_index
        self.period = period_s
        self.samples = []  # (host time, sm MHz, max sm MHz, reasons set)
        self.proc = None
        self.thread = None
        self.nvml = None
        self.source = None
        self._stop = threading.Event()

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:  # noqa: BLE001 - fall back to the NVML index
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        return pynvml, h

    def start(self):
        try:
            self.nvml = self._nvml_handle()
            self.source = "nvml"
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
            self.thread.start()
            return
        except Exception:  # noqa: BLE001 - no NVML: sample through nvidia-smi
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.source = "nvidia-smi"
        self.thread = threading.Thread(target=self._read_smi, daemon=True)
        self.thread.start()

    def _poll_nvml(self):
        nv, h = self.nvml
        smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                              getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
        while not self._stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                bits = int(get_reasons(h)) if get_reasons else 0
            except Exception:  # noqa: BLE001 - a failed read is skipped
                time.sleep(self.period)
                continue
            reasons = {n for n, b in self.REASON_BITS.items() if bits & b}
            self.samples.append((time.perf_counter(), sm, smax, reasons))
            time.sleep(self.period)

    def _read_smi(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.proc.stdout:
            f = [x.strip() for x in line.strip().split(",")]
            if len(f) < 9:
                continue
            try:
                sm, smax = float(f[1]), float(f[2])
            except ValueError:
                continue
            reasons = {n for n, v in zip(names, f[5:9]) if v.lower() == "active"}
            self.samples.append((time.perf_counter(), sm, smax, reasons))

    def summary(self, t0=None, t1=None, min_samples=3, widen_to=None):
        """Median SM clock, max clock and the reasons seen in the samples taken in [t0, t1]
        (host perf_counter times of a timed region).  With fewer than min_samples there,
        the window is widened back to widen_to (the start of the untimed steps that ran
        just before at the same load) and the summary says so."""
        pts = list(self.samples)
        window = "all"
        if t0 is not None:
            sel = [x for x in pts if t0 <= x[0] <= t1 + self.period]
            window = "timed region"
            if len(sel) < min_samples and widen_to is not None:
                sel = [x for x in pts if widen_to <= x[0] <= t1 + self.period]
                window = "timed region and the untimed steps just before it"
            pts = sel
        if not pts:
            return None
        reasons = set()
        for x in pts:
            reasons |= x[3]
        return {"sm_mhz": statistics.median(x[1] for x in pts), "sm_max_mhz": pts[-1][2],
                "sm_mhz_min": min(x[1] for x in pts), "reasons": sorted(reasons),
                "samples": len(pts), "window": window, "source": self.source}

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        if self.nvml is not None:
            try:
                self.nvml[0].nvmlShutdown()
            except Exception:  # noqa: BLE001
                pass


def spin_up(step, seconds=0.5):
    """Run `step` untimed for `seconds` of device time so that the SM clocks have left their
    idle state before the warm-up and timed steps; returns the number of calls."""
    n, t_end = 0, time.perf_counter() + seconds
    while time.perf_counter() < t_end:
        step()
        n += 1
        if n % 8 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    return n


# ---------------------------------------------------------------------- workload

def make_inputs(cfg, device, seed=0, weights=True):
    idx, w = routing(cfg, seed)
    x = gen_hidden(cfg.T, cfg.H, seed)
    out = dict(hidden=x.to(device), idx=torch.from_numpy(idx).to(device),
               w=torch.from_numpy(w).to(device), hidden_cpu=x, idx_cpu=idx, w_cpu=w)
    if weights:
        out["wgu"], out["wd"] = expert_weights(cfg.E, cfg.H, cfg.I, seed, device=device)
    return out


def algorithmic_units(cfg, counts, n_live, dispatch="separate", pair_gemms=False):
    """Per-kernel algorithmic work of one step (bytes or flops), from the chunk counts.
    With the fused dispatch the gate/up GEMM reads each token row of `hidden` (T rows)
    instead of the T*k permuted rows, and with pair GEMMs each GEMM launch serves the two
    chunks of a pair, so an expert's weights are streamed once per pair."""
    H, I, k, T = cfg.H, cfg.I, cfg.k, cfg.T
    rows = int(counts.sum())
    if pair_gemms:
        counts = np.stack([counts[i:i + 2].sum(0) for i in range(0, counts.shape[0], 2)])
    active = int((counts > 0).sum())  # (launch, expert) pairs with rows: weights streamed
    return {
        # permute: read T rows once, write T*k rows, plus the k destination indices per token
        "permute_bytes": (T + rows) * H * 2 + rows * 4,
        # unpermute: read T*k rows and their weights and indices, write T rows
        "unpermute_bytes": (rows + T) * H * 2 + rows * 8,
        "gateup_flops": 4.0 * rows * H * I,
        "down_flops": 2.0 * rows * H * I,
        # weights of every active expert, re-read once per chunk (the method's N-fold stream)
        "gateup_weight_bytes": active * 2 * I * H * 2,
        "down_weight_bytes": active * H * I * 2,
        # gate/up kernel, whole step: W_gate_up of each chunk's active experts (re-read per
        # chunk), permuted rows read, Act written
        "gateup_alg_bytes": active * 2 * I * H * 2 + (T if dispatch == "fused" else rows) * H * 2
        + rows * I * 2,
    }


def gemm_src_hash():
    with open(GEMM_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_per_launch(cfg_name, chunks, dispatch, pair_gemms=False):
    """DRAM bytes per gate/up launch from the committed ncu summary, if it was taken on
    the current kernel source, this workload, this chunking and this dispatch; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    if (d.get("gemm_src_sha256_16") != gemm_src_hash() or d.get("num_chunks") != chunks
            or d.get("config") != cfg_name or d.get("dispatch") != dispatch
            or bool(d.get("pair_gemms", False)) != pair_gemms):
        return None
    return d.get("dram_bytes_per_launch_full_size")


# ------------------------------------------------------------------------- oracle arm

def oracle_tokens_per_s(cfg, inputs, budget_s, sample_seed=0, max_tokens=None, seed=0,
                        kind="forward"):
    """Oracle throughput on a bounded, seeded sample of the workload's tokens.

    kind: "forward", "backward" (gradients of sum(out * d_out)) or "train" (both).
    Draws the weights of the sampled tokens' experts on the host; returns
    (tokens/s, tokens, seconds, threads)."""
    import oracle
    from gen import bits, expert_down, expert_gate_up

    rng = np.random.default_rng(1000 + sample_seed)
    idx, w = inputs["idx_cpu"], inputs["w_cpu"]
    xb = bits(inputs["hidden_cpu"])

    def run(n):
        toks = np.sort(rng.choice(cfg.T, size=n, replace=False))
        used = sorted(set(idx[toks].reshape(-1).tolist()))
        remap = {e: i for i, e in enumerate(used)}
        sidx = np.vectorize(remap.get)(idx[toks]).astype(np.int32)
        wgu = np.stack([bits(expert_gate_up(e, cfg.H, cfg.I, seed)) for e in used])
        wd = np.stack([bits(expert_down(e, cfg.H, cfg.I, seed)) for e in used])
        dout = bits(gen_hidden(n, cfg.H, 50 + sample_seed)) if kind != "forward" else None
        t0 = time.perf_counter()
        if kind != "backward":
            oracle.forward(xb[toks], sidx, w[toks], wgu, wd)
        if kind != "forward":
            oracle.backward(xb[toks], sidx, w[toks], wgu, wd, dout)
        return time.perf_counter() - t0

    threads = oracle.max_threads()
    n = max(1, min(threads, cfg.T))
    dt = run(n)
    per_tok = dt / n
    target = int(budget_s / max(per_tok, 1e-9))
    n2 = max(n, min(cfg.T, target, max_tokens or cfg.T))
    if n2 > n:
        n, dt = n2, run(n2)
    return n / dt, n, dt, threads


def run_reference(args, cfg):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    inputs = make_inputs(cfg, device="cpu", weights=False)
    per_step = max(1.0, 150.0 / (args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_tokens_per_s(cfg, inputs, per_step / 4, max_tokens=64)
    total_tok, total_s, threads, toks = 0, 0.0, 1, 0
    for i in range(args.steps):
        tps, toks, dt, threads = oracle_tokens_per_s(cfg, inputs, per_step, sample_seed=i)
        total_tok += toks
        total_s += dt
    value = total_tok / total_s
    sample = (f"{args.steps} steps, each a seeded sample of ~{toks} of the {cfg.T} tokens "
              f"(all k={cfg.k} experts per token, fp64), ~{per_step:.0f} s each")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(cfg, args.chunks, args.dispatch),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(cfg, chunks, dispatch="auto"):
    """The workload as both arms print it: the requested dispatch ("auto" = the library's
    own choice for the shape; the line's top-level `dispatch_resolved` says which ran)."""
    wbytes = 6 * cfg.E * cfg.H * cfg.I
    return {"workload": workload_name(cfg), "T": cfg.T, "H": cfg.H, "E": cfg.E, "k": cfg.k,
            "I": cfg.I, "ep_groups": cfg.G, "num_chunks": chunks, "dispatch": dispatch,
            "routing": cfg.routing,
            "ffn": "SwiGLU", "parallelism": "replicas",
            "l2": f"inputs larger than L2 ({wbytes / 1e9:.2f} GB of expert weights read per step)"}


def tensor_peak(peaks, clk):
    """bf16 tensor roof of a launch at the SM clock sampled while it ran: the measured cuBLAS
    throughput at that clock, i.e. the sustained figure scaled linearly from the clock it was
    measured at, capped by the burst figure (which also bounds it at the burst figure's own
    clock).  A GEMM under the 1 kW power cap runs near 1.3-1.5 GHz, where the burst figure
    scaled by (clock / max clock) would understate what cuBLAS reaches there.  Without a
    clock sample: the burst figure.  Returns (peak TFLOP/s, peak / burst)."""
    burst = peaks["bf16_tflops"]
    f = clk.get("sm_mhz") if clk else None
    if not f:
        return burst, 1.0
    fmax = clk.get("sm_max_mhz") or f
    cands = [burst * f / (peaks.get("burst_mhz") or fmax)]
    if peaks.get("sustained_mhz"):
        cands.append(peaks["bf16_tflops_sustained"] * f / peaks["sustained_mhz"])
    roof = min(burst, max(cands))
    return roof, roof / burst


def kernel_rates(prof, units, steps):
    """Per-kind launches and times of `steps` steps, with each GEMM kind's TFLOP/s and each
    row kernel's GB/s from the algorithmic work of one step."""
    kinds = {}
    for kind in ("metadata", "permute", "gateup", "down", "unpermute"):
        p = prof[kind]
        kinds[kind] = dict(launches=p["launches"], ms=p["ms"],
                           ms_per_step=p["ms"] / steps if steps else 0.0)

    def rate(work, ms, scale):
        return work * steps / (ms / 1e3) / scale if ms > 0 else 0.0

    kinds["gateup"]["tflops"] = rate(units["gateup_flops"], prof["gateup"]["ms"], 1e12)
    kinds["down"]["tflops"] = rate(units["down_flops"], prof["down"]["ms"], 1e12)
    kinds["permute"]["gbs"] = rate(units["permute_bytes"], prof["permute"]["ms"], 1e9)
    kinds["unpermute"]["gbs"] = rate(units["unpermute_bytes"], prof["unpermute"]["ms"], 1e9)
    gm = prof["gateup"]["ms"] + prof["down"]["ms"]
    kinds["grouped_gemm_tflops"] = rate(units["gateup_flops"] + units["down_flops"], gm, 1e12)
    return kinds


# ------------------------------------------------------------------------- our arm

L2_FLUSH_BYTES = 512 << 20  # written before each cold launch: 4x the B200's 126 MB of L2


def row_kernels_cold(moe, cfg, inp, dev, stream, reps):
    """permute and unpermute of the whole layer as one chunk, called through their stage
    entry points (the kernels the separate dispatch launches), each launch preceded by a
    512 MB write on the same stream: the data starts cold in HBM, and the start event
    fires when that write ends, so no host launch latency falls inside the interval.
    Median over `reps` launches; GB/s from the algorithmic bytes."""
    meta = moe.metadata(inp["idx"], cfg.E, cfg.G, 1, with_permutation=True)
    dst = meta["dst"]
    X = torch.empty((cfg.T * cfg.k, cfg.H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def cold(fn):
        ts = []
        for _ in range(reps):
            with torch.cuda.stream(stream):
                flush.fill_(1)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            stream.synchronize()
            ts.append(a.elapsed_time(b))
        return float(np.median(ts))

    moe.permute(inp["hidden"], dst, cfg.k, X=X, stream=stream)  # warm-up (and X's contents)
    ms_p = cold(lambda: moe.permute(inp["hidden"], dst, cfg.k, X=X, stream=stream))
    ms_u = cold(lambda: moe.unpermute(X, dst, inp["w"], cfg.k, out=out, stream=stream))
    rows = cfg.T * cfg.k
    pb = (cfg.T + rows) * cfg.H * 2 + rows * 4
    ub = (cfg.T + rows) * cfg.H * 2 + rows * 8
    del X, out, flush
    return {"permute_ms": ms_p, "unpermute_ms": ms_u, "permute_bytes": pb, "unpermute_bytes": ub,
            "permute_gbs": pb / (ms_p / 1e3) / 1e9, "unpermute_gbs": ub / (ms_u / 1e3) / 1e9}

def time_steps(moe, inp, cfg, chunks, ws, steps, stream, dispatch="auto", pair_gemms=True):
    """Device time of `steps` back-to-back forward calls, ms (CUDA events on `stream`)."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(steps):
        moe.forward(inp["hidden"], inp["idx"], inp["w"], inp["wgu"], inp["wd"],
                    num_chunks=chunks, ep_groups=cfg.G, out=out, workspace=ws, stream=stream,
                    dispatch=dispatch, pair_gemms=pair_gemms)
    end.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(end), out


class Runner:
    """One workload on one GPU: times moe_forward at a given chunk count and dispatch with
    the library's per-launch events on, with the clock samples of exactly that region."""

    def __init__(self, moe, cfg, inp, dev, stream, clocks, pg=None):
        self.moe, self.cfg, self.inp, self.dev, self.stream = moe, cfg, inp, dev, stream
        self.clocks, self.pg = clocks, pg

    def workspace(self, chunks):
        c = self.cfg
        return self.moe.alloc_workspace(
            self.moe.workspace_bytes(c.T, c.H, c.I, c.E, c.k, c.G, chunks), self.dev)

    def resolve(self, chunks, dispatch, per_chunk_gemms=False):
        c = self.cfg
        d = self.moe.forward_dispatch(c.T, c.H, c.I, c.E, c.k, dispatch, c.G, chunks)
        return d, d == "fused" and not per_chunk_gemms

    def measure(self, chunks, dispatch, steps, warmup, per_chunk_gemms=False, spin_s=0.3):
        moe, c, inp = self.moe, self.cfg, self.inp
        ws = self.workspace(chunks)
        resolved, pair = self.resolve(chunks, dispatch, per_chunk_gemms)
        meta = moe.metadata(inp["idx"], c.E, c.G, chunks)
        n_live = int((np.diff(meta["bounds"]) > 0).sum())
        units = algorithmic_units(c, meta["counts"], n_live, resolved, pair)

        def step():
            moe.forward(inp["hidden"], inp["idx"], inp["w"], inp["wgu"], inp["wd"],
                        num_chunks=chunks, ep_groups=c.G, workspace=ws, dispatch=dispatch,
                        pair_gemms=not per_chunk_gemms)

        t_load = time.perf_counter()
        spin = spin_up(step, spin_s)
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        if self.pg:
            self.pg.barrier()
        torch.cuda.synchronize()
        moe.profile_enable(True)
        t0 = time.perf_counter()
        ms, _ = time_steps(moe, inp, c, chunks, ws, steps, self.stream, dispatch,
                           not per_chunk_gemms)
        t1 = time.perf_counter()
        if self.pg:
            self.pg.barrier()
        prof = moe.profile_read()
        moe.profile_enable(False)
        clk = self.clocks.summary(t0, t1, widen_to=t_load) if self.clocks else None
        del ws
        return dict(ms=ms, ms_per_step=ms / steps, steps=steps, prof=prof, clk=clk,
                    units=units, meta=meta, n_live=n_live, dispatch=resolved, pair_gemms=pair,
                    spinup_steps=spin,
                    kinds=kernel_rates(prof, units, steps))

    def timeline(self, chunks, dispatch, calls=3):
        """Launch records of the last of `calls` back-to-back forward calls, times relative
        to that call's first launch."""
        moe, c, inp = self.moe, self.cfg, self.inp
        ws = self.workspace(chunks)
        resolved, pair = self.resolve(chunks, dispatch)
        for _ in range(3):
            moe.forward(inp["hidden"], inp["idx"], inp["w"], inp["wgu"], inp["wd"],
                        num_chunks=chunks, ep_groups=c.G, workspace=ws, dispatch=dispatch)
        torch.cuda.synchronize()
        moe.profile_enable(True)
        for _ in range(calls):
            moe.forward(inp["hidden"], inp["idx"], inp["w"], inp["wgu"], inp["wd"],
                        num_chunks=chunks, ep_groups=c.G, workspace=ws, dispatch=dispatch)
        recs = [r for r in moe.profile_timeline() if r["call"] == calls]
        moe.profile_enable(False)
        del ws
        t0 = min(r["start_ms"] for r in recs) if recs else 0.0
        for r in recs:
            r["start_ms"] = round(r["start_ms"] - t0, 4)
            r["end_ms"] = round(r["end_ms"] - t0, 4)
        return {"num_chunks": chunks, "dispatch": resolved,
                "gemm_sweep": "per pair of chunks" if pair and chunks > 1 else "per chunk",
                "step_ms": max((r["end_ms"] for r in recs), default=0.0), "launches": recs}


def gemm_roofline(m, peaks, peak_src):
    """Roofline object of the gate/up GEMM (the dominant kernel) for one measurement: per
    launch algorithmic flops and bytes over its event time; the tensor roof is the measured
    burst bf16 figure scaled to the clock sampled during the timed region."""
    units, g, steps = m["units"], m["prof"]["gateup"], m["steps"]
    n_gu = max(1, g["launches"] // max(1, steps))
    flops_l = units["gateup_flops"] / n_gu
    bytes_l = units["gateup_alg_bytes"] / n_gu
    t_l = g["ms"] / max(1, g["launches"]) / 1e3  # s per launch
    peak_tc, scale = tensor_peak(peaks, m["clk"])
    peak_bw = peaks["hbm_gbs"]
    t_tensor = flops_l / (peak_tc * 1e12)
    t_mem = bytes_l / (peak_bw * 1e9)
    if t_mem > t_tensor:
        r = {"bound": "hbm", "achieved": bytes_l / t_l / 1e9 if t_l else 0.0, "peak": peak_bw,
             "unit": "GB/s"}
    else:
        r = {"bound": "tensor", "achieved": flops_l / t_l / 1e12 if t_l else 0.0,
             "peak": peak_tc, "unit": "TFLOP/s"}
    r["frac"] = r["achieved"] / r["peak"]
    tf = flops_l / t_l / 1e12 if t_l else 0.0
    r.update({
        "kernel": "grouped_gemm_kernel<gate/up + SwiGLU" +
                  (", gathered A rows" if m["dispatch"] == "fused" else "") + "> (tcgen05)",
        "peak_source": f"{peak_src}: min(bf16_tflops, bf16_tflops_sustained x sampled SM MHz / "
                       f"its measurement MHz) = {scale:.3f} x bf16_tflops; HBM copy hbm_gbs",
        "clock_scale": scale,
        "per_launch": {"flops": flops_l, "bytes": bytes_l, "ms": t_l * 1e3,
                       "roofline_ms": max(t_tensor, t_mem) * 1e3},
        "frac_of_roofline_time": max(t_tensor, t_mem) / t_l if t_l else None,
        "tensor_frac_of_burst": tf / peaks["bf16_tflops"],
        "tensor_frac_of_sustained": tf / peaks["bf16_tflops_sustained"],
        "tensor_frac_of_burst_x_clock_ratio":
            tf / (peaks["bf16_tflops"] * m["clk"]["sm_mhz"] / m["clk"]["sm_max_mhz"])
            if m["clk"] and m["clk"].get("sm_mhz") and m["clk"].get("sm_max_mhz") else None,
        "hbm_frac": bytes_l / t_l / 1e9 / peak_bw if t_l else None})
    return r


def per_n_entry(moe, cfg, m, peaks):
    k = m["kinds"]
    peak_tc, _ = tensor_peak(peaks, m["clk"])
    e = {"ms_per_step": m["ms_per_step"], "tokens_per_s": cfg.T / (m["ms_per_step"] / 1e3),
         "dispatch": m["dispatch"],
         "gemm_sweep": "per pair of chunks" if m["pair_gemms"] and m["n_live"] > 1
         else "per chunk",
         "gateup_tflops": k["gateup"]["tflops"], "down_tflops": k["down"]["tflops"],
         "grouped_gemm_tflops": k["grouped_gemm_tflops"],
         "gateup_frac_of_tensor_roof": k["gateup"]["tflops"] / peak_tc,
         "gateup_frac_of_burst": k["gateup"]["tflops"] / peaks["bf16_tflops"],
         "unpermute_ms_per_step": k["unpermute"]["ms_per_step"],
         "gemm_ms_per_step": k["gateup"]["ms_per_step"] + k["down"]["ms_per_step"],
         "workspace_bytes": moe.workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.G,
                                                m["meta"]["counts"].shape[0]),
         "clocks": m["clk"]}
    if cfg.G > 1:
        e["send_splits"] = m["meta"]["send"].tolist()
    return e


def run_ours(args, cfg):
    import expert_router_top_b200 as moe

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist
    moe.load()
    dev = torch.device("cuda", local)
    inp = make_inputs(cfg, dev)
    chunks = args.chunks
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    run = Runner(moe, cfg, inp, dev, stream, clocks, pg)
    peaks, peak_src = load_peaks()

    # ---- the headline: K timed steps at the requested chunk count and dispatch
    head = run.measure(chunks, args.dispatch, args.steps, args.warmup, args.per_chunk_gemms,
                       spin_s=args.spinup_s)
    ms_max = max_over_ranks(head["ms"], pg, dev)
    ms_per_step = ms_max / args.steps
    value = job_tokens_per_s(world, cfg.T, args.steps, ms_max)
    units, kinds = head["units"], head["kinds"]
    weight_stream = float(units["gateup_weight_bytes"] + units["down_weight_bytes"])

    # ---- end to end through the public call, host buffers, copies inside the region
    ws = run.workspace(chunks)
    e2e = run_e2e(moe, inp, cfg, chunks, ws, args, stream, dev, pg, world)
    del ws

    roofline = gemm_roofline(head, peaks, peak_src)
    roofline["traffic"] = traffic_per_launch(cfg.name, chunks, head["dispatch"],
                                             head["pair_gemms"])

    per_n, isolated, timelines = {}, None, None
    if not args.headline_only:
        # ---- the same workload at N = 1, 2, 4 (the library's own dispatch choice each),
        # each after the same spin-up as the headline, so that every region runs at the
        # power-capped clock of sustained work (after a short one the clock is still high)
        for n in args.per_n:
            m = head if (n == chunks and args.dispatch == "auto" and not args.per_chunk_gemms) \
                else run.measure(n, "auto", args.steps, args.warmup, spin_s=args.spinup_s)
            per_n[str(n)] = per_n_entry(moe, cfg, m, peaks)
        # ---- permute and unpermute alone: cold-cache launches of the kernels, and the
        # same kernels inside an exposed step (separate dispatch, one chunk)
        cold = row_kernels_cold(moe, cfg, inp, dev, stream, max(args.steps, 5))
        iso = run.measure(1, "separate", args.steps, args.warmup)
        ik = iso["kinds"]
        isolated = {
            "permute_gbs": cold["permute_gbs"],
            "permute_frac_of_hbm": cold["permute_gbs"] / peaks["hbm_gbs"],
            "unpermute_gbs": cold["unpermute_gbs"],
            "unpermute_frac_of_hbm": cold["unpermute_gbs"] / peaks["hbm_gbs"],
            "permute_ms": cold["permute_ms"], "unpermute_ms": cold["unpermute_ms"],
            "permute_bytes": cold["permute_bytes"], "unpermute_bytes": cold["unpermute_bytes"],
            "how": "the whole layer as one chunk through the stage entry points (the kernels the "
                   "separate dispatch launches), each launch after a 512 MB write on its stream "
                   "(cold L2; the start event fires when the write ends); median of "
                   f"{max(args.steps, 5)} launches; bytes = (T + T*k)*H*2 + 4 (permute) or 8 "
                   "(unpermute) bytes per (t, j)",
            "in_step": {
                "permute_gbs": ik["permute"]["gbs"], "unpermute_gbs": ik["unpermute"]["gbs"],
                "how": "num_chunks=1, separate dispatch, events around each launch inside the "
                       "step: the permute's interval also holds the launch latency after the "
                       "metadata's host copy (the GPU is idle when its start event is recorded)",
                "ms_per_step": iso["ms_per_step"], "clocks": iso["clk"]}}
        if args.timeline:
            timelines = [run.timeline(chunks, "auto"), run.timeline(1, "auto"),
                         run.timeline(chunks, "separate")]
            with open(args.timeline, "w") as f:
                json.dump({"workload": workload_name(cfg), "config": config_block(cfg, chunks),
                           "timelines": timelines}, f, indent=1)
    if clocks:
        clocks.stop()
        if args.clock_trace:
            with open(args.clock_trace, "w") as f:
                json.dump([(round(t - clocks.samples[0][0], 4), mhz, sorted(r))
                           for t, mhz, _, r in clocks.samples], f)

    ms_n1 = per_n.get("1", {}).get("ms_per_step")
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; random-init expert weights of the layer's shape)",
        "config": config_block(cfg, chunks, args.dispatch),
        "dispatch_resolved": head["dispatch"],
        "gemm_sweep": "per pair of chunks" if head["pair_gemms"] and head["n_live"] > 1
        else "per chunk",
        "roofline": roofline,
        "grouped_gemm_tflops": kinds["grouped_gemm_tflops"],
        "grouped_gemm_frac_of_tensor_roof":
            kinds["grouped_gemm_tflops"] / tensor_peak(peaks, head["clk"])[0],
        "grouped_gemm_frac_of_burst": kinds["grouped_gemm_tflops"] / peaks["bf16_tflops"],
        "permute_gbs": kinds["permute"]["gbs"],
        "permute_frac_of_hbm": kinds["permute"]["gbs"] / peaks["hbm_gbs"],
        "unpermute_gbs": kinds["unpermute"]["gbs"],
        "unpermute_frac_of_hbm": kinds["unpermute"]["gbs"] / peaks["hbm_gbs"],
        "row_kernels_isolated": isolated,
        "kernels": {k2: v for k2, v in kinds.items() if isinstance(v, dict)},
        "weight_bytes_streamed_per_step": weight_stream,
        "workspace_bytes": {str(n): moe.workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.G,
                                                        n) for n in (1, 2, 4)},
        "per_n": per_n or None,
        "ms_per_step_num_chunks_1": ms_n1,
        "send_splits": head["meta"]["send"].tolist() if cfg.G > 1 else None,
        "gpu_launches": int(head["prof"]["kernels"]),
        "spinup_steps": head["spinup_steps"], "spinup_s": args.spinup_s,
        "e2e": e2e,
        "clocks": head["clk"],
        "peaks": dict(peaks, source=peak_src),
    }
    if timelines:
        line["timeline_file"] = args.timeline
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, ntok, dt, threads = oracle_tokens_per_s(cfg, inp, args.cpu_budget_s)
        line["cpu_baseline"] = {
            "value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{ntok} seeded tokens of the {cfg.T}-token workload, all k={cfg.k} "
                      f"experts each, fp64, {dt:.1f} s"}
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def backward_units(cfg, counts):
    """Algorithmic work of one moe_backward call from the chunk counts: flops per GEMM
    kind and the weight-gradient GEMMs' bytes.  The weight gradients run once per pair of
    adjacent chunks (0,1), (2,3), ...: operands are read once; dW is written by the pair in
    which an expert first has rows and read and written by every later pair with its rows."""
    H, I = cfg.H, cfg.I
    rows_c = counts.sum(1).astype(np.float64)
    rows = float(rows_c.sum())
    pairs = np.stack([counts[i:i + 2].sum(0) for i in range(0, counts.shape[0], 2)])
    active = pairs > 0
    seen_before = np.cumsum(active, axis=0) - active  # earlier pairs with rows
    dw_bytes = 12.0 * H * I * (active.sum() + (active & (seen_before > 0)).sum())
    return {
        "flops": {"bwd_gateup": 4 * rows * H * I, "bwd_dswiglu": 2 * rows * H * I,
                  "bwd_dx": 4 * rows * H * I, "bwd_wgrad": 6 * rows * H * I},
        "wgrad_bytes": float((rows_c * (2 * H + 3 * I) * 2).sum()) + dw_bytes,
    }


def run_backward(args, cfg):
    """--pass backward|train: time moe_backward (train: moe_forward then moe_backward) per
    step; the roofline object is for the weight-gradient GEMMs, the largest backward kind."""
    import expert_router_top_b200 as moe

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist
    moe.load()
    dev = torch.device("cuda", local)
    inp = make_inputs(cfg, dev)
    chunks = args.chunks
    train = args.pass_ == "train"
    dout = gen_hidden(cfg.T, cfg.H, 77).to(dev)
    bws = moe.alloc_workspace(moe.backward_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k,
                                                           cfg.G, chunks), dev)
    fws = moe.alloc_workspace(moe.workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.G,
                                                  chunks), dev) if train else None
    stream = torch.cuda.current_stream()
    meta = moe.metadata(inp["idx"], cfg.E, cfg.G, chunks)
    units = backward_units(cfg, meta["counts"])
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    grads = moe.backward_buffers(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, dev)

    def step():
        if train:
            moe.forward(inp["hidden"], inp["idx"], inp["w"], inp["wgu"], inp["wd"],
                        num_chunks=chunks, ep_groups=cfg.G, out=out, workspace=fws,
                        stream=stream)
        moe.backward(inp["hidden"], inp["idx"], inp["w"], inp["wgu"], inp["wd"], dout,
                     num_chunks=chunks, ep_groups=cfg.G, workspace=bws, stream=stream,
                     out=grads)

    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    t_load = time.perf_counter()
    spinup = spin_up(step, args.spinup_s)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    moe.profile_enable(True)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    if pg:
        pg.barrier()
    prof = moe.profile_read()
    moe.profile_enable(False)
    clk = clocks.summary(t0, t1, widen_to=t_load) if clocks else None
    if clocks:
        clocks.stop()
    ms_max = max_over_ranks(start.elapsed_time(end), pg, dev)
    steps = args.steps
    peaks, peak_src = load_peaks()
    kinds = {}
    for kind in moe.KERNEL_KINDS:
        p = prof[kind]
        if not p["launches"]:
            continue
        kinds[kind] = dict(launches=p["launches"], ms_per_step=p["ms"] / steps)
        fl = units["flops"].get(kind)
        if fl and p["ms"] > 0:
            kinds[kind]["tflops"] = fl * steps / (p["ms"] / 1e3) / 1e12
    # roofline of the weight-gradient GEMMs (both launches of every chunk, whole step)
    wg = prof["bwd_wgrad"]
    t = wg["ms"] / steps / 1e3
    f, b = units["flops"]["bwd_wgrad"], units["wgrad_bytes"]
    peak_tc, scale = tensor_peak(peaks, clk)  # burst figure at the sampled clock
    t_tensor, t_mem = f / (peak_tc * 1e12), b / (peaks["hbm_gbs"] * 1e9)
    if t_mem > t_tensor:
        roofline = {"bound": "hbm", "achieved": b / t / 1e9, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s"}
    else:
        roofline = {"bound": "tensor", "achieved": f / t / 1e12, "peak": peak_tc,
                    "unit": "TFLOP/s"}
    roofline["frac"] = roofline["achieved"] / roofline["peak"]
    n_wg = max(1, wg["launches"] // max(1, steps))
    roofline.update({
        "traffic": None,
        "kernel": "bwd_gemm_kernel<weight gradient> (tcgen05, TMA store / add-reduce epilogue)",
        "peak_source": f"{peak_src}: min(bf16_tflops, bf16_tflops_sustained x sampled SM MHz / "
                       f"its measurement MHz) = {scale:.3f} x bf16_tflops; HBM copy hbm_gbs",
        "clock_scale": scale,
        "per_launch": {"flops": f / n_wg, "bytes": b / n_wg, "ms": t * 1e3 / n_wg,
                       "roofline_ms": max(t_tensor, t_mem) * 1e3 / n_wg},
        "tensor_frac_of_burst": f / t / 1e12 / peaks["bf16_tflops"],
        "tensor_frac_of_sustained": f / t / 1e12 / peaks["bf16_tflops_sustained"],
        "hbm_frac": b / t / 1e9 / peaks["hbm_gbs"]})
    gemm_fl = sum(v for k2, v in units["flops"].items())
    gemm_ms = sum(prof[k2]["ms"] for k2 in units["flops"]) / steps
    ws_per_n = {str(n): moe.backward_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.G, n)
                for n in (1, 2, 4)}
    line = {
        "metric": METRIC_TRAIN if train else METRIC_BWD,
        "value": job_tokens_per_s(world, cfg.T, steps, ms_max), "unit": "tokens/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": ms_max / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; random-init expert weights of the layer's shape)",
        "config": dict(config_block(cfg, chunks), **{"pass": args.pass_}),
        "roofline": roofline,
        "grouped_gemm_tflops": gemm_fl / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else None,
        "kernels": kinds,
        "backward_workspace_bytes": ws_per_n,
        "gpu_launches": int(prof["kernels"]),
        "spinup_steps": spinup, "spinup_s": args.spinup_s,
        "e2e": None,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, ntok, dt, threads = oracle_tokens_per_s(cfg, inp, args.cpu_budget_s,
                                                     kind=args.pass_)
        line["cpu_baseline"] = {
            "value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{ntok} seeded tokens of the {cfg.T}-token workload, all k={cfg.k} "
                      f"experts each, fp64 {args.pass_}, {dt:.1f} s"}
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_e2e(moe, inp, cfg, chunks, ws, args, stream, dev, pg, world):
    """The same metric through moe_forward_host: each step copies its hidden rows, routing
    indices and weights from pinned host memory and its output back to pinned host memory
    (per chunk, beside the kernels), all inside the timed region."""
    steps = max(3, min(args.steps, 20))
    h_pin = inp["hidden_cpu"].pin_memory()
    i_pin = torch.from_numpy(inp["idx_cpu"]).pin_memory()
    w_pin = torch.from_numpy(inp["w_cpu"]).pin_memory()
    o_pin = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory()
    wsh = moe.alloc_workspace(
        moe.workspace_bytes_host(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, cfg.G, chunks), dev)

    def step():
        moe.forward_host(h_pin, i_pin, w_pin, inp["wgu"], inp["wd"], num_chunks=chunks,
                         ep_groups=cfg.G, out=o_pin, workspace=wsh, stream=stream)

    step()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        step()
    e.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(s.elapsed_time(e), pg, dev)
    h2d = h_pin.numel() * 2 + i_pin.numel() * 4 + w_pin.numel() * 4
    del wsh
    return {"value": job_tokens_per_s(world, cfg.T, steps, ms), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": o_pin.numel() * 2,
            "steps": steps, "api": "moe_forward_host (pinned host activations)"}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", choices=sorted(CONFIGS), default=DEFAULT_CONFIG)
    ap.add_argument("--chunks", type=int, default=DEFAULT_CHUNKS)
    ap.add_argument("--dispatch", choices=["auto", "separate", "fused"], default="auto",
                    help="separate: permute kernel first; fused: the gate/up GEMM gathers its "
                         "rows from hidden; auto: the library's choice for the shape")
    ap.add_argument("--pass", dest="pass_", choices=["forward", "backward", "train"],
                    default="forward",
                    help="forward (the layer's headline), backward (moe_backward alone) or "
                         "train (forward then backward per step)")
    ap.add_argument("--per-chunk-gemms", action="store_true",
                    help="fused dispatch: one GEMM sweep per chunk instead of per pair")
    ap.add_argument("--spinup-s", type=float, default=2.0,
                    help="untimed steps before the first timed region, in seconds: long enough "
                         "for the power-capped SM clock to settle after an idle GPU starts")
    ap.add_argument("--clock-trace", default="",
                    help="write every SM clock sample of the run (host time, MHz, reasons) here")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's token count (small cases for profiling)")
    ap.add_argument("--per-n", type=int, nargs="*", default=[1, 2, 4],
                    help="chunk counts timed for the per_n object (each with the library's "
                         "own dispatch choice)")
    ap.add_argument("--headline-only", action="store_true",
                    help="time the headline case only (no per_n, isolated row kernels, "
                         "timeline)")
    ap.add_argument("--timeline", default="",
                    help="write the launch timeline of one step (headline N and dispatch, "
                         "N=1, and the separate dispatch at the headline N) to this JSON file")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)  # at least 3 untimed warm-up steps, always
    cfg = CONFIGS[args.config]
    if args.tokens > 0:
        cfg = dataclasses.replace(cfg, T=args.tokens)
    if args.impl == "reference":
        return run_reference(args, cfg)
    if args.pass_ != "forward":
        return run_backward(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
