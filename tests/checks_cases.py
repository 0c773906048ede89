"""The cases that test_gpu_checks.py runs with both builds of the library: forward in both
dispatches and several chunk counts (an empty trailing chunk, duplicate experts, idle
experts) and backward; each returns its outputs (on the CPU) and the range flags read
right after it."""
import torch

from gen import CONFIGS, LayerConfig, bf16_normal, layer_inputs

MID = LayerConfig("mid", 300, 512, 16, 4, 384, "normal")


def run_cases(moe):
    out = {}
    for name, chunks in (("tiny", (1, 2)), ("edge", (8, 7, 3)), ("edge_pair01", (8,)),
                         ("edge_varlen", (8,))):
        cfg = CONFIGS[name]
        gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
        for N in chunks:
            for dispatch in ("separate", "fused"):
                y = moe.forward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"], gpu["wd"],
                                num_chunks=N, ep_groups=cfg.G, dispatch=dispatch)
                torch.cuda.synchronize()
                out[f"fwd {name} N={N} {dispatch}"] = ([y.cpu()], moe.checks_read())
    for cfg, N in ((CONFIGS["tiny"], 2), (MID, 3), (CONFIGS["edge_varlen"], 8)):
        gpu = {k: v.cuda() for k, v in layer_inputs(cfg).items()}
        dout = bf16_normal((cfg.T, cfg.H), 1.0, 99).cuda()
        r = moe.backward(gpu["hidden"], gpu["idx"], gpu["w"], gpu["wgu"], gpu["wd"], dout,
                         num_chunks=N, ep_groups=cfg.G)
        torch.cuda.synchronize()
        out[f"bwd {cfg.name} N={N}"] = ([t.cpu() for t in r], moe.checks_read())
    return out
