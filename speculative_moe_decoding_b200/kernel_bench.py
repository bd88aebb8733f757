"""Times single kernels of the library through its single-kernel entry points.

    python -m speculative_moe_decoding_b200.kernel_bench --op lm_argmax --rows 4
    python -m speculative_moe_decoding_b200.kernel_bench --op norm_gemv --n 64 --k 1280 --rows 4

Weights are random bf16 on the device (values do not matter for timing).  L2 is
flushed (a 256 MB write) before every timed launch; times are CUDA events on the
launching stream around a CUDA-graph replay of the launch (no host overhead
inside the timed region).  Also the small, bounded case used for ncu captures.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import build


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["lm_argmax", "norm_gemv"], default="lm_argmax")
    ap.add_argument("--n", type=int, default=129280)
    ap.add_argument("--k", type=int, default=1280)
    ap.add_argument("--rows", type=int, default=4)
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--no-flush", action="store_true")
    a = ap.parse_args()
    build.build()
    from . import ocrdec
    torch.manual_seed(0)
    W = (torch.randn(a.n, a.k, device="cuda") * 0.02).to(torch.bfloat16)
    g = torch.ones(a.k, device="cuda", dtype=torch.bfloat16)
    x = torch.randn(a.rows, a.k, device="cuda")
    scratch = ocrdec.op_scratch()
    tok = torch.empty(a.rows, dtype=torch.int32, device="cuda")
    y = torch.empty(a.rows, a.n, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream()

    def launch():
        if a.op == "lm_argmax":
            ocrdec.op_lm_argmax(W, x, g, 1e-6, tok, None, scratch)
        else:
            ocrdec.op_norm_gemv(W, x, g, 1e-6, y, scratch)

    launch()  # one-time kernel set-up outside the graph
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        launch()
    times = []
    for i in range(a.warmup + a.iters):
        if not a.no_flush:
            flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        graph.replay()
        e1.record(s)
        torch.cuda.synchronize()
        if i >= a.warmup:
            times.append(e0.elapsed_time(e1))
    ms = sum(times) / len(times)
    nbytes = a.n * a.k * 2 + a.rows * a.k * 4
    print(json.dumps({"op": a.op, "n": a.n, "k": a.k, "rows": a.rows, "mean_us": ms * 1e3,
                      "min_us": min(times) * 1e3, "GBps": nbytes / (ms / 1e3) / 1e9}))


if __name__ == "__main__":
    main()
