"""Times single kernels of the library through its single-kernel entry points.

    python -m speculative_moe_decoding_b200.kernel_bench --op lm_argmax --rows 4
    python -m speculative_moe_decoding_b200.kernel_bench --op norm_gemv --n 64 --k 1280 --rows 4
    python -m speculative_moe_decoding_b200.kernel_bench --op moe --rows 4
    python -m speculative_moe_decoding_b200.kernel_bench --op attention --rows 4 --ctx 832

--op moe builds a two-layer decoder whose second layer is the full-size MoE
layer (d = 1280, 64 routed + 2 shared experts of ffn 896, top-6; vocabulary
4,096 to keep the model near 0.6 GB), decodes a few k = rows - 1 steps and then
times that layer's MoE FFN alone (ocrdec_replay_moe_ffn on the last pass's
routing).  With --eager the launches go straight to the stream (for ncu: the
layer's launches are the 4th and later of the MoE kernel).

--op attention builds the same two-layer decoder with a --ctx-position
context (832: the middle of the full_spec decode) and runs k = rows - 1 decode
steps straight to the stream inside an NVTX range "timed_steps": each step
launches the attention block three times for the draft and then once per
verifier layer, so the MoE layer's attention block (router partials, pass rows
read before the dependency wait) is launch 4 of each step in that range.

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
    ap.add_argument("--op", choices=["lm_argmax", "norm_gemv", "moe", "attention"], default="lm_argmax")
    ap.add_argument("--eager", action="store_true", help="moe: launch without a graph (ncu)")
    ap.add_argument("--ctx", type=int, default=832, help="attention: context positions before the steps")
    ap.add_argument("--n", type=int, default=129280)
    ap.add_argument("--k", type=int, default=1280)
    ap.add_argument("--rows", type=int, default=4)
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--no-flush", action="store_true")
    a = ap.parse_args()
    build.build()
    if a.op == "moe":
        return moe(a)
    if a.op == "attention":
        return attention(a)
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


def two_layer_dims():
    from . import synth
    return synth.ModelDims(d_model=1280, n_layers=2, n_heads=10, head_dim=128, n_dense_first=1, n_experts=64,
                           n_shared=2, top_k=6, expert_ffn=896, shared_ffn=896, dense_ffn=6848, draft_ffn=6848,
                           vocab=4096)


def attention(a):
    from . import ocrdec, synth
    m = two_layer_dims()
    bits, _ = synth.make_weights(m, 1)
    names = [n for n, _ in synth.manifest(m)]
    k = a.rows - 1
    steps = 3
    dec = ocrdec.Decoder(m.as_dict(), bits, names, max_k=3, max_batch=1, kv_capacity=a.ctx + 64)
    inp = synth.make_inputs(m, 101, a.ctx - 32, 32)
    dec.prefill(0, torch.from_numpy(inp.visual).cuda(), torch.from_numpy(inp.prompt).cuda())
    for _ in range(2):
        dec.step(1, k)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed_steps")
    e0.record(s)
    for _ in range(steps):
        dec.step(1, k)
    e1.record(s)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    print(json.dumps({"op": "attention", "rows": a.rows, "ctx": a.ctx, "eager_steps": steps,
                      "eager_step_us": e0.elapsed_time(e1) * 1e3 / steps, "status": dec.status()}))
    dec.close()
    return 0


def moe(a):
    import numpy as np

    from . import ocrdec, synth
    m = two_layer_dims()
    bits, _ = synth.make_weights(m, 1)
    names = [n for n, _ in synth.manifest(m)]
    k = a.rows - 1
    dec = ocrdec.Decoder(m.as_dict(), bits, names, max_k=3, max_batch=1, kv_capacity=256)
    inp = synth.make_inputs(m, 101, 4, 4)
    dec.prefill(0, torch.from_numpy(inp.visual).cuda(), torch.from_numpy(inp.prompt).cuda())
    for _ in range(2):
        dec.step(1, k)  # the last one leaves a k+1-row pass's rows and router partials
    torch.cuda.synchronize()
    assert dec.status() == 0
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream()
    dec.reset_counters()
    launch = lambda: dec.replay_moe_ffn(1, k, 1, 1)
    if a.eager:
        for i in range(3):
            flush.fill_(i & 0xFF)
            launch()
        torch.cuda.synchronize()
        print(json.dumps({"op": "moe", "eager_launches": 3, "status": dec.status()}))
        return 0
    launch()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        launch()
    times = []
    for i in range(a.warmup + a.iters):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        graph.replay()
        e1.record(s)
        torch.cuda.synchronize()
        if i >= a.warmup:
            times.append(e0.elapsed_time(e1))
    touched, passes = dec.counters()
    U = touched / max(1, passes)
    ms = float(np.mean(times))
    nbytes = (U + m.n_shared) * 3 * m.d_model * m.expert_ffn * 2 + 2 * a.rows * m.d_model * 4
    print(json.dumps({"op": "moe", "rows": a.rows, "touched_routed": U, "mean_us": ms * 1e3,
                      "min_us": min(times) * 1e3, "bytes": nbytes, "GBps": nbytes / (ms / 1e3) / 1e9,
                      "status": dec.status()}))
    dec.close()
    return 0


if __name__ == "__main__":
    main()
