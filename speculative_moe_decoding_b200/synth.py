"""Seeded synthetic inputs for the speculative MoE decode step.

This module only draws numbers: model dimensions, the weight manifest (names and
shapes in the order the C ABI expects them), N(0, 0.02) weights rounded to
bfloat16, N(0, 1) visual embeddings, uniform prompt tokens, and the uniform
tables that drive the forced-acceptance proposal stream.  It holds none of the
decoder's arithmetic, and it is the only code that both the CPU oracle's tests
and the CUDA path's callers share.

Model dimensions follow the jina-ocr-v1 pages (news article "jina-ocr-v1:
faster document parsing on low-budget GPUs", model specification table:
12 layers, d = 1280, 64 routed + 2 shared experts, top-6, vocabulary 129,280,
RoPE theta = 10^6; FastMTP = one shared dense block recursed K = 3 times).  Head
layout, expert width, the dense first layer and the draft-block structure are
not on the pages; the values used here are the assumed ones listed beside each
config.

Weights are drawn per chunk of at most ``CHUNK`` elements from
``numpy.random.default_rng([seed, tensor_index, chunk_index])`` so the result is
the same whatever the number of worker processes.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ProcessPoolExecutor
from typing import Dict, List, Optional, Tuple

import numpy as np

CHUNK = 1 << 24  # elements per independently keyed RNG stream


@dataclasses.dataclass(frozen=True)
class ModelDims:
    d_model: int
    n_layers: int
    n_heads: int
    head_dim: int
    n_dense_first: int  # leading layers with a dense SwiGLU FFN instead of MoE
    n_experts: int
    n_shared: int
    top_k: int
    expert_ffn: int
    shared_ffn: int
    dense_ffn: int  # FFN width of the dense leading layers
    draft_ffn: int  # FFN width of the FastMTP draft block
    vocab: int
    rope_theta: float = 1.0e6
    rms_eps: float = 1.0e-6

    def as_dict(self) -> dict:
        return dataclasses.asdict(self)


# Tiny decoder: hidden 256, 2 layers, 4x64 MHA, 8 routed experts (ffn 128) +
# 1 shared (ffn 128), top-2, vocabulary 4096, draft fc 512->256 + dense block
# with ffn 512.  Both layers are MoE.
TINY = ModelDims(d_model=256, n_layers=2, n_heads=4, head_dim=64, n_dense_first=0,
                 n_experts=8, n_shared=1, top_k=2, expert_ffn=128, shared_ffn=128,
                 dense_ffn=0, draft_ffn=512, vocab=4096)

# Full decoder (DeepSeek-3B-MoE shape from the specification table; assumed:
# 10x128 MHA, layer 0 dense SwiGLU ffn 6848, expert/shared ffn 896, draft block
# dense SwiGLU ffn 6848).
FULL = ModelDims(d_model=1280, n_layers=12, n_heads=10, head_dim=128, n_dense_first=1,
                 n_experts=64, n_shared=2, top_k=6, expert_ffn=896, shared_ffn=896,
                 dense_ffn=6848, draft_ffn=6848, vocab=129280)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dims: ModelDims
    weight_seed: int
    input_seed: int
    n_visual: int
    n_prompt: int
    n_generate: int
    ks: Tuple[int, ...]
    stream_seed: Optional[int] = None  # forced-acceptance tables; None = real draft proposals
    accept_p: Tuple[float, ...] = (0.83, 0.69, 0.58)
    batch: int = 1


WORKLOADS: Dict[str, Workload] = {
    # tiny decoder, greedy decode of 64 tokens at k = 0..3 with the real draft
    "tiny": Workload("tiny", TINY, 0, 100, 64, 16, 64, (0, 1, 2, 3)),
    # full decoder, plain greedy baseline (k = 0)
    "full_k0": Workload("full_k0", FULL, 1, 101, 256, 32, 1085, (0,)),
    # full decoder + draft at k = 1, 2, 3 with the forced acceptance model
    "full_spec": Workload("full_spec", FULL, 1, 101, 256, 32, 1085, (1, 2, 3), stream_seed=202),
    # dynamic-resolution long context: 256 + 100 x 9 visual + 64 prompt, 4096 tokens, k = 3
    "full_long": Workload("full_long", FULL, 1, 103, 1156, 64, 4096, (3,), stream_seed=203),
    # batched serving, 32 concurrent sequences at k = 1 (p = 0.83), finished
    # sequences refilled; per-sequence visual counts and lengths from
    # make_batch_sequences (n_visual / n_generate here are the means)
    "full_batch32": Workload("full_batch32", FULL, 1, 104, 706, 32, 1085, (1,), stream_seed=204,
                             accept_p=(0.83,), batch=32),
}


def make_batch_sequences(seed: int, n: int) -> Tuple[np.ndarray, np.ndarray]:
    """Shapes of n sequences of the batched-serving workload: visual count
    256 + 100 u with u uniform on 0..9 (dynamic resolution), and an output
    length drawn lognormal with sigma 0.5 and mean 1,085 (mu = ln 1085 -
    sigma^2 / 2), rounded to an integer in [1, 4096]."""
    rng = np.random.default_rng([seed, 4])
    u = rng.integers(0, 10, n)
    sigma = 0.5
    mu = np.log(1085.0) - sigma * sigma / 2
    lengths = np.clip(np.rint(rng.lognormal(mu, sigma, n)), 1, 4096).astype(np.int64)
    return (256 + 100 * u).astype(np.int64), lengths


def manifest(m: ModelDims) -> List[Tuple[str, Tuple[int, ...]]]:
    """Weight tensors in C-ABI order: (name, shape).  Matrices are [out, in]."""
    d, H, Dh = m.d_model, m.n_heads, m.head_dim
    assert H * Dh == d
    out: List[Tuple[str, Tuple[int, ...]]] = [("embed", (m.vocab, d))]
    for layer in range(m.n_layers):
        p = f"layers.{layer}."
        out += [(p + "attn_norm", (d,)), (p + "wqkv", (3 * d, d)), (p + "wo", (d, d)),
                (p + "ffn_norm", (d,))]
        if layer < m.n_dense_first:
            out += [(p + "w_gate_up", (2 * m.dense_ffn, d)), (p + "w_down", (d, m.dense_ffn))]
        else:
            out += [(p + "router", (m.n_experts, d)),
                    (p + "exp_gate_up", (m.n_experts, 2 * m.expert_ffn, d)),
                    (p + "exp_down", (m.n_experts, d, m.expert_ffn)),
                    (p + "sh_gate_up", (m.n_shared, 2 * m.shared_ffn, d)),
                    (p + "sh_down", (m.n_shared, d, m.shared_ffn))]
    out += [("final_norm", (d,)), ("lm_head", (m.vocab, d))]
    out += [("draft.norm_h", (d,)), ("draft.norm_e", (d,)), ("draft.fc", (d, 2 * d)),
            ("draft.attn_norm", (d,)), ("draft.wqkv", (3 * d, d)), ("draft.wo", (d, d)),
            ("draft.ffn_norm", (d,)), ("draft.w_gate_up", (2 * m.draft_ffn, d)),
            ("draft.w_down", (d, m.draft_ffn)), ("draft.final_norm", (d,))]
    return out


def is_gain(name: str) -> bool:
    return name.endswith("norm") or name.endswith("norm_h") or name.endswith("norm_e")


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).copy()
    u += np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (u >> np.uint32(16)).astype(np.uint16)


def _draw_chunk(args):
    seed, tidx, cidx, n, std = args
    rng = np.random.default_rng([seed, tidx, cidx])
    a = rng.standard_normal(n, dtype=np.float32)
    a *= np.float32(std)
    return a


def _chunks(total: int):
    return [(c, min(CHUNK, total - c * CHUNK)) for c in range((total + CHUNK - 1) // CHUNK)]


def make_weights(m: ModelDims, seed: int, keep_f32: bool = False,
                 workers: Optional[int] = None, std: float = 0.02):
    """Draw the manifest's tensors.

    Returns ``(bits, f32)``: ``bits[name]`` is a uint16 array of bfloat16 bit
    patterns; ``f32[name]`` is the unrounded float32 draw (only if ``keep_f32``).
    Matrices and embeddings are N(0, std); norm gains are exactly 1.
    """
    man = manifest(m)
    jobs = []
    for tidx, (name, shape) in enumerate(man):
        if is_gain(name):
            continue
        total = int(np.prod(shape))
        for cidx, n in _chunks(total):
            jobs.append((seed, tidx, cidx, n, std))
    total_elems = sum(j[3] for j in jobs)
    if workers is None:
        workers = 1 if total_elems < (1 << 26) else min(32, os.cpu_count() or 1)
    if workers > 1:
        import multiprocessing as mp
        with ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn")) as ex:
            drawn = list(ex.map(_draw_chunk, jobs, chunksize=1))
    else:
        drawn = [_draw_chunk(j) for j in jobs]
    bits: Dict[str, np.ndarray] = {}
    f32: Dict[str, np.ndarray] = {}
    k = 0
    for tidx, (name, shape) in enumerate(man):
        if is_gain(name):
            g = np.ones(shape, np.float32)
            bits[name] = f32_to_bf16_bits(g)
            if keep_f32:
                f32[name] = g
            continue
        total = int(np.prod(shape))
        parts = []
        for _ in _chunks(total):
            parts.append(drawn[k])
            k += 1
        a = parts[0] if len(parts) == 1 else np.concatenate(parts)
        bits[name] = f32_to_bf16_bits(a).reshape(shape)
        if keep_f32:
            f32[name] = a.reshape(shape)
    return bits, (f32 if keep_f32 else None)


@dataclasses.dataclass
class SeqInputs:
    visual: np.ndarray  # float32 [n_visual, d]
    prompt: np.ndarray  # int32 [n_prompt]


def make_inputs(m: ModelDims, seed: int, n_visual: int, n_prompt: int, index: int = 0) -> SeqInputs:
    """Visual embeddings N(0,1) standing in for the vision encoder output, and
    prompt tokens uniform over the vocabulary.  ``index`` selects a sequence."""
    rng = np.random.default_rng([seed, index])
    visual = rng.standard_normal((n_visual, m.d_model), dtype=np.float32)
    prompt = rng.integers(0, m.vocab, size=n_prompt, dtype=np.int64).astype(np.int32)
    return SeqInputs(visual, prompt)


@dataclasses.dataclass
class ForcedTables:
    """Per (target position, draft depth) draws for the forced acceptance model.

    ``u[pos, j]`` is uniform in [0, 1); ``r[pos, j]`` is uniform over
    {0, ..., vocab - 2}.  A proposal at depth j+1 for target position ``pos``
    keeps the reference token when ``u < p[j]`` and otherwise takes the
    ``r``-th token of the vocabulary with the reference token removed.
    """
    u: np.ndarray  # float32 [n_pos, max_k]
    r: np.ndarray  # int32 [n_pos, max_k]
    p: Tuple[float, ...]


def make_forced_tables(seed: int, n_pos: int, vocab: int, max_k: int = 3,
                       p: Tuple[float, ...] = (0.83, 0.69, 0.58), index: int = 0) -> ForcedTables:
    rng = np.random.default_rng([seed, index, 7])
    u = rng.random((n_pos, max_k), dtype=np.float32)
    r = rng.integers(0, vocab - 1, size=(n_pos, max_k), dtype=np.int64).astype(np.int32)
    return ForcedTables(u, r, tuple(p[:max_k]))
