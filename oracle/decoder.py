"""CPU oracle of the greedy-verified speculative MoE decode step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this module.  It shares no code with
the CUDA library and imports nothing from it.

Plain numpy in float32 (the decoder's weights are the bfloat16-rounded values,
upcast here; every product and sum is float32).  Decode work goes one row at a
time through :meth:`Oracle.forward_rows` with a single row, so the committed
tokens of a speculative run and of a plain greedy run come from literally the
same sequence of floating-point operations.

Sources (jina-ocr-v1 pages; the news article "jina-ocr-v1: faster document
parsing on low-budget GPUs" and the jina-ocr-v1 model page):

* decoder shape - model specification table (12 layers, d = 1280, 64 routed +
  2 shared experts, top-6, vocabulary 129,280, RoPE theta = 10^6);
* draft - section "Model and training": FastMTP applies ONE dense block
  recursively for K = 3 prediction steps; section "Getting started": the head is
  trained with recursive hidden-state feedback (each draft step feeds its own
  hidden state forward, drafts are not re-verified one by one);
* verification - section "Model and training": the verifier greedily checks
  the proposal and accepts the longest prefix on which draft and verifier
  agree, so the committed sequence equals the verifier's greedy sequence
  (model page: bit-identical to plain autoregressive decoding);
* tau - section "Speculative decoding on L4": tau counts the tokens committed
  per speculative step including the bonus token.

Readings where the pages are silent (each is the plainest one):
pre-norm blocks with RMSNorm (eps 1e-6, gain vector), no biases; multi-head
attention with scale 1/sqrt(head_dim) and a causal mask; rotate-half RoPE over
the whole head with angle p * theta^(-2i/head_dim) evaluated in float64 and cast
to float32; SwiGLU experts y = W_down (silu(W_gate x) * (W_up x)); router =
softmax over all experts, then top-k (ties to the lower expert id), gates are
the softmax values without renormalisation; shared experts are added with gate
1; greedy argmax takes the lowest index on ties.  Draft block: u = W_fc
[RMSNorm(h); RMSNorm(e_next)], then one pre-norm block (attention over the
draft's own KV cache + dense SwiGLU), then its own final RMSNorm and the
verifier's LM head (tied).  The pair (hidden at position p, input at p + 1)
runs at RoPE position p.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Dict, List, Optional, Sequence, Tuple

import numpy as np

F32 = np.float32


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(F32)


# --------------------------------------------------------------------------
# elementary operations
# --------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g."""
    x = x.astype(F32, copy=False)
    ms = np.mean(x * x, axis=-1, keepdims=True, dtype=F32)
    return (x / np.sqrt(ms + F32(eps))) * g


def silu(x: np.ndarray) -> np.ndarray:
    return x / (F32(1) + np.exp(-x))


def softmax(x: np.ndarray) -> np.ndarray:
    z = x - np.max(x, axis=-1, keepdims=True)
    e = np.exp(z)
    return e / np.sum(e, axis=-1, keepdims=True, dtype=F32)


def rope_cos_sin(pos: int, head_dim: int, theta: float) -> Tuple[np.ndarray, np.ndarray]:
    """cos/sin of the rotary angles for one position (float64 math, float32 result)."""
    half = head_dim // 2
    i = np.arange(half, dtype=np.float64)
    inv_freq = np.power(np.float64(theta), -2.0 * i / head_dim)
    ang = np.float64(pos) * inv_freq
    return np.cos(ang).astype(F32), np.sin(ang).astype(F32)


def apply_rope(v: np.ndarray, pos: int, theta: float) -> np.ndarray:
    """Rotate-half RoPE on [..., head_dim] vectors at one position."""
    dh = v.shape[-1]
    half = dh // 2
    c, s = rope_cos_sin(pos, dh, theta)
    a, b = v[..., :half], v[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1).astype(F32)


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """One query head against keys/values [L, Dh]: softmax(q K^T / sqrt(Dh)) V."""
    s = (K @ q) / np.sqrt(F32(q.shape[-1]))
    p = softmax(s.astype(F32))
    return (p @ V).astype(F32)


def swiglu(x: np.ndarray, w_gate_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """y = W_down (silu(W_gate x) * (W_up x)); W_gate = first half of the rows of w_gate_up."""
    f = w_gate_up.shape[0] // 2
    gu = x @ w_gate_up.T
    h = silu(gu[..., :f]) * gu[..., f:]
    return (h @ w_down.T).astype(F32)


def route(xn: np.ndarray, w_router: np.ndarray, top_k: int):
    """Router for rows xn [n, d]: softmax over all experts, then the top_k
    largest probabilities (ties to the lower id).  Returns (ids, gates, probs)."""
    probs = softmax((xn @ w_router.T).astype(F32))
    ids = np.argsort(-probs, axis=-1, kind="stable")[:, :top_k]
    gates = np.take_along_axis(probs, ids, axis=-1)
    return ids, gates, probs


def greedy_argmax(logits: np.ndarray) -> int:
    return int(np.argmax(logits))  # first maximum = lowest index on ties


def top2_margin(logits: np.ndarray) -> float:
    t = np.partition(logits, -2)[-2:]
    return float(t[1] - t[0])


# --------------------------------------------------------------------------
# KV cache
# --------------------------------------------------------------------------

class KV:
    """Per-layer key/value storage for one sequence; rows are positions."""

    def __init__(self, n_layers: int, n_heads: int, head_dim: int, cap: int = 64):
        self.k = [np.zeros((cap, n_heads, head_dim), F32) for _ in range(n_layers)]
        self.v = [np.zeros((cap, n_heads, head_dim), F32) for _ in range(n_layers)]
        self.length = 0

    def _grow(self, need: int):
        cap = self.k[0].shape[0]
        if need <= cap:
            return
        new = max(need, 2 * cap)
        for lst in (self.k, self.v):
            for i, a in enumerate(lst):
                b = np.zeros((new,) + a.shape[1:], F32)
                b[:cap] = a
                lst[i] = b

    def write(self, layer: int, pos: int, k: np.ndarray, v: np.ndarray):
        self._grow(pos + 1)
        self.k[layer][pos] = k
        self.v[layer][pos] = v

    def truncate(self, length: int):
        self.length = length


# --------------------------------------------------------------------------
# model
# --------------------------------------------------------------------------

@dataclasses.dataclass
class RowsOut:
    hidden: np.ndarray            # [n, d] residual after the last layer (pre final norm)
    layer_hidden: List[np.ndarray]  # per layer, [n, d] residual after that layer
    logits: Optional[np.ndarray]  # [n, V] or None


class Oracle:
    """The decoder plus its FastMTP draft block, on the CPU."""

    def __init__(self, dims: dict, weights: Dict[str, np.ndarray], weights_are_bits: bool = True):
        self.m = dims
        conv = bf16_bits_to_f32 if weights_are_bits else (lambda a: np.asarray(a, F32))
        self.w = {k: conv(v) for k, v in weights.items()}
        d = dims["d_model"]
        self.H = dims["n_heads"]
        self.Dh = dims["head_dim"]
        assert self.H * self.Dh == d
        self.eps = dims["rms_eps"]
        self.theta = dims["rope_theta"]

    # ---- verifier ---------------------------------------------------------
    def new_cache(self) -> KV:
        return KV(self.m["n_layers"], self.H, self.Dh)

    def ffn(self, layer: int, xn: np.ndarray) -> np.ndarray:
        """FFN of one layer on normalised rows xn [n, d]."""
        m, w, p = self.m, self.w, f"layers.{layer}."
        if layer < m["n_dense_first"]:
            return swiglu(xn, w[p + "w_gate_up"], w[p + "w_down"])
        return self.moe(layer, xn)

    def moe(self, layer: int, xn: np.ndarray) -> np.ndarray:
        """Routed experts (top-k, softmax gates) plus the always-on shared experts."""
        m, w, p = self.m, self.w, f"layers.{layer}."
        ids, gates, _ = route(xn, w[p + "router"], m["top_k"])
        out = np.zeros_like(xn, dtype=F32)
        gu, dn = w[p + "exp_gate_up"], w[p + "exp_down"]
        for e in range(m["n_experts"]):
            rows, slot = np.nonzero(ids == e)
            if rows.size == 0:
                continue
            y = swiglu(xn[rows], gu[e], dn[e])
            out[rows] += gates[rows, slot][:, None] * y
        for s in range(m["n_shared"]):
            out += swiglu(xn, w[p + "sh_gate_up"][s], w[p + "sh_down"][s])
        return out

    def block(self, x: np.ndarray, positions: Sequence[int], cache: KV, layer_names: dict,
              layer: int, ffn: Callable[[np.ndarray], np.ndarray]) -> np.ndarray:
        """One pre-norm transformer block over rows x [n, d] at the given
        positions.  Each row's key/value is written into ``cache`` at its
        position before attention; row i attends to positions 0..positions[i]."""
        w = self.w
        H, Dh = self.H, self.Dh
        d = x.shape[1]
        xn = rmsnorm(x, w[layer_names["attn_norm"]], self.eps)
        qkv = xn @ w[layer_names["wqkv"]].T
        q = qkv[:, :d].reshape(-1, H, Dh)
        k = qkv[:, d:2 * d].reshape(-1, H, Dh)
        v = qkv[:, 2 * d:].reshape(-1, H, Dh)
        for i, p in enumerate(positions):
            q[i] = apply_rope(q[i], p, self.theta)
            cache.write(layer, p, apply_rope(k[i], p, self.theta), v[i])
        att = np.zeros((x.shape[0], H, Dh), F32)
        for i, p in enumerate(positions):
            K = cache.k[layer][:p + 1]
            V = cache.v[layer][:p + 1]
            for h in range(H):
                att[i, h] = attend(q[i, h], K[:, h], V[:, h])
        x = x + att.reshape(-1, d) @ w[layer_names["wo"]].T
        xn = rmsnorm(x, w[layer_names["ffn_norm"]], self.eps)
        return (x + ffn(xn)).astype(F32)

    def forward_rows(self, x: np.ndarray, positions: Sequence[int], cache: KV,
                     want_logits: bool = True) -> RowsOut:
        """Verifier forward for input rows x [n, d] (embeddings or visual
        vectors) at consecutive or arbitrary positions; appends to ``cache``."""
        x = np.asarray(x, F32)
        per_layer = []
        for layer in range(self.m["n_layers"]):
            p = f"layers.{layer}."
            names = {"attn_norm": p + "attn_norm", "wqkv": p + "wqkv", "wo": p + "wo",
                     "ffn_norm": p + "ffn_norm"}
            x = self.block(x, positions, cache, names, layer, lambda xn, l=layer: self.ffn(l, xn))
            per_layer.append(x.copy())
        cache.length = max(cache.length, max(positions) + 1)
        logits = self.lm_logits(x, "final_norm") if want_logits else None
        return RowsOut(x, per_layer, logits)

    def lm_logits(self, x: np.ndarray, norm_name: str) -> np.ndarray:
        xn = rmsnorm(x, self.w[norm_name], self.eps)
        return (xn @ self.w["lm_head"].T).astype(F32)

    def embed(self, tokens: Sequence[int]) -> np.ndarray:
        return self.w["embed"][np.asarray(tokens, dtype=np.int64)].astype(F32)

    # ---- draft ------------------------------------------------------------
    def new_draft_cache(self) -> KV:
        return KV(1, self.H, self.Dh)

    def draft_rows(self, h: np.ndarray, e_next: np.ndarray, positions: Sequence[int],
                   dcache: KV) -> np.ndarray:
        """FastMTP block on pairs (hidden h_p, next input e_{p+1}) at positions
        p.  Returns the block's pre-norm outputs [n, d]."""
        w = self.w
        z = np.concatenate([rmsnorm(h, w["draft.norm_h"], self.eps),
                            rmsnorm(e_next, w["draft.norm_e"], self.eps)], axis=-1)
        u = (z @ w["draft.fc"].T).astype(F32)
        names = {"attn_norm": "draft.attn_norm", "wqkv": "draft.wqkv", "wo": "draft.wo",
                 "ffn_norm": "draft.ffn_norm"}
        out = self.block(u, positions, dcache, names, 0,
                         lambda xn: swiglu(xn, w["draft.w_gate_up"], w["draft.w_down"]))
        dcache.length = max(dcache.length, max(positions) + 1)
        return out

    def draft_token(self, hprime_row: np.ndarray, margins: Optional[list] = None) -> int:
        logits = self.lm_logits(hprime_row[None, :], "draft.final_norm")[0]
        if margins is not None:
            margins.append(logits)
        return greedy_argmax(logits)


# --------------------------------------------------------------------------
# sequence state and the decode loops
# --------------------------------------------------------------------------

@dataclasses.dataclass
class SeqState:
    cache: KV
    dcache: Optional[KV]
    tokens: Dict[int, int]          # committed token at each generated position
    kv_len: int                     # positions 0..kv_len-1 are in the verifier cache
    bonus: int                      # token at position kv_len (committed, not yet in cache)
    pend_h: np.ndarray              # hiddens of the pairs the draft has not consumed
    pend_pos: List[int]             # their positions
    n_generated: int
    steps: int = 0
    tau_sum: int = 0
    accepted_at_depth: Optional[List[int]] = None


def prefill(orc: Oracle, visual: np.ndarray, prompt: Sequence[int], with_draft: bool = True,
            block_rows: int = 64) -> SeqState:
    """Context = visual rows then prompt tokens at positions 0..C-1.  Returns the
    state whose bonus token is the first generated token (argmax at C-1).
    The draft consumes the context pairs (h_p, input_{p+1}) for p < C-1; the
    last pair (h_{C-1}, first generated token) is left pending."""
    inputs = np.concatenate([np.asarray(visual, F32), orc.embed(prompt)], axis=0)
    C = inputs.shape[0]
    cache = orc.new_cache()
    hid = []
    last_logits = None
    for s in range(0, C, block_rows):
        e = min(C, s + block_rows)
        out = orc.forward_rows(inputs[s:e], list(range(s, e)), cache, want_logits=(e == C))
        hid.append(out.hidden)
        if e == C:
            last_logits = out.logits[-1]
    H = np.concatenate(hid, axis=0)
    first = greedy_argmax(last_logits)
    dcache = None
    if with_draft:
        dcache = orc.new_draft_cache()
        for s in range(0, C - 1, block_rows):
            e = min(C - 1, s + block_rows)
            orc.draft_rows(H[s:e], inputs[s + 1:e + 1], list(range(s, e)), dcache)
        dcache.truncate(C - 1)
    return SeqState(cache=cache, dcache=dcache, tokens={C: first}, kv_len=C, bonus=first,
                    pend_h=H[C - 1:C].copy(), pend_pos=[C - 1], n_generated=1,
                    accepted_at_depth=[0, 0, 0, 0])


def draft_propose(orc: Oracle, st: SeqState, k: int, margins: Optional[list] = None) -> List[int]:
    """(``margins``, if given, receives each recursion's draft logits.)"""
    """k recursions of the shared draft block.  Recursion 1 consumes the pending
    pairs (verifier hidden at p, committed token at p+1); recursion j >= 2 feeds
    the block's own output hidden with the previous draft token."""
    assert st.dcache is not None
    nxt = [st.tokens[p + 1] for p in st.pend_pos]
    out = orc.draft_rows(st.pend_h, orc.embed(nxt), st.pend_pos, st.dcache)
    base = st.kv_len  # == pend_pos[-1] + 1
    hprime = out[-1]
    props = [orc.draft_token(hprime, margins)]
    for j in range(2, k + 1):
        pos = base + j - 2
        out = orc.draft_rows(hprime[None, :], orc.embed([props[-1]]), [pos], st.dcache)
        hprime = out[-1]
        props.append(orc.draft_token(hprime, margins))
    st.dcache.truncate(base)  # recursion rows beyond the committed prefix are discarded
    st.pend_h = st.pend_h[:0]
    st.pend_pos = []
    return props


def verify_commit(orc: Oracle, st: SeqState, proposals: Sequence[int],
                  record: Optional[list] = None, forced_g: Optional[Sequence[int]] = None) -> List[int]:
    """One verifier pass over [bonus, d_1..d_k] at positions n..n+k, processed one
    row at a time; commits the longest agreeing prefix plus the bonus token and
    rolls the KV length back to n + a + 1.  ``forced_g`` (tests only) replaces the
    rows' greedy tokens - teacher forcing onto another implementation's choices."""
    n = st.kv_len
    rows = [st.bonus] + list(proposals)
    g, hs = [], []
    for i, tok in enumerate(rows):
        out = orc.forward_rows(orc.embed([tok]), [n + i], st.cache)
        g.append(greedy_argmax(out.logits[0]))
        hs.append(out.hidden[0])
        if record is not None:
            record.append((n + i, tok, out))
    if forced_g is not None:
        g = [int(t) for t in forced_g]
    a = 0
    while a < len(proposals) and proposals[a] == g[a]:
        a += 1
    committed = g[:a + 1]
    for i, t in enumerate(committed):
        st.tokens[n + 1 + i] = t
    st.kv_len = n + a + 1
    st.cache.truncate(st.kv_len)
    st.bonus = committed[-1]
    st.pend_h = np.stack(hs[:a + 1])
    st.pend_pos = list(range(n, n + a + 1))
    st.n_generated += a + 1
    st.steps += 1
    st.tau_sum += a + 1
    if st.accepted_at_depth is not None:
        st.accepted_at_depth[a] += 1
    return committed


def forced_proposals(ref: Dict[int, int], n: int, k: int, u: np.ndarray, r: np.ndarray,
                     p: Sequence[float], vocab: int) -> List[int]:
    """Acceptance model for benchmarking: the proposal for target position n+j
    keeps the reference (greedy) token when u[n+j, j-1] < p[j-1]; otherwise it
    is a token drawn uniformly from the vocabulary without the reference token
    (index r[n+j, j-1] into that reduced vocabulary)."""
    out = []
    for j in range(1, k + 1):
        t = n + j
        want = ref[t]
        if u[t, j - 1] < np.float32(p[j - 1]):
            out.append(want)
        else:
            alt = int(r[t, j - 1])
            out.append(alt if alt < want else alt + 1)
    return out


def decode(orc: Oracle, st: SeqState, k: int, n_generate: int,
           proposer: Optional[Callable[[SeqState], List[int]]] = None,
           record: Optional[list] = None) -> List[int]:
    """Run steps until ``n_generate`` tokens are generated (the prefill's first
    token counts).  ``proposer`` overrides the draft's proposals (the draft still
    runs when ``st.dcache`` is present, as in the timed benchmark path)."""
    while st.n_generated < n_generate:
        props: List[int] = []
        if k > 0:
            props = draft_propose(orc, st, k) if st.dcache is not None else []
            if proposer is not None:
                props = proposer(st)
        verify_commit(orc, st, props, record)
    C = min(st.tokens)
    return [st.tokens[C + i] for i in range(n_generate)]


def active_param_count(dims: dict) -> Tuple[int, int]:
    """(total, active-per-token) parameter counts of the decoder (embedding
    lookup counts one row; LM head counts fully)."""
    d, L, V = dims["d_model"], dims["n_layers"], dims["vocab"]
    attn = 4 * d * d
    dense = 3 * d * dims["dense_ffn"]
    exp = 3 * d * dims["expert_ffn"]
    sh = 3 * d * dims["shared_ffn"]
    router = dims["n_experts"] * d
    nd, nm = dims["n_dense_first"], L - dims["n_dense_first"]
    total = L * attn + nd * dense + nm * (dims["n_experts"] * exp + dims["n_shared"] * sh + router) + 2 * V * d
    active = L * attn + nd * dense + nm * (dims["top_k"] * exp + dims["n_shared"] * sh + router) + V * d + d
    return total, active
