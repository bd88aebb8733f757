"""Pins of the CPU oracle against facts fixed outside it: the pages' printed
numbers, closed forms, textbook special cases and brute force."""
import os

import numpy as np
import pytest
import scipy.special

from oracle import decoder as O
from speculative_moe_decoding_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _tiny_oracle(bits):
    return O.Oracle(synth.TINY.as_dict(), bits)


def _read_kv(path):
    out = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split()
        out[k] = float(v)
    return out


# ---------------------------------------------------------------- dimensions
def test_param_counts_match_model_spec_table():
    """Specification table: ~570M active / ~3B total decoder parameters.  The
    assumed head layout, expert width and dense first layer must reproduce both."""
    spec = _read_kv(os.path.join(GOLDEN, "model_spec.txt"))
    m = synth.FULL.as_dict()
    for key in ("n_layers", "d_model", "n_experts", "n_shared", "top_k", "vocab", "rope_theta"):
        assert m[key] == spec[key], key
    total, active = O.active_param_count(m)
    assert abs(active / spec["active_params_approx"] - 1) < 0.02, active
    assert abs(total / spec["total_params_approx"] - 1) < 0.05, total
    # the manifest holds exactly the counted decoder tensors (plus norms and the draft)
    man = dict(synth.manifest(synth.FULL))
    counted = sum(int(np.prod(s)) for n, s in man.items()
                  if not n.startswith("draft.") and not synth.is_gain(n))
    assert counted == total


# ---------------------------------------------------------------- closed forms
def test_rmsnorm_constant_vector():
    for c in (0.5, -3.0, 1e-2):
        x = np.full((1, 64), c, np.float32)
        y = O.rmsnorm(x, np.ones(64, np.float32), 1e-6)
        want = np.sign(c) / np.sqrt(1 + 1e-6 / c ** 2)
        np.testing.assert_allclose(y, want, rtol=1e-6)


def test_rmsnorm_scale_invariance_and_gain():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((3, 128)).astype(np.float32)
    g = rng.standard_normal(128).astype(np.float32)
    np.testing.assert_allclose(O.rmsnorm(7.0 * x, g, 0.0), O.rmsnorm(x, g, 0.0), rtol=2e-6, atol=1e-6)
    y = O.rmsnorm(x, np.ones(128, np.float32), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-6)


def test_silu_and_softmax_textbook():
    x = np.linspace(-20, 20, 101).astype(np.float32)
    np.testing.assert_allclose(O.silu(x), x * scipy.special.expit(x), rtol=1e-6, atol=1e-7)
    z = np.random.default_rng(1).standard_normal((4, 64)).astype(np.float32) * 5
    np.testing.assert_allclose(O.softmax(z), scipy.special.softmax(z, axis=-1), rtol=1e-5, atol=1e-8)
    np.testing.assert_allclose(O.softmax(z).sum(-1), 1.0, rtol=1e-6)


def test_rope_identity_at_zero_and_norm_preserving():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((4, 64)).astype(np.float32)
    np.testing.assert_array_equal(O.apply_rope(v, 0, 1e6), v)
    for p in (1, 17, 5000, 32767):
        r = O.apply_rope(v, p, 1e6)
        np.testing.assert_allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(v, axis=-1), rtol=1e-5)


def test_rope_two_dims_is_plane_rotation():
    """head_dim = 2: the only frequency is theta^0 = 1, so position p rotates the
    pair (a, b) by p radians - the textbook 2-D rotation."""
    for p in (0, 1, 3, 10):
        r = O.apply_rope(np.array([[1.0, 0.0], [0.0, 1.0]], np.float32), p, 1e6)
        c, s = np.cos(p), np.sin(p)
        np.testing.assert_allclose(r, [[c, s], [-s, c]], atol=1e-6)


def test_rope_dot_depends_on_relative_position_only():
    rng = np.random.default_rng(3)
    q = rng.standard_normal(128).astype(np.float32)
    k = rng.standard_normal(128).astype(np.float32)
    ref = O.apply_rope(q, 40, 1e6) @ O.apply_rope(k, 33, 1e6)
    for shift in (0, 100, 2000):
        got = O.apply_rope(q, 40 + shift, 1e6) @ O.apply_rope(k, 33 + shift, 1e6)
        np.testing.assert_allclose(got, ref, rtol=2e-4, atol=2e-4)


def test_attention_special_cases():
    rng = np.random.default_rng(4)
    q = rng.standard_normal(64).astype(np.float32)
    K = rng.standard_normal((1, 64)).astype(np.float32)
    V = rng.standard_normal((1, 64)).astype(np.float32)
    np.testing.assert_allclose(O.attend(q, K, V), V[0], rtol=1e-6)  # one position -> v
    K = np.repeat(K, 9, axis=0)
    V = rng.standard_normal((9, 64)).astype(np.float32)
    np.testing.assert_allclose(O.attend(q, K, V), V.mean(0), rtol=1e-5, atol=1e-6)  # equal keys -> mean


# ---------------------------------------------------------------- MoE
def _moe_dense_bruteforce(orc, layer, xn):
    """Evaluate every expert densely and mask by the top-k gates."""
    m, w, p = orc.m, orc.w, f"layers.{layer}."
    logits = xn.astype(np.float64) @ w[p + "router"].T.astype(np.float64)
    probs = scipy.special.softmax(logits, axis=-1)
    out = np.zeros(xn.shape, np.float64)
    for r in range(xn.shape[0]):
        order = sorted(range(m["n_experts"]), key=lambda e: (-probs[r, e], e))[: m["top_k"]]
        for e in range(m["n_experts"]):
            gate = probs[r, e] if e in order else 0.0
            g = w[p + "exp_gate_up"][e].astype(np.float64) @ xn[r]
            f = g.shape[0] // 2
            h = g[:f] * scipy.special.expit(g[:f]) * g[f:]
            out[r] += gate * (w[p + "exp_down"][e].astype(np.float64) @ h)
        for s in range(m["n_shared"]):
            g = w[p + "sh_gate_up"][s].astype(np.float64) @ xn[r]
            f = g.shape[0] // 2
            out[r] += w[p + "sh_down"][s].astype(np.float64) @ (g[:f] * scipy.special.expit(g[:f]) * g[f:])
    return out


def test_moe_routed_equals_dense_bruteforce(tiny_weights):
    orc = _tiny_oracle(tiny_weights[0])
    xn = np.random.default_rng(5).standard_normal((6, 256)).astype(np.float32)
    got = orc.moe(1, xn)
    want = _moe_dense_bruteforce(orc, 1, xn)
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel < 1e-6, rel


def test_moe_topk_all_is_full_softmax_mixture(tiny_weights):
    dims = dict(synth.TINY.as_dict(), top_k=synth.TINY.n_experts, n_shared=0)
    orc = O.Oracle(dims, tiny_weights[0])
    xn = np.random.default_rng(6).standard_normal((3, 256)).astype(np.float32)
    got = orc.moe(0, xn)
    w, p = orc.w, "layers.0."
    probs = scipy.special.softmax(xn.astype(np.float64) @ w[p + "router"].T, axis=-1)
    want = sum(probs[:, e:e + 1] * O.swiglu(xn, w[p + "exp_gate_up"][e], w[p + "exp_down"][e])
               for e in range(dims["n_experts"]))
    np.testing.assert_allclose(got, want, rtol=1e-4, atol=1e-6)


def test_router_tie_breaks_to_lower_id():
    xn = np.ones((1, 4), np.float32)
    wr = np.zeros((5, 4), np.float32)  # all logits equal
    ids, gates, _ = O.route(xn, wr, 3)
    assert ids.tolist() == [[0, 1, 2]]
    np.testing.assert_allclose(gates, 0.2)
    assert O.greedy_argmax(np.array([1.0, 3.0, 3.0, 2.0], np.float32)) == 1


# ---------------------------------------------------------------- plumbing
def _zeroed(bits, names):
    b = dict(bits)
    for n in names:
        b[n] = np.zeros_like(b[n])
    return b


def test_zero_sublayer_outputs_reduce_to_bigram(tiny_weights):
    """With every attention output projection and every FFN down projection
    zero, the residual stream stays the input embedding, so the logits are
    W_lm RMSNorm(emb(token))."""
    bits = tiny_weights[0]
    names = [n for n in bits if n.endswith(".wo") or n.endswith("_down")]
    orc = _tiny_oracle(_zeroed(bits, names))
    toks = [5, 77, 4000]
    cache = orc.new_cache()
    out = orc.forward_rows(orc.embed(toks), [0, 1, 2], cache)
    emb = O.bf16_bits_to_f32(bits["embed"])[toks]
    lm = O.bf16_bits_to_f32(bits["lm_head"])
    want = (emb / np.sqrt((emb ** 2).mean(-1, keepdims=True) + 1e-6)) @ lm.T
    np.testing.assert_allclose(out.logits, want, rtol=1e-4, atol=1e-5)


def test_zero_query_gives_causal_mean_of_values(tiny_weights):
    """Wq = 0 makes every score 0, so attention returns the mean of the values
    at positions 0..p (causal)."""
    bits = dict(tiny_weights[0])
    d = 256
    wqkv = bits["layers.0.wqkv"].copy()
    wqkv[:d] = 0
    bits["layers.0.wqkv"] = wqkv
    orc = _tiny_oracle(bits)
    x = np.random.default_rng(7).standard_normal((5, d)).astype(np.float32)
    cache = orc.new_cache()
    w = orc.w
    captured = {}
    real_attend = O.attend

    def spy(q, K, V):
        captured.setdefault(K.shape[0], []).append(real_attend(q, K, V))
        return captured[K.shape[0]][-1]

    O.attend = spy
    try:
        orc.block(x, range(5), cache, {"attn_norm": "layers.0.attn_norm", "wqkv": "layers.0.wqkv",
                                       "wo": "layers.0.wo", "ffn_norm": "layers.0.ffn_norm"},
                  0, lambda xn: np.zeros_like(xn))
    finally:
        O.attend = real_attend
    xn = O.rmsnorm(x, w["layers.0.attn_norm"], 1e-6)
    v = (xn @ w["layers.0.wqkv"][2 * d:].T).reshape(5, 4, 64)
    for L in range(1, 6):
        for h in range(4):
            np.testing.assert_allclose(captured[L][h], v[:L, h].mean(0), rtol=1e-4, atol=1e-6)


def test_causality_and_block_equals_rows(tiny_weights):
    orc = _tiny_oracle(tiny_weights[0])
    x = np.random.default_rng(9).standard_normal((7, 256)).astype(np.float32)
    full = orc.forward_rows(x, list(range(7)), orc.new_cache())
    part = orc.forward_rows(x[:4], list(range(4)), orc.new_cache())
    np.testing.assert_allclose(part.hidden, full.hidden[:4], rtol=1e-5, atol=1e-5)
    c = orc.new_cache()
    rows = [orc.forward_rows(x[i:i + 1], [i], c).hidden[0] for i in range(7)]
    np.testing.assert_allclose(np.stack(rows), full.hidden, rtol=1e-5, atol=1e-5)


# ---------------------------------------------------------------- draft closed forms
def _draft_closed_form_oracle(bits, take):
    """Draft block with zero output projections and fc = [I 0] (take='h') or
    [0 I] (take='e')."""
    b = _zeroed(bits, ["draft.wo", "draft.w_down"])
    d = 256
    fc = np.zeros((d, 2 * d), np.float32)
    fc[:, :d] = np.eye(d) if take == "h" else 0
    fc[:, d:] = np.eye(d) if take == "e" else 0
    b["draft.fc"] = synth.f32_to_bf16_bits(fc)
    return _tiny_oracle(b)


def test_draft_identity_fc_on_hidden_proposes_the_bonus(tiny_weights, tiny_inputs):
    """fc = [I 0] and zero sublayer outputs make the draft's output the
    normalised verifier hidden at p, whose tied-LM-head argmax is the token at
    p + 1: the first proposal must equal the bonus token."""
    orc = _draft_closed_form_oracle(tiny_weights[0], "h")
    st = O.prefill(orc, tiny_inputs.visual[:8], tiny_inputs.prompt[:4])
    for _ in range(4):
        props = O.draft_propose(orc, st, 1)
        assert props[0] == st.bonus
        O.verify_commit(orc, st, props)


def test_draft_identity_fc_on_embedding_is_bigram(tiny_weights, tiny_inputs):
    orc = _draft_closed_form_oracle(tiny_weights[0], "e")
    st = O.prefill(orc, tiny_inputs.visual[:8], tiny_inputs.prompt[:4])
    emb = O.bf16_bits_to_f32(tiny_weights[0]["embed"])
    lm = O.bf16_bits_to_f32(tiny_weights[0]["lm_head"])
    for _ in range(3):
        e = emb[st.bonus]
        want = int(np.argmax(lm @ (e / np.sqrt((e ** 2).mean() + 1e-6))))
        props = O.draft_propose(orc, st, 2)
        assert props[0] == want
        e2 = emb[want]
        assert props[1] == int(np.argmax(lm @ (e2 / np.sqrt((e2 ** 2).mean() + 1e-6))))
        O.verify_commit(orc, st, props)


# ---------------------------------------------------------------- speculative == greedy
@pytest.fixture(scope="module")
def tiny_run(tiny_weights, tiny_inputs):
    orc = _tiny_oracle(tiny_weights[0])
    w = synth.WORKLOADS["tiny"]
    st = O.prefill(orc, tiny_inputs.visual, tiny_inputs.prompt)
    ref = O.decode(orc, st, 0, w.n_generate)
    C = w.n_visual + w.n_prompt
    return orc, ref, C


@pytest.mark.parametrize("k", [1, 2, 3])
@pytest.mark.parametrize("stream", ["draft", "correct", "wrong", "random", "forced"])
def test_speculative_commit_equals_greedy(tiny_run, tiny_inputs, k, stream):
    """Model page: greedy verification makes the speculative output identical to
    plain autoregressive decoding, for any proposal stream; 1 <= tau <= k+1."""
    orc, ref, C = tiny_run
    V = synth.TINY.vocab
    refd = {C + i: t for i, t in enumerate(ref)}
    n_gen = len(ref)
    rng = np.random.default_rng(10 + k)
    tables = synth.make_forced_tables(202, C + n_gen + 8, V, 3)

    def get(pos):
        return refd.get(pos, 0)

    proposers = {
        "draft": None,
        "correct": lambda st: [get(st.kv_len + j) for j in range(1, k + 1)],
        "wrong": lambda st: [(get(st.kv_len + j) + 1) % V for j in range(1, k + 1)],
        "random": lambda st: [int(t) for t in rng.integers(0, V, k)],
        "forced": lambda st: O.forced_proposals(
            {p: get(p) for p in range(st.kv_len, st.kv_len + k + 1)}, st.kv_len, k,
            tables.u, tables.r, tables.p, V),
    }
    st = O.prefill(orc, tiny_inputs.visual, tiny_inputs.prompt)
    taus = []
    orig = O.verify_commit

    def vc(o, s, props, record=None):
        out = orig(o, s, props, record)
        taus.append(len(out))
        return out

    O.verify_commit = vc
    try:
        got = O.decode(orc, st, k, n_gen, proposer=proposers[stream])
    finally:
        O.verify_commit = orig
    assert got == ref
    assert all(1 <= t <= k + 1 for t in taus)
    if stream == "correct":
        assert all(t == k + 1 for t in taus[:-1])
    if stream == "wrong":
        assert all(t == 1 for t in taus)


def test_attention_two_keys_is_logistic_in_scaled_score_gap():
    """Two positions with one-hot values: the output is the attention weights,
    and the weight on key 1 is the logistic function of (q.k1 - q.k2)/sqrt(Dh)."""
    rng = np.random.default_rng(11)
    for dh in (64, 128):
        q = rng.standard_normal(dh).astype(np.float32)
        K = rng.standard_normal((2, dh)).astype(np.float32)
        V = np.zeros((2, dh), np.float32)
        V[0, 0] = 1.0
        V[1, 1] = 1.0
        out = O.attend(q, K, V)
        gap = float(q.astype(np.float64) @ (K[0] - K[1]).astype(np.float64)) / np.sqrt(dh)
        np.testing.assert_allclose(out[0], scipy.special.expit(gap), rtol=1e-5)
        np.testing.assert_allclose(out[0] + out[1], 1.0, rtol=1e-6)


# ---------------------------------------------------------------- RoPE frequencies
def _pair_rotation_matrix(dh, angles):
    """Block rotation of the rotate-half layout, built entry by entry: dims i
    and i + dh/2 form plane i, turned by angles[i] (a counter-clockwise turn of
    the column vector (a, b))."""
    half = dh // 2
    M = np.zeros((dh, dh), np.float64)
    for i in range(half):
        c, s = np.cos(angles[i]), np.sin(angles[i])
        M[i, i], M[i, i + half] = c, -s
        M[i + half, i], M[i + half, i + half] = s, c
    return M


@pytest.mark.parametrize("dh", [4, 8, 128])
def test_rope_pair_frequencies_follow_the_inverse_power_schedule(dh):
    """Plane i at position p turns by p * theta^(-2i/dh), theta = 10^6 (model
    specification table, RoPE row).  At dh = 4 the second plane turns by
    p * 10^-3 radians; a schedule theta^(-i/dh), a different theta or swapped
    halves all give other angles and fail."""
    spec = _read_kv(os.path.join(GOLDEN, "model_spec.txt"))
    theta = spec["rope_theta"]
    assert theta == 1e6
    half = dh // 2
    rng = np.random.default_rng(dh)
    v = rng.standard_normal(dh).astype(np.float32)
    for p in (1, 7, 250, 4095):
        # the frequencies written out for the small cases
        if dh == 4:
            want_ang = [p * 1.0, p * 1e-3]
        elif dh == 8:
            want_ang = [p * 1.0, p * 10 ** -1.5, p * 1e-3, p * 10 ** -4.5]
        else:
            want_ang = [p * 10.0 ** (-6.0 * 2 * i / dh) for i in range(half)]
        c, s = O.rope_cos_sin(p, dh, theta)
        np.testing.assert_allclose(c, np.cos(want_ang), atol=1e-7)
        np.testing.assert_allclose(s, np.sin(want_ang), atol=1e-7)
        got = O.apply_rope(v, p, theta)
        want = _pair_rotation_matrix(dh, want_ang) @ v.astype(np.float64)
        np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-5)


def test_rope_dh4_second_plane_turns_by_a_thousandth_per_position():
    """Direct reading at dh = 4: unit vector on dim 1 (plane 1's first axis)
    goes to (cos(p/1000), sin(p/1000)) on dims (1, 3)."""
    for p in (1, 500, 3141):
        e1 = np.array([0.0, 1.0, 0.0, 0.0], np.float32)
        r = O.apply_rope(e1, p, 1e6)
        np.testing.assert_allclose(r, [0.0, np.cos(p * 1e-3), 0.0, np.sin(p * 1e-3)], atol=1e-6)


# ---------------------------------------------------------------- argmax margin
def test_top2_margin_hand_built_logits():
    """The gap between the largest and second-largest logit: the quantity the
    teacher-forced token comparison is gated on (margin < 0.1 is exempt)."""
    cases = [
        ([1.0, 3.0, 2.0], 1.0),           # max in the middle
        ([9.0, 1.0, 2.0], 7.0),           # max at index 0
        ([0.5, 0.25, 4.0], 3.5),          # max at the last index
        ([5.0, 5.0, 1.0], 0.0),           # tie at the top
        ([2.0, 7.0, 7.0, 7.0], 0.0),      # three-way tie
        ([-1.0, -5.0, -3.0], 2.0),        # all negative
        ([0.0, 0.125], 0.125),            # two entries
        ([3.0, 3.0 - 2 ** -20, -1e9], 2 ** -20),  # tiny gap, float32-exact
    ]
    for logits, want in cases:
        got = O.top2_margin(np.array(logits, np.float32))
        assert got == want, (logits, got, want)
    # invariant under a permutation and a common shift; never negative
    rng = np.random.default_rng(12)
    z = rng.standard_normal(4096).astype(np.float32)
    m = O.top2_margin(z)
    srt = np.sort(z)
    assert m == float(srt[-1] - srt[-2]) and m >= 0
    assert O.top2_margin(rng.permutation(z)) == m
    np.testing.assert_allclose(O.top2_margin(z + np.float32(10.0)), m, atol=2e-6)
