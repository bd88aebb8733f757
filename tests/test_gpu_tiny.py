"""GPU parity of the CUDA path against the CPU oracle on the tiny decoder, and
the bit-identity of speculative decoding with the library's own k = 0 run.

Tolerances (from the bfloat16 storage of activations, weights and KV on the GPU
against float32 arithmetic in the oracle): per-layer hidden-state relative L2
<= 1e-2, logits max-abs <= 5e-2, and greedy tokens equal wherever the oracle's
top-1/top-2 logit margin is at least 0.1."""
import numpy as np
import pytest

from oracle import decoder as O
from speculative_moe_decoding_b200 import synth

from .gpu_util import gpu_decode, make_decoder, to_dev

pytestmark = pytest.mark.gpu

HIDDEN_REL_L2 = 1e-2
LOGIT_ABS = 5e-2
MARGIN = 0.1
W = synth.WORKLOADS["tiny"]


@pytest.fixture(scope="module")
def tiny_bits():
    bits, _ = synth.make_weights(synth.TINY, W.weight_seed, workers=1)
    return bits


@pytest.fixture(scope="module")
def inputs():
    return synth.make_inputs(synth.TINY, W.input_seed, W.n_visual, W.n_prompt)


@pytest.fixture(scope="module")
def dec(tiny_bits):
    d = make_decoder(synth.TINY, tiny_bits, max_k=3, max_batch=1, kv_capacity=256)
    yield d
    d.close()


@pytest.fixture(scope="module")
def orc(tiny_bits):
    return O.Oracle(synth.TINY.as_dict(), tiny_bits)


@pytest.fixture(scope="module")
def k0_tokens(dec, inputs):
    toks, st, _ = gpu_decode(dec, inputs, 0, W.n_generate)
    return toks


# ---------------------------------------------------------------- single kernels
def _bf16(a):
    return O.bf16_bits_to_f32(synth.f32_to_bf16_bits(a))


def _split_bound(xn, Wf):
    """Error bound of the GEMV against the float32 product xn W^T.  The kernel
    feeds each normalised activation as two bfloat16 parts (x ~ hi + lo, error
    at most 2^-17 |x|) and multiplies both with the bfloat16 weights, so the
    products are exact and only that split and about K/32 float32
    accumulation steps remain (each at most 2^-24 of the running sum): well
    under 2^-15 of sum |W||x|.  Using the high part alone (error up to 2^-9 |x|)
    breaks this bound."""
    return (np.abs(xn) @ np.abs(Wf).T) * 2.0 ** -15 + 1e-6


# K = 2048 is the largest normalised width; K = 1984 ends in a slice of three
# 64-column chunks; N values that are not multiples of 32 leave ragged tiles
@pytest.mark.parametrize("R,N,K", [(1, 72, 256), (3, 1280, 1280), (8, 64, 2048), (4, 3840, 1280), (5, 100, 1984)])
def test_op_norm_gemv(R, N, K):
    import torch
    from speculative_moe_decoding_b200 import build
    build.build()
    from speculative_moe_decoding_b200 import ocrdec
    rng = np.random.default_rng(R * 1000 + K)
    Wb = synth.f32_to_bf16_bits(rng.standard_normal((N, K), dtype=np.float32) * 0.02)
    gb = synth.f32_to_bf16_bits(1 + 0.1 * rng.standard_normal(K, dtype=np.float32))
    x = rng.standard_normal((R, K), dtype=np.float32) * 3
    Wf, gf = O.bf16_bits_to_f32(Wb), O.bf16_bits_to_f32(gb)
    xn = O.rmsnorm(x, gf, 1e-6)
    want = xn @ Wf.T
    bound = _split_bound(xn, Wf)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    y = torch.empty((R, N), dtype=torch.float32, device="cuda")
    ocrdec.op_norm_gemv(t(Wb.view(np.int16)), t(x), t(gb.view(np.int16)), 1e-6, y, ocrdec.op_scratch())
    got = y.cpu().numpy()
    assert np.all(np.abs(got - want) <= bound), np.max(np.abs(got - want) - bound)


@pytest.mark.parametrize("R,N,K", [(1, 4096, 256), (4, 4104, 256), (2, 129280, 1280)])
def test_op_lm_argmax(R, N, K):
    import torch
    from speculative_moe_decoding_b200 import ocrdec
    rng = np.random.default_rng(N + R)
    Wb = synth.f32_to_bf16_bits(rng.standard_normal((N, K), dtype=np.float32) * 0.02)
    gb = synth.f32_to_bf16_bits(np.ones(K, np.float32))
    x = rng.standard_normal((R, K), dtype=np.float32)
    Wf = O.bf16_bits_to_f32(Wb)
    xn = O.rmsnorm(x, np.ones(K, np.float32), 1e-6)
    want = xn @ Wf.T
    bound = _split_bound(xn, Wf)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    tok = torch.empty(R, dtype=torch.int32, device="cuda")
    logits = torch.empty((R, N), dtype=torch.float32, device="cuda")
    ocrdec.op_lm_argmax(t(Wb.view(np.int16)), t(x), t(gb.view(np.int16)), 1e-6, tok, logits, ocrdec.op_scratch())
    got = logits.cpu().numpy()
    assert np.all(np.abs(got - want) <= bound)
    tk = tok.cpu().numpy()
    for r in range(R):
        assert tk[r] == int(np.argmax(got[r]))  # exact argmax of the kernel's own logits (ties: lower index)
        srt = np.sort(want[r])
        if srt[-1] - srt[-2] > 2 * bound[r].max():
            assert tk[r] == int(np.argmax(want[r]))


# ---------------------------------------------------------------- decoder parity
def test_greedy_decode_matches_oracle_teacher_forced(dec, orc, inputs, k0_tokens):
    """Oracle runs over the GPU's own token sequence; the GPU's greedy choice must
    equal the oracle's argmax wherever the oracle's margin is >= 0.1."""
    st = O.prefill(orc, inputs.visual, inputs.prompt)
    C = W.n_visual + W.n_prompt
    toks = list(k0_tokens)
    n_checked = 0
    # the first token comes from the prefill
    for i in range(1, len(toks)):
        out = orc.forward_rows(orc.embed([toks[i - 1]]), [C + i - 1], st.cache)
        lg = out.logits[0]
        if O.top2_margin(lg) >= MARGIN:
            assert toks[i] == O.greedy_argmax(lg), i
            n_checked += 1
    assert n_checked >= len(toks) // 3


def test_hidden_and_logits_parity(dec, orc, inputs):
    """Per-layer residual stream and logits of one verify pass (k = 3 rows of
    proposals) against the oracle at the same positions."""
    import torch
    vis, prm = to_dev(inputs)
    d, L, V = synth.TINY.d_model, synth.TINY.n_layers, synth.TINY.vocab
    hid = torch.zeros((L, 8, d), dtype=torch.float32, device="cuda")
    lg = torch.zeros((8, V), dtype=torch.float32, device="cuda")
    dec.set_forced_acceptance(None, None, None, ())
    first = int(dec.prefill(0, vis, prm).item())
    for _ in range(5):
        dec.verify_commit(1, 0)
    torch.cuda.synchronize()
    n = dec.stats(0).kv_len
    bonus = dec.stats(0).bonus
    props = torch.tensor([7, 1234, 4095], dtype=torch.int32, device="cuda")
    dec.set_debug_taps(hid, lg)
    dec.verify_commit(1, 3, props)
    dec.set_debug_taps(None, None)
    torch.cuda.synchronize()
    hid_np, lg_np = hid.cpu().numpy(), lg.cpu().numpy()
    # oracle: same committed prefix (GPU tokens), then the 4 verify rows
    hist = dec.history(0, W.n_visual + W.n_prompt, n - (W.n_visual + W.n_prompt) + 1).cpu().numpy()
    st = O.prefill(orc, inputs.visual, inputs.prompt)
    C = W.n_visual + W.n_prompt
    assert hist[0] == first
    for i in range(n - C):
        orc.forward_rows(orc.embed([hist[i]]), [C + i], st.cache)
    rows = [bonus, 7, 1234, 4095]
    for i, tok in enumerate(rows):
        out = orc.forward_rows(orc.embed([tok]), [n + i], st.cache)
        for l in range(L):
            a, b = hid_np[l, i], out.layer_hidden[l][0]
            rel = np.linalg.norm(a - b) / np.linalg.norm(b)
            assert rel <= HIDDEN_REL_L2, (i, l, rel)
        assert np.max(np.abs(lg_np[i] - out.logits[0])) <= LOGIT_ABS, i


@pytest.mark.parametrize("k", [1, 2, 3])
def test_speculative_is_bit_identical_to_k0(dec, inputs, k0_tokens, k):
    toks, st, _ = gpu_decode(dec, inputs, k, W.n_generate)
    assert np.array_equal(toks, k0_tokens)
    assert st.steps > 0 and 1.0 <= st.tau_sum / st.steps <= k + 1


@pytest.mark.parametrize("k", [1, 3])
def test_forced_acceptance_is_bit_identical_and_accepts(dec, inputs, k0_tokens, k):
    import torch
    C = W.n_visual + W.n_prompt
    n_pos = C + W.n_generate + 64
    ref = np.zeros(n_pos, np.int32)
    ref[C:C + W.n_generate] = k0_tokens
    tab = synth.make_forced_tables(202, n_pos, synth.TINY.vocab, 3)
    forced = (torch.from_numpy(ref).cuda(), torch.from_numpy(tab.u).cuda(), torch.from_numpy(tab.r).cuda(), tab.p)
    toks, st, _ = gpu_decode(dec, inputs, k, W.n_generate - 8, forced=forced)
    assert np.array_equal(toks, k0_tokens[:W.n_generate - 8])
    tau = st.tau_sum / st.steps
    assert tau > 1.0 + 0.5 * tab.p[0]  # proposals are mostly right, so most steps accept


def test_eager_path_equals_graph_and_draft_matches_oracle(dec, orc, inputs, k0_tokens):
    """Eager draft + verify commits the same tokens as the graph path, and each
    draft recursion's logits match the oracle's draft (same committed history,
    same previous proposals) within the logits tolerance."""
    import torch
    k = 3
    V = synth.TINY.vocab
    C = W.n_visual + W.n_prompt
    vis, prm = to_dev(inputs)
    taps = torch.zeros((3, 1, V), dtype=torch.float32, device="cuda")
    dec.set_forced_acceptance(None, None, None, ())
    dec.prefill(0, vis, prm)
    dec.set_draft_taps(taps)
    ost = O.prefill(orc, inputs.visual, inputs.prompt)
    compared = 0
    try:
        for step in range(12):
            p = dec.draft(1, k)[:k].cpu().numpy().copy()
            lg = taps[:, 0].cpu().numpy()
            ologits = []
            oprops = O.draft_propose(orc, ost, k, ologits)
            for j in range(k):
                assert np.max(np.abs(lg[j] - ologits[j])) <= LOGIT_ABS, (step, j)
                compared += 1
                if oprops[j] != p[j]:
                    break  # later recursions see different draft tokens
            committed, _ = dec.verify_commit(1, k, torch.from_numpy(p).cuda())
            g = committed[:k + 1].cpu().numpy()
            # teacher forcing: the oracle commits the GPU's tokens (its own argmax may
            # differ at near-ties), keeping both draft states on the same history
            O.verify_commit(orc, ost, list(p), forced_g=[int(t) for t in g])
        n = dec.stats(0).n_generated
        gpu_hist = dec.history(0, C, n).cpu().numpy()
        assert np.array_equal(gpu_hist[:min(n, 32)], k0_tokens[:min(n, 32)])
    finally:
        dec.set_draft_taps(None)
    assert compared >= 12


def test_capacity_overflow_sets_status_and_stops(tiny_bits, inputs):
    import torch
    d = make_decoder(synth.TINY, tiny_bits, max_k=3, max_batch=1, kv_capacity=96)
    try:
        vis, prm = to_dev(inputs)
        d.prefill(0, vis, prm)  # C = 80; every step commits >= 1 token
        for _ in range(20):
            d.step(1, 3)
        torch.cuda.synchronize()
        from speculative_moe_decoding_b200 import ocrdec
        assert d.status() == ocrdec.ECAPACITY
        st = d.stats(0)
        assert st.kv_len + 4 > 96 and st.kv_len <= 96
        kv = st.kv_len
        d.step(1, 3)
        assert d.stats(0).kv_len == kv  # no device work while the status is set
        d.clear_status()
        assert d.status() == 0
    finally:
        d.close()


def test_runs_are_deterministic(tiny_bits, inputs, k0_tokens):
    d = make_decoder(synth.TINY, tiny_bits, max_k=3, max_batch=1, kv_capacity=256)
    try:
        toks, _, _ = gpu_decode(d, inputs, 2, W.n_generate)
        assert np.array_equal(toks, k0_tokens)
    finally:
        d.close()
