"""Full-size GPU checks at the benchmark's own shapes.

* Losslessness at the benchmark's configuration (model page: speculative
  output bit-identical to plain autoregressive decoding): context 256 visual +
  32 prompt rows, k = 3 with the real draft and with the forced acceptance
  stream of the benchmark, 96 generated tokens, all bit-identical to the
  library's own k = 0 run.
* The dynamic-resolution long context (1,156 visual + 64 prompt rows, Gundam
  mode's largest page) decoded to 1,604 positions, so the attention kernel
  runs its head-dim-128 chunks in two groups per CTA and rescales its online
  softmax between them: teacher-forced greedy tokens against the oracle over
  all 384 generated tokens, then the per-layer residual stream and the logits
  of one k = 3 verify pass at that length."""
import numpy as np
import pytest

from oracle import decoder as O
from speculative_moe_decoding_b200 import synth

from .gpu_util import gpu_decode, make_decoder, to_dev

pytestmark = pytest.mark.gpu

HIDDEN_REL_L2 = 1e-2
LOGIT_ABS = 5e-2
MARGIN = 0.1


def test_bench_workload_speculative_is_bit_identical_to_k0(full_bits):
    import torch
    m = synth.FULL
    w = synth.WORKLOADS["full_spec"]
    inp = synth.make_inputs(m, w.input_seed, w.n_visual, w.n_prompt)  # the benchmark's sequence
    C = w.n_visual + w.n_prompt
    n_gen, n_ref = 96, 160  # the reference runs past n_gen: steps overshoot by up to k + 1 tokens
    dec = make_decoder(m, full_bits, max_k=3, max_batch=1, kv_capacity=C + n_ref + 64)
    try:
        k0, _, _ = gpu_decode(dec, inp, 0, n_ref)
        ref_hist = dec.history(0, 0, C + n_ref).clone()
        # the real draft's proposals (random weights: mostly rejected)
        real, st_real, _ = gpu_decode(dec, inp, 3, n_gen)
        assert np.array_equal(real, k0[:n_gen])
        # the benchmark's forced acceptance stream (p = 0.83 / 0.69 / 0.58 per depth)
        tab = synth.make_forced_tables(w.stream_seed, C + n_ref, m.vocab, 3, w.accept_p)
        forced = (ref_hist, torch.from_numpy(tab.u).cuda(), torch.from_numpy(tab.r).cuda(), tab.p)
        got, st_f, _ = gpu_decode(dec, inp, 3, n_gen, forced=forced)
        assert dec.status() == 0
        assert np.array_equal(got, k0[:n_gen])
        tau = st_f.tau_sum / st_f.steps
        assert 2.0 < tau <= 4.0, tau  # acceptance happened (expected tau about 2.7)
        assert sum(st_f.accepted_hist) == st_f.steps and st_f.accepted_hist[3] > 0
    finally:
        dec.close()


def test_long_context_full_size_matches_oracle(full_bits):
    import torch
    m = synth.FULL
    w = synth.WORKLOADS["full_long"]
    inp = synth.make_inputs(m, w.input_seed, w.n_visual, w.n_prompt)
    C = w.n_visual + w.n_prompt
    n_dec = 384
    d, L, V = m.d_model, m.n_layers, m.vocab
    dec = make_decoder(m, full_bits, max_k=3, max_batch=1, kv_capacity=C + n_dec + 64)
    try:
        vis, prm = to_dev(inp)
        dec.set_forced_acceptance(None, None, None, ())
        first = int(dec.prefill(0, vis, prm).item())
        for _ in range(n_dec):
            dec.step(1, 0)
        torch.cuda.synchronize()
        st = dec.stats(0)
        n, bonus = st.kv_len, st.bonus
        assert n == C + n_dec
        assert (n + 3) // 64 + 1 > 3 * 8  # more than three chunks for some CTA: two groups
        toks = dec.history(0, C, n - C + 1).cpu().numpy()
        hid = torch.zeros((L, 8, d), dtype=torch.float32, device="cuda")
        lg = torch.zeros((8, V), dtype=torch.float32, device="cuda")
        props_l = [11, 65000, 129279]
        dec.set_debug_taps(hid, lg)
        dec.verify_commit(1, 3, torch.tensor(props_l, dtype=torch.int32, device="cuda"))
        dec.set_debug_taps(None, None)
        torch.cuda.synchronize()
        assert dec.status() == 0
        hid_np, lg_np = hid.cpu().numpy(), lg.cpu().numpy()
    finally:
        dec.close()
    orc = O.Oracle(m.as_dict(), full_bits)
    ost = O.prefill(orc, inp.visual, inp.prompt, with_draft=False)
    n_checked = 0
    for i in range(n - C):
        out = orc.forward_rows(orc.embed([int(toks[i])]), [C + i], ost.cache)
        if O.top2_margin(out.logits[0]) >= MARGIN:
            assert toks[i + 1] == O.greedy_argmax(out.logits[0]), i
            n_checked += 1
    assert n_checked >= (n - C) // 4, n_checked
    for i, tok in enumerate([bonus] + props_l):
        out = orc.forward_rows(orc.embed([tok]), [n + i], ost.cache)
        for l in range(L):
            a, b = hid_np[l, i], out.layer_hidden[l][0]
            rel = np.linalg.norm(a - b) / np.linalg.norm(b)
            assert rel <= HIDDEN_REL_L2, (i, l, rel)
        assert np.max(np.abs(lg_np[i] - out.logits[0])) <= LOGIT_ABS, i
    assert first == toks[0]
