"""GPU paths the single-slot, short-context tests do not reach.

* Two slots in one pass (8 rows at k = 3): every kernel treats a row on its
  own (batch invariance), so each slot commits exactly the tokens it commits
  alone.
* A long context (1,708 positions): the attention kernel then takes its
  chunks in more than one group and rescales its online softmax between
  them; hidden states and logits of one verify pass are compared with the
  oracle, and teacher-forced greedy tokens with the oracle's argmax."""
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


def test_two_slots_commit_what_each_commits_alone(tiny_bits):
    import torch
    ins = [synth.make_inputs(synth.TINY, W.input_seed, W.n_visual, W.n_prompt, index=i) for i in (0, 1)]
    n_ref = 48
    alone = make_decoder(synth.TINY, tiny_bits, max_k=3, max_batch=1, kv_capacity=256)
    try:
        refs = [gpu_decode(alone, inp, 0, n_ref)[0] for inp in ins]
    finally:
        alone.close()
    assert not np.array_equal(refs[0], refs[1])
    C = W.n_visual + W.n_prompt
    dec = make_decoder(synth.TINY, tiny_bits, max_k=3, max_batch=2, kv_capacity=256)
    try:
        dec.set_forced_acceptance(None, None, None, ())
        for slot, inp in enumerate(ins):
            vis, prm = to_dev(inp)
            dec.prefill(slot, vis, prm)
        for _ in range(40):
            dec.step(2, 3)
            if min(dec.stats(0).n_generated, dec.stats(1).n_generated) >= n_ref - 4:
                break
        torch.cuda.synchronize()
        assert dec.status() == 0
        for slot in (0, 1):
            n = min(dec.stats(slot).n_generated, n_ref)
            assert n >= 16
            got = dec.history(slot, C, n).cpu().numpy()
            assert np.array_equal(got, refs[slot][:n]), slot
    finally:
        dec.close()


def test_long_context_matches_oracle(tiny_bits):
    import torch
    n_visual, n_prompt = 1700, 8
    C = n_visual + n_prompt
    inp = synth.make_inputs(synth.TINY, W.input_seed, n_visual, n_prompt, index=3)
    orc = O.Oracle(synth.TINY.as_dict(), tiny_bits)
    d, L, V = synth.TINY.d_model, synth.TINY.n_layers, synth.TINY.vocab
    dec = make_decoder(synth.TINY, tiny_bits, max_k=3, max_batch=1, kv_capacity=2048)
    try:
        vis, prm = to_dev(inp)
        dec.set_forced_acceptance(None, None, None, ())
        first = int(dec.prefill(0, vis, prm).item())
        n_dec = 12
        for _ in range(n_dec):
            dec.verify_commit(1, 0)
        torch.cuda.synchronize()
        st = dec.stats(0)
        n, bonus = st.kv_len, st.bonus
        toks = dec.history(0, C, n - C + 1).cpu().numpy()
        hid = torch.zeros((L, 8, d), dtype=torch.float32, device="cuda")
        lg = torch.zeros((8, V), dtype=torch.float32, device="cuda")
        props = torch.tensor([11, 2047, 4000], dtype=torch.int32, device="cuda")
        dec.set_debug_taps(hid, lg)
        dec.verify_commit(1, 3, props)
        dec.set_debug_taps(None, None)
        torch.cuda.synchronize()
        assert dec.status() == 0
        hid_np, lg_np = hid.cpu().numpy(), lg.cpu().numpy()
    finally:
        dec.close()
    ost = O.prefill(orc, inp.visual, inp.prompt, with_draft=False)
    assert toks[0] == first
    n_checked = 0
    for i in range(n - C):
        out = orc.forward_rows(orc.embed([toks[i]]), [C + i], ost.cache)
        if O.top2_margin(out.logits[0]) >= MARGIN:
            assert toks[i + 1] == O.greedy_argmax(out.logits[0]), i
            n_checked += 1
    assert n_checked >= (n - C) // 3
    for i, tok in enumerate([bonus, 11, 2047, 4000]):
        out = orc.forward_rows(orc.embed([tok]), [n + i], ost.cache)
        for l in range(L):
            a, b = hid_np[l, i], out.layer_hidden[l][0]
            rel = np.linalg.norm(a - b) / np.linalg.norm(b)
            assert rel <= HIDDEN_REL_L2, (i, l, rel)
        assert np.max(np.abs(lg_np[i] - out.logits[0])) <= LOGIT_ABS, i
