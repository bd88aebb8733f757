"""Parity of the CUDA path with the oracle on the full-size model (12 layers,
d = 1280, 64 + 2 experts, top-6, V = 129,280, FastMTP draft), at a short
context so the oracle finishes in seconds: the first generated token and
teacher-forced greedy tokens, the per-layer residual stream and the logits of
one k = 3 verify pass, and the draft's logits for every recursion.  The same
kernels, launch shapes and tolerances as the bench's workload; only the
context is shorter (40 rows instead of 288)."""
import numpy as np
import pytest

from oracle import decoder as O
from speculative_moe_decoding_b200 import synth

from .gpu_util import make_decoder, to_dev

pytestmark = pytest.mark.gpu

HIDDEN_REL_L2 = 1e-2
LOGIT_ABS = 5e-2
MARGIN = 0.1


def test_full_model_matches_oracle(full_bits):
    import torch
    m = synth.FULL
    w = synth.WORKLOADS["full_spec"]
    inp = synth.make_inputs(m, w.input_seed, 32, 8, index=5)
    C = 40
    d, L, V = m.d_model, m.n_layers, m.vocab
    dec = make_decoder(m, full_bits, max_k=3, max_batch=1, kv_capacity=256)
    try:
        vis, prm = to_dev(inp)
        dec.set_forced_acceptance(None, None, None, ())
        first = int(dec.prefill(0, vis, prm).item())
        for _ in range(4):
            dec.verify_commit(1, 0)
        torch.cuda.synchronize()
        st = dec.stats(0)
        n, bonus = st.kv_len, st.bonus
        toks = dec.history(0, C, n - C + 1).cpu().numpy()
        # one draft of k = 3 with its logits, then a verify pass with taps
        dtaps = torch.zeros((3, 1, V), dtype=torch.float32, device="cuda")
        dec.set_draft_taps(dtaps)
        props = dec.draft(1, 3)[:3].clone()
        dec.set_draft_taps(None)
        hid = torch.zeros((L, 8, d), dtype=torch.float32, device="cuda")
        lg = torch.zeros((8, V), dtype=torch.float32, device="cuda")
        dec.set_debug_taps(hid, lg)
        dec.verify_commit(1, 3, props)
        dec.set_debug_taps(None, None)
        torch.cuda.synchronize()
        assert dec.status() == 0
        p = props.cpu().numpy()
        dlg, hid_np, lg_np = dtaps[:, 0].cpu().numpy(), hid.cpu().numpy(), lg.cpu().numpy()
    finally:
        dec.close()

    orc = O.Oracle(m.as_dict(), full_bits)
    ost = O.prefill(orc, inp.visual, inp.prompt)
    # teacher forcing: the oracle continues on the GPU's tokens; the GPU's choice
    # must be the oracle's argmax wherever the oracle's margin is >= 0.1
    ost.bonus = int(toks[0])
    ost.tokens[C] = int(toks[0])
    n_checked = 0
    for i in range(n - C):
        rec = []
        O.verify_commit(orc, ost, [], record=rec, forced_g=[int(toks[i + 1])])
        lg0 = rec[0][2].logits[0]
        if O.top2_margin(lg0) >= MARGIN:
            assert toks[i + 1] == O.greedy_argmax(lg0), i
            n_checked += 1
    assert ost.kv_len == n and ost.bonus == bonus
    # draft: the oracle's recursions on the same history, logits within tolerance
    ologits = []
    oprops = O.draft_propose(orc, ost, 3, ologits)
    for j in range(3):
        assert np.max(np.abs(dlg[j] - ologits[j])) <= LOGIT_ABS, j
        if oprops[j] != p[j]:
            break  # later recursions see different draft tokens
    # verify pass: per-layer residual and logits of the 4 rows
    for i, tok in enumerate([bonus] + [int(t) for t in p]):
        out = orc.forward_rows(orc.embed([tok]), [n + i], ost.cache)
        for l in range(L):
            a, b = hid_np[l, i], out.layer_hidden[l][0]
            rel = np.linalg.norm(a - b) / np.linalg.norm(b)
            assert rel <= HIDDEN_REL_L2, (i, l, rel)
        assert np.max(np.abs(lg_np[i] - out.logits[0])) <= LOGIT_ABS, i
