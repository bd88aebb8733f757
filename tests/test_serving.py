"""Slot refill for batched serving (``serving.serve``) on the CPU: with a
scripted decoder (bookkeeping, capacity) and with the oracle (every request's
output equals its own greedy decode, whatever shares its pass)."""
from types import SimpleNamespace

import numpy as np
import pytest

from oracle import decoder as O
from speculative_moe_decoding_b200 import serving, synth


class ScriptedDecoder:
    """Commits 1..k+1 tokens per slot per step (seeded); token i of a request
    is a function of (its prompt's first token, i), so outputs identify their
    request.  Asserts that no slot exceeds its KV capacity."""

    def __init__(self, cap: int, seed: int = 0):
        self.cap = cap
        self.rng = np.random.default_rng(seed)
        self.slots = {}
        self.prefills = 0
        self.steps = 0

    @staticmethod
    def token(key: int, i: int) -> int:
        return (key * 7919 + i * 31) % 50021

    def prefill(self, slot, visual, prompt):
        n_ctx = len(visual) + len(prompt)
        key = int(prompt[0])
        self.slots[slot] = SimpleNamespace(key=key, n_context=n_ctx, toks=[self.token(key, 0)], kv=n_ctx)
        self.prefills += 1

    def step(self, batch, k):
        counts = np.zeros(batch, np.int32)
        for s in range(batch):
            st = self.slots[s]
            # the pass writes K/V at kv .. kv + k (the library's capacity check)
            assert st.kv + k + 1 <= self.cap, "slot decoded past its capacity"
            m = int(self.rng.integers(1, k + 2))
            for _ in range(m):
                st.toks.append(self.token(st.key, len(st.toks)))
            st.kv += m
            counts[s] = m
        self.steps += 1
        return None, counts

    def stats(self, slot):
        st = self.slots[slot]
        return SimpleNamespace(n_context=st.n_context, n_generated=len(st.toks))

    def history(self, slot, start, n):
        st = self.slots[slot]
        return np.array(st.toks[start - st.n_context:start - st.n_context + n])


def _requests(lengths, n_visual=5, n_prompt=3):
    return [serving.Request(rid=i, visual=np.zeros((n_visual, 4), np.float32),
                            prompt=np.array([100 + i] + [0] * (n_prompt - 1), np.int32), n_generate=L)
            for i, L in enumerate(lengths)]


@pytest.mark.parametrize("batch,k", [(1, 0), (3, 1), (4, 3)])
def test_every_request_gets_exactly_its_tokens(batch, k):
    lengths = [1, 7, 30, 2, 15, 15, 9, 40, 3]
    reqs = _requests(lengths)
    dec = ScriptedDecoder(cap=serving.required_capacity(reqs, k))
    res = serving.serve(dec, reqs, batch, k, max_steps=500)
    assert sorted(res.outputs) == list(range(len(reqs)))
    for r in reqs:
        want = [ScriptedDecoder.token(100 + r.rid, i) for i in range(r.n_generate)]
        assert list(res.outputs[r.rid]) == want, r.rid
    assert res.useful_tokens == sum(lengths)
    assert dec.prefills >= len(reqs)


def test_single_token_requests_are_collected_without_a_step():
    reqs = _requests([1, 1, 1])
    dec = ScriptedDecoder(cap=serving.required_capacity(reqs, 1))
    res = serving.serve(dec, reqs, 2, 1, max_steps=10)
    assert res.steps == 0 and dec.steps == 0
    for r in reqs:
        assert list(res.outputs[r.rid]) == [ScriptedDecoder.token(100 + r.rid, 0)]


def test_fewer_requests_than_slots_and_empty_queue():
    reqs = _requests([4, 6])
    dec = ScriptedDecoder(cap=serving.required_capacity(reqs, 2))
    res = serving.serve(dec, reqs, 4, 2, max_steps=100)
    assert sorted(res.outputs) == [0, 1]
    assert serving.serve(dec, [], 2, 1).steps == 0
    with pytest.raises(ValueError):
        serving.serve(dec, reqs, 0, 1)


class OracleSlots:
    """The serving interface over the oracle: one SeqState per slot; a step
    drafts k tokens with the real draft and verifies them."""

    def __init__(self, orc):
        self.orc = orc
        self.st = {}

    def prefill(self, slot, visual, prompt):
        self.st[slot] = O.prefill(self.orc, visual, list(prompt))

    def step(self, batch, k):
        counts = np.zeros(batch, np.int32)
        for s in range(batch):
            props = O.draft_propose(self.orc, self.st[s], k) if k > 0 else []
            counts[s] = len(O.verify_commit(self.orc, self.st[s], props))
        return None, counts

    def stats(self, slot):
        st = self.st[slot]
        return SimpleNamespace(n_context=min(st.tokens), n_generated=st.n_generated)

    def history(self, slot, start, n):
        return np.array([self.st[slot].tokens[p] for p in range(start, start + n)])


def test_refilled_slots_decode_like_a_single_sequence():
    m = synth.TINY
    bits, _ = synth.make_weights(m, synth.WORKLOADS["tiny"].weight_seed, workers=1)
    orc = O.Oracle(m.as_dict(), bits)
    reqs = []
    for i, (nv, L) in enumerate([(12, 9), (20, 14), (8, 6)]):
        inp = synth.make_inputs(m, 300, nv, 4, index=i)
        reqs.append(serving.Request(rid=i, visual=inp.visual, prompt=inp.prompt, n_generate=L))
    res = serving.serve(OracleSlots(orc), reqs, 2, 2, max_steps=100)
    for r in reqs:
        want = O.decode(orc, O.prefill(orc, r.visual, list(r.prompt), with_draft=False), 0, r.n_generate)
        assert list(res.outputs[r.rid]) == list(want[:r.n_generate]), r.rid
