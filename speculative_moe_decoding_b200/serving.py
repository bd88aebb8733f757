"""Slot refill for batched serving: the host-side loop of the batched
workload (32 concurrent sequences in the pages' A100 serving figure; here any
batch the library's pass holds).

The library steps slots 0..batch-1 together (``step(batch, k)``); each slot
carries its own sequence state (KV length, pending draft pairs, history), so
sequences of different lengths share a pass.  This scheduler keeps every slot
busy: after each step it harvests the slots whose request has produced its
target number of tokens and prefills the next queued request into them.
Once the queue is empty a finished slot is re-prefilled with its own request
again (its further tokens are discarded), so no slot decodes past the KV
capacity while the others finish.

The decoder needs ``prefill(slot, visual, prompt)``, ``step(batch, k)``
(returning the step's committed tokens and their count per slot, as
``speculative_moe_decoding_b200.ocrdec.Decoder`` does) and
``history(slot, start, n)``.  The loop counts each slot's tokens on the host:
one after the prefill (its first token), then the step's counts, read with
one device-to-host copy per step.  A request whose target is already met after
its prefill (n_generate <= 1) is collected without a step."""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Any, Dict, List, Optional, Sequence

import numpy as np


@dataclass
class Request:
    rid: int
    visual: Any          # [n_visual, d] float32 (on the decoder's device)
    prompt: Any          # [n_prompt] int32
    n_generate: int      # tokens to produce (the prefill's first token included)


@dataclass
class ServeResult:
    outputs: Dict[int, np.ndarray] = field(default_factory=dict)  # rid -> its n_generate tokens
    steps: int = 0
    useful_tokens: int = 0   # tokens that belong to a request's output
    slot_steps: int = 0      # slot x step products spent on live requests


def required_capacity(requests: Sequence[Request], k: int, max_k: int = 3) -> int:
    """KV positions a slot needs for the longest request.  A slot steps while
    it has fewer than n_generate tokens, i.e. at kv_len <= context +
    n_generate - 2, and a pass writes K/V at kv_len .. kv_len + k; a prefill
    itself needs context + max_k + 2 (max_k of the decoder's config)."""
    return max(int(r.visual.shape[0]) + int(r.prompt.shape[0]) + max(r.n_generate + k, max_k) + 2
               for r in requests)


def serve(dec, requests: Sequence[Request], batch: int, k: int, max_steps: Optional[int] = None) -> ServeResult:
    """Runs every request to completion on ``batch`` slots at k draft tokens
    per step; returns each request's tokens and step counts."""
    if batch < 1:
        raise ValueError("batch must be at least 1")
    queue: List[Request] = list(requests)
    res = ServeResult()
    if not queue:
        return res
    slot_req: List[Optional[Request]] = [None] * batch
    live = [False] * batch  # the slot's request still needs tokens
    gen = [0] * batch       # tokens the slot's request has produced

    def fill(slot: int, req: Request, counts: bool):
        dec.prefill(slot, req.visual, req.prompt)
        slot_req[slot] = req
        live[slot] = counts
        gen[slot] = 1  # the prefill's first token

    def collect(slot: int) -> None:
        """Records a finished request and gives the slot its next one."""
        req = slot_req[slot]
        n_ctx = int(req.visual.shape[0]) + int(req.prompt.shape[0])
        toks = dec.history(slot, n_ctx, req.n_generate)
        res.outputs[req.rid] = np.asarray(toks.cpu() if hasattr(toks, "cpu") else toks).copy()
        res.useful_tokens += req.n_generate
        if queue:
            fill(slot, queue.pop(0), True)
        else:
            fill(slot, req, False)  # idle slot: start over, stay within capacity

    def harvest() -> None:
        # a refilled slot may be done at once (n_generate <= 1): loop until none is
        done = True
        while done:
            done = False
            for s in range(batch):
                if live[s] and gen[s] >= slot_req[s].n_generate:
                    collect(s)
                    done = True
                elif not live[s] and gen[s] >= slot_req[s].n_generate:
                    fill(s, slot_req[s], False)

    for s in range(batch):
        if queue:
            fill(s, queue.pop(0), True)
        else:  # fewer requests than slots: idle slots repeat the first request
            fill(s, requests[0], False)
    harvest()
    while any(live):
        if max_steps is not None and res.steps >= max_steps:
            raise RuntimeError(f"requests unfinished after {max_steps} steps")
        _, n_committed = dec.step(batch, k)
        counts = np.asarray(n_committed.cpu() if hasattr(n_committed, "cpu") else n_committed).reshape(-1)
        res.steps += 1
        res.slot_steps += sum(live)
        for s in range(batch):
            gen[s] += int(counts[s])
        harvest()
    return res
