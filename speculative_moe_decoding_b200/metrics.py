"""Speculative-decoding metrics as the jina-ocr-v1 pages define them.

Section "Speculative decoding on L4" of the news article: tau is the mean number
of tokens committed per speculative step including the bonus token; S is the
speed-up over plain greedy decoding; c = tau / S is the cost of one speculative
step measured in plain autoregressive steps.  The acceptance column equals
(tau - 1) / k.  The serving figure caption defines pages/s as output tokens/s
divided by output tokens per page.
"""
from __future__ import annotations

from typing import Sequence


def speedup(tok_per_s: float, base_tok_per_s: float) -> float:
    return tok_per_s / base_tok_per_s


def step_cost(tau: float, s: float) -> float:
    """c = tau / S."""
    return tau / s


def acceptance_rate(tau: float, k: int) -> float:
    """Fraction of the k drafted tokens that were accepted, (tau - 1) / k."""
    return (tau - 1.0) / k


def pages_per_s(tok_per_s: float, tok_per_page: float) -> float:
    return tok_per_s / tok_per_page


def expected_tau(p: Sequence[float]) -> float:
    """E[tau] when depth j is accepted independently with probability p[j-1]
    given all shallower depths were: 1 + p1 + p1 p2 + ..."""
    tau, run = 1.0, 1.0
    for pj in p:
        run *= pj
        tau += run
    return tau
