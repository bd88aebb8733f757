"""The pages' metric arithmetic and the forced acceptance model."""
import os

import numpy as np
import pytest

from oracle import decoder as O
from speculative_moe_decoding_b200 import metrics, synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _l4_rows():
    rows = []
    for line in open(os.path.join(GOLDEN, "l4_speculative_table.txt")):
        if line.startswith("#") or not line.strip():
            continue
        mode, k, tps, s, acc, tau, c = line.split()
        rows.append(dict(mode=mode, k=int(k), tps=float(tps), s=float(s),
                         acc=None if acc == "-" else float(acc) / 100,
                         tau=None if tau == "-" else float(tau), c=float(c)))
    return rows


def test_l4_table_identities():
    """c = tau / S, S = tok/s over the same mode's k = 0 row, acceptance = (tau-1)/k,
    each to the table's printed rounding."""
    rows = _l4_rows()
    base = {r["mode"]: r["tps"] for r in rows if r["k"] == 0}
    for r in rows:
        assert abs(metrics.speedup(r["tps"], base[r["mode"]]) - r["s"]) <= 0.006, r
        if r["k"] == 0:
            continue
        assert abs(metrics.step_cost(r["tau"], r["s"]) - r["c"]) <= 0.011, r
        assert abs(metrics.acceptance_rate(r["tau"], r["k"]) - r["acc"]) <= 0.006, r


def test_pages_per_second_identity():
    for line in open(os.path.join(GOLDEN, "serving_throughput.txt")):
        if line.startswith("#") or not line.strip():
            continue
        _, tps, tpp, pps = line.split()
        assert abs(metrics.pages_per_s(float(tps), float(tpp)) - float(pps)) <= 0.006


def test_expected_tau_against_l4_table():
    """The per-depth acceptance probabilities (0.83, 0.69, 0.58) give E[tau]
    within about 1 % of the printed tau at k = 1, 2, 3."""
    rows = {(r["mode"], r["k"]): r for r in _l4_rows()}
    p = (0.83, 0.69, 0.58)
    for k in (1, 2, 3):
        e = metrics.expected_tau(p[:k])
        assert abs(e / rows[("eager", k)]["tau"] - 1) < 0.012, (k, e)
    assert metrics.expected_tau([]) == 1.0
    assert abs(metrics.expected_tau([0.5, 0.5]) - 1.75) < 1e-12


@pytest.mark.parametrize("k", [1, 2, 3])
def test_forced_stream_tau_statistics(k):
    """Under an ideal verifier (greedy token = reference token) the forced
    stream's mean tau matches 1 + p1 + p1 p2 + ... within 3 sigma."""
    V = 129280
    n_steps = 6000
    n_pos = n_steps * (k + 1) + 16
    tab = synth.make_forced_tables(202, n_pos, V, 3)
    rng = np.random.default_rng(99)
    ref_arr = rng.integers(0, V, n_pos)
    ref = {i: int(t) for i, t in enumerate(ref_arr)}
    n = 0
    taus = []
    for _ in range(n_steps):
        props = O.forced_proposals(ref, n, k, tab.u, tab.r, tab.p, V)
        a = 0
        while a < k and props[a] == ref[n + a + 1]:
            a += 1
        for j in range(a, k):  # a miss is never the reference token
            if j == a:
                assert props[j] != ref[n + j + 1]
        taus.append(a + 1)
        n += a + 1
    taus = np.array(taus, float)
    e = metrics.expected_tau(tab.p[:k])
    sigma = taus.std() / np.sqrt(len(taus))
    assert abs(taus.mean() - e) < 3 * sigma + 1e-9, (taus.mean(), e, sigma)


def test_forced_miss_is_uniform_over_other_tokens():
    V = 7
    tab = synth.make_forced_tables(5, 20000, V, 1, p=(0.0,))
    ref = {i: 3 for i in range(20001)}
    seen = np.zeros(V, int)
    for n in range(0, 20000 - 1):
        seen[O.forced_proposals(ref, n, 1, tab.u, tab.r, tab.p, V)[0]] += 1
    assert seen[3] == 0
    others = seen[np.arange(V) != 3]
    assert others.min() > 0.9 * others.mean() and others.max() < 1.1 * others.mean()


def test_batch_workload_shapes():
    """The batched-serving stand-in: lengths lognormal with mean 1,085 capped at
    4,096, visual counts 256 + 100 n with n uniform on 0..9."""
    from speculative_moe_decoding_b200 import synth
    vis, lengths = synth.make_batch_sequences(synth.WORKLOADS["full_batch32"].input_seed, 40000)
    assert lengths.min() >= 1 and lengths.max() <= 4096
    assert abs(lengths.mean() - 1085) < 0.01 * 1085
    # lognormal: the median is exp(mu) = 1085 * exp(-sigma^2 / 2)
    assert abs(np.median(lengths) - 1085 * np.exp(-0.125)) < 0.02 * 1085
    assert set(np.unique(vis)) == {256 + 100 * n for n in range(10)}
    counts = np.bincount((vis - 256) // 100, minlength=10)
    assert counts.min() > 0.9 * len(vis) / 10
    again = synth.make_batch_sequences(synth.WORKLOADS["full_batch32"].input_seed, 40000)
    assert np.array_equal(again[1], lengths)
