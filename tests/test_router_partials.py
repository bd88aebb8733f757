"""The decomposition behind the router partials.

The attention kernel writes, for each of 8 output-row blocks of the new
residual x, the dot products of that block's columns of W_r with g * x and
the block's sum of squares of x; the expert gate/up GEMV finishes the router
logits as (sum of the 8 dot products) * rsqrt(sum of the 8 sums / d + eps).
Because RMSNorm is a per-row scale, that equals the router applied to
RMSNorm(x) * g, which is how the oracle (and the model definition) computes
it.  These CPU checks pin the decomposition, in the kernel's block order,
against the oracle's rmsnorm and route."""
import numpy as np

from oracle import decoder as O

BLOCKS = 8


def block_partials(x, g, w_r):
    d = x.shape[-1]
    nb = d // BLOCKS
    dots = np.zeros((x.shape[0], BLOCKS, w_r.shape[0]))
    ss = np.zeros((x.shape[0], BLOCKS))
    for k in range(BLOCKS):
        cols = slice(k * nb, (k + 1) * nb)
        dots[:, k] = (g[cols] * x[:, cols]) @ w_r[:, cols].T
        ss[:, k] = np.sum(x[:, cols] ** 2, axis=-1)
    return dots, ss


def logits_from_partials(dots, ss, d, eps):
    dot = np.zeros(dots.shape[::2])
    s = np.zeros(ss.shape[0])
    for k in range(BLOCKS):  # block order, as the GEMV adds them
        dot = dot + dots[:, k]
        s = s + ss[:, k]
    return dot / np.sqrt(s / d + eps)[:, None]


def test_partials_give_the_router_logits():
    rng = np.random.default_rng(7)
    for d, E in ((256, 8), (1280, 64)):
        x = rng.normal(0, 3, (4, d))
        g = rng.uniform(0.5, 1.5, d)
        w_r = rng.normal(0, 0.02, (E, d))
        eps = 1e-6
        want = O.rmsnorm(x.astype(np.float64), g, eps) @ w_r.T
        got = logits_from_partials(*block_partials(x, g, w_r), d, eps)
        np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-7)  # the oracle normalises in float32


def test_partials_route_like_the_oracle():
    rng = np.random.default_rng(11)
    d, E, K = 1280, 64, 6
    x = rng.normal(0, 1, (8, d)).astype(np.float32)
    g = np.ones(d, dtype=np.float32)
    w_r = rng.normal(0, 0.02, (E, d)).astype(np.float32)
    ids_o, gates_o, _ = O.route(O.rmsnorm(x, g, 1e-6), w_r, K)
    lg = logits_from_partials(*block_partials(x.astype(np.float64), g.astype(np.float64),
                                              w_r.astype(np.float64)), d, 1e-6)
    p = np.exp(lg - lg.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    ids = np.argsort(-p, axis=-1, kind="stable")[:, :K]
    assert np.array_equal(np.sort(ids, -1), np.sort(ids_o, -1))
    np.testing.assert_allclose(np.take_along_axis(p, ids_o, -1), gates_o, rtol=1e-5)


def test_gain_and_block_mistakes_are_caught():
    # a dropped gain or a block that skips its last column changes the logits
    rng = np.random.default_rng(3)
    d, E = 256, 8
    x = rng.normal(0, 1, (2, d))
    g = rng.uniform(0.5, 1.5, d)
    w_r = rng.normal(0, 0.02, (E, d))
    want = O.rmsnorm(x, g, 1e-6) @ w_r.T
    no_gain = logits_from_partials(*block_partials(x, np.ones(d), w_r), d, 1e-6)
    assert not np.allclose(no_gain, want, rtol=1e-5, atol=1e-7)
    dots, ss = block_partials(x, g, w_r)
    ss[:, -1] -= x[:, -1] ** 2
    assert not np.allclose(logits_from_partials(dots, ss, d, 1e-6), want, rtol=1e-5, atol=1e-7)
