"""MTP draft / verify: the oracle pinned by what the method and the
mathematics fix (CPU), then the library's kernels against the oracle (GPU)."""
import numpy as np
import pytest
import scipy.special

from oracle import spec as OS

RNG = np.random.default_rng(91)


# ---------------------------------------------------------------- oracle pins
def test_dist_is_the_library_softmax():
    for T in (0.5, 1.0, 3.0):
        l = RNG.normal(0, 4, 1000)
        assert np.allclose(OS.dist(l, T), scipy.special.softmax(l / T), rtol=1e-12, atol=0)
    l = np.array([0.0, -np.inf, 1.0, -np.inf])
    p = OS.dist(l, 1.0)
    assert p[1] == 0 and p[3] == 0 and np.isclose(p[2] / p[0], np.e)


def test_sample_closed_forms():
    n = 1000
    for u in (0.0, 0.1234, 0.5, 0.999999):
        assert OS.sample(np.ones(n), u) == int(np.floor(u * n))  # uniform weights: floor(u n)
    w = np.zeros(50)
    w[17] = 3.0
    assert all(OS.sample(w, u) == 17 for u in (0.0, 0.4, 0.99))  # one positive weight
    w = np.array([0.0, 0.0, 1.0, 0.0, 1.0, 0.0])
    assert OS.sample(w, 0.0) == 2 and OS.sample(w, 0.49) == 2 and OS.sample(w, 0.5) == 4  # boundary to the right
    # the draw is a function of the running sum: a random case by brute force
    w = RNG.random(200) * (RNG.random(200) < 0.3)
    for u in RNG.random(50):
        t = u * w.sum()
        i = OS.sample(w, u)
        assert w[:i].sum() <= t < w[: i + 1].sum()


def _first_token_distribution(target, drafts, vmap, T, G=64, verify=OS.verify):
    """Distribution of the first emitted token of one verify step with one
    draft: the draft row enumerated exactly with its probability q, the two
    uniforms on a G x G grid of cell midpoints."""
    V = target.shape[1]
    q = OS.dist(drafts[0], T)
    grid = (np.arange(G) + 0.5) / G
    out = np.zeros(V)
    for row in range(len(vmap)):
        if q[row] == 0:
            continue
        for ua in grid:
            for ur in grid:
                _, toks = verify(target, drafts, vmap, np.array([row]), np.array([ua, ur, 0.5]), T)
                out[toks[0]] += q[row] / (G * G)
    return out


def test_verify_preserves_the_target_distribution():
    """The point of the method: the first emitted token is distributed as the
    main model's p, whatever the draft distribution, including tokens outside
    the draft's map."""
    V, T = 7, 1.0
    vmap = np.array([1, 2, 4, 6])
    target = RNG.normal(0, 1.0, (2, V))
    drafts = RNG.normal(0, 1.5, (1, len(vmap)))
    got = _first_token_distribution(target, drafts, vmap, T)
    p = OS.dist(target[0], T)
    assert 0.5 * np.abs(got - p).sum() < 2.5 / 64


def test_the_distribution_pin_catches_an_inverted_ratio():
    """A planted mistake (keeping d with probability min(1, q/p)) moves the
    first-token distribution far from p."""
    V, T = 7, 1.0
    vmap = np.array([1, 2, 4, 6])
    rng = np.random.default_rng(5)
    target = rng.normal(0, 1.0, (2, V))
    drafts = rng.normal(0, 1.5, (1, len(vmap)))

    def wrong(target, drafts, vmap, rows, u, T):
        p, q = OS.dist(target[0], T), np.zeros(V)
        q[vmap] = OS.dist(drafts[0], T)
        d = int(vmap[rows[0]])
        if u[0] * p[d] < q[d]:  # inverted
            return 1, [d]
        return 0, [OS.sample(np.maximum(p - q, 0.0), u[1])]

    got = _first_token_distribution(target, drafts, vmap, T, G=32, verify=wrong)
    assert 0.5 * np.abs(got - OS.dist(target[0], T)).sum() > 0.1


def test_draft_equal_to_target_keeps_every_draft():
    V, n = 50, 3
    vmap = np.arange(V)
    target = RNG.normal(0, 2, (n + 1, V))
    for trial in range(20):
        u = RNG.random(2 * n + 1) * 0.999
        rows = np.array([OS.draft(target[j], vmap, 1.0, RNG.random())[1] for j in range(n)])
        a, toks = OS.verify(target, target[:n], vmap, rows, u, 1.0)
        assert a == n and toks[:n] == list(rows) and len(toks) == n + 1


def test_zero_target_probability_is_always_rejected_and_never_emitted():
    V, n = 40, 2
    vmap = np.arange(0, V, 2)
    target = RNG.normal(0, 1, (n + 1, V))
    target[0, vmap[3]] = -np.inf
    for ua in (0.0, 0.3, 0.99):
        a, toks = OS.verify(target, RNG.normal(0, 1, (n, len(vmap))), vmap, np.array([3, 0]),
                            np.array([ua, 0.5, 0.5, 0.5, 0.5]), 1.0)
        assert a == 0 and toks[0] != vmap[3] and len(toks) == 1


def test_greedy_is_argmax():
    V, n = 30, 3
    vmap = np.arange(5, 25)
    target = RNG.normal(0, 1, (n + 1, V))
    target[:, 5:25] -= 10.0  # only one draft can match: make row 0's best mapped
    target[0, 9] = 100.0
    best = [int(np.argmax(target[j])) for j in range(n + 1)]
    rows = np.array([9 - 5, 0, 0])
    a, toks = OS.verify(target, np.zeros((n, 20)), vmap, rows, np.zeros(2 * n + 1), 0.0)
    assert best[0] == 9 and a == 1 and toks == [9, best[1]]
    assert OS.draft(np.array([1.0, 3.0, 3.0, 2.0]), np.array([7, 8, 9, 10]), 0.0, 0.3) == (8, 1, 1.0)  # first max


def test_stops_at_the_first_rejection():
    V, n = 20, 3
    vmap = np.arange(V)
    target = np.zeros((n + 1, V))
    drafts = np.zeros((n, V))
    target[1, 4] = -np.inf  # position 1 rejects token 4 for any u
    u = np.array([0.1, 0.1, 0.1, 0.25, 0.5, 0.75, 0.5])
    a, toks = OS.verify(target, drafts, vmap, np.array([2, 4, 6]), u, 1.0)
    assert a == 1 and toks[0] == 2 and len(toks) == 2 and toks[1] != 4


def test_inverse_map():
    inv = OS.inverse_map(np.array([3, 0, 7]), 9)
    assert inv.tolist() == [1, -1, -1, 0, -1, -1, -1, 2, -1]
