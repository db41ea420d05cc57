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


# ---------------------------------------------------------------- device (GPU)
# fp32 on the device vs fp64 here: a draw or a keep decision may differ only
# where the oracle's margin to the decision boundary is below the fp32 error
# bound of the device's sums; elsewhere every integer result must match
# exactly.  A device running sum at any index is a chain of at most
# 7 (CTAs) + 31 (warps) + 31 (steps of 32) + 5 (scan levels) = 74 fp32
# additions of positive terms, so its relative error is below 74 * 2^-24 =
# 4.4e-6 of the total; expf adds 2 ulp per term.  Hence CDF_TOL = 5e-6 of the
# total mass for draws from p or q.  A residual weight max(0, p - q) carries
# the errors of both p and q (each normalised by such a sum): up to 1e-5 of
# the whole probability mass, plus its own sum's 5e-6 of R.  A keep decision
# u q < p compares two such quotients: KEEP_TOL = 2e-5 relative.
CDF_TOL = 5e-6
KEEP_TOL = 2e-5


def _torch():
    import torch

    return torch


def _dev(a, dtype):
    torch = _torch()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=dtype)).cuda()


def _check_draw(w, u, got, what, tol=None):
    """got must be a valid inverse-CDF draw of weights w at u (within `tol`,
    in the units of w; default CDF_TOL of the total), and equal to the
    oracle's unless u * total lies within tol of a boundary.  Returns whether
    the exact comparison applied."""
    w = np.asarray(w, dtype=np.float64)
    c = np.cumsum(w)
    total = c[-1]
    tol = CDF_TOL * total if tol is None else tol
    t = u * total
    want = OS.sample(w, u)
    lo = c[got - 1] if got > 0 else 0.0
    assert w[got] > 0, f"{what}: drew a zero-weight index {got}"
    assert lo - tol <= t <= c[got] + tol, f"{what}: {got} is not a valid draw (oracle {want})"
    lo_w = c[want - 1] if want > 0 else 0.0
    if min(t - lo_w, c[want] - t) > tol:
        assert got == want, f"{what}: {got} != oracle {want}"
        return True
    return False


def _synthetic_map(rng, V, n_map):
    return np.sort(rng.choice(V, n_map, replace=False)).astype(np.int32)


@pytest.mark.gpu
@pytest.mark.parametrize("n_map,T", [(65536, 1.0), (65536, 0.6), (1000, 2.0), (37, 1.0), (1, 1.0)])
def test_draft_parity(cuda_device, n_map, T):
    import bit_weight_gemv_q4_b200 as q4

    torch = _torch()
    rng = np.random.default_rng(n_map)
    V = max(248320, n_map)
    vmap = _synthetic_map(rng, V, n_map)
    z = rng.normal(0, 2.0, n_map).astype(np.float32)
    zd, md = _dev(z, np.float32), _dev(vmap, np.int32)
    row = torch.empty(1, dtype=torch.int32, device="cuda")
    tok = torch.empty_like(row)
    q = torch.empty(1, dtype=torch.float32, device="cuda")
    qref = OS.dist(z, T)
    exact = 0
    for u in list(rng.random(40)) + [0.0, 0.999999]:
        q4.q4_spec_draft(zd, n_map, md, T, _dev([u], np.float32), row, tok, q)
        torch.cuda.synchronize()
        r = int(row.item())
        exact += _check_draw(qref, float(np.float32(u)), r, f"draft u={u}")
        assert int(tok.item()) == vmap[r]
        assert abs(float(q.item()) - qref[r]) <= 1e-4 * qref[r] + 1e-12
    assert exact >= 25  # of 42: ~80 % of these draws lie farther than CDF_TOL from a boundary


@pytest.mark.gpu
def test_draft_greedy_is_first_maximum(cuda_device):
    import bit_weight_gemv_q4_b200 as q4

    torch = _torch()
    n_map = 65536
    z = np.random.default_rng(3).normal(0, 1, n_map).astype(np.float32)
    for pos in (0, 12345, 40000, n_map - 1):
        zz = z.copy()
        zz[pos] = 10.0
        zz[(pos + 7777) % n_map] = 10.0  # a tie: the lower index wins
        vmap = np.arange(n_map, dtype=np.int32) * 3
        row = torch.empty(1, dtype=torch.int32, device="cuda")
        tok, q = torch.empty_like(row), torch.empty(1, dtype=torch.float32, device="cuda")
        q4.q4_spec_draft(_dev(zz, np.float32), n_map, _dev(vmap, np.int32), 0.0, _dev([0.5], np.float32), row, tok, q)
        torch.cuda.synchronize()
        want = min(pos, (pos + 7777) % n_map)
        assert (int(row.item()), int(tok.item()), float(q.item())) == (want, 3 * want, 1.0)


def _run_verify(q4, target, drafts, vmap, rows, u, T, V):
    torch = _torch()
    n = len(rows)
    inv = OS.inverse_map(vmap, V)
    out = torch.full((3 * n + 3,), -7, dtype=torch.int32, device="cuda")
    q4.q4_spec_verify(_dev(target, np.float32), V, _dev(drafts, np.float32) if n else None, len(vmap),
                      _dev(vmap, np.int32), _dev(inv, np.int32), _dev(rows, np.int32) if n else None, n, T,
                      _dev(u, np.float32), out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _check_verify(target, drafts, vmap, rows, u, T, out):
    """Per position: the keep decision (exact unless within KEEP_TOL of the
    boundary) and the draw (a valid draw, exact away from boundaries); then
    the assembled output from the per-position results."""
    n, V = len(rows), target.shape[1]
    t64 = target.astype(np.float64)
    keep = out[n + 2: 2 * n + 2]
    draw = out[2 * n + 2: 3 * n + 3]
    exact, n_exact, n_checks = True, 0, 0
    for j in range(n):
        d = int(vmap[rows[j]])
        p = OS.dist(t64[j], T)
        q = np.zeros(V)
        q[vmap] = OS.dist(drafts[j].astype(np.float64), T)
        uq, pd = float(np.float32(u[j])) * q[d], p[d]
        want = uq < pd
        n_checks += 1
        if abs(uq - pd) > KEEP_TOL * max(uq, pd):
            assert bool(keep[j]) == want, f"position {j}: keep {keep[j]} vs oracle {want} (u q = {uq}, p = {pd})"
            n_exact += 1
        else:
            exact = False
        if keep[j]:
            assert draw[j] == -1
        else:
            r = np.maximum(p - q, 0.0)
            if r.sum() > 0:
                e = _check_draw(r, float(np.float32(u[n + j])), int(draw[j]), f"correction {j}",
                                tol=1e-5 + CDF_TOL * r.sum())
            else:
                e = _check_draw(p, float(np.float32(u[n + j])), int(draw[j]), f"correction {j}")
            exact &= e
            n_exact += e
            n_checks += 1
    e = _check_draw(OS.dist(t64[n], T), float(np.float32(u[2 * n])), int(draw[n]), "bonus")
    exact &= e
    n_exact += e
    n_checks += 1
    a = 0
    while a < n and keep[a]:
        a += 1
    assert out[0] == a
    assert list(out[1: a + 1]) == [int(vmap[r]) for r in rows[:a]]
    assert out[a + 1] == draw[a] and all(out[a + 2: n + 2] == -1)
    if exact:  # no boundary case anywhere: the whole step equals the oracle's
        a_ref, toks = OS.verify(t64, drafts, vmap, rows, np.float32(u).astype(np.float64), T)
        assert a_ref == a and toks == list(out[1: a + 2])
    return n_exact, n_checks


@pytest.mark.gpu
@pytest.mark.parametrize("T", [1.0, 1.7])
def test_verify_parity_full_vocabulary(cuda_device, T):
    """V = 248,320, a synthetic map of 65,536 tokens, three drafts whose
    logits follow the target's with noise (so p/q spans both sides of 1)."""
    import bit_weight_gemv_q4_b200 as q4

    rng = np.random.default_rng(int(T * 10))
    V, n_map, n = 248320, 65536, 3
    vmap = _synthetic_map(rng, V, n_map)
    n_exact = n_checks = 0
    for trial in range(12):
        target = rng.normal(0, 3.0, (n + 1, V)).astype(np.float32)
        target[:, vmap] += 2.0  # the mapped tokens carry most of the mass
        drafts = (target[:n][:, vmap] + rng.normal(0, 0.7, (n, n_map))).astype(np.float32)
        rows = np.array([OS.draft(drafts[j].astype(np.float64), vmap, T, rng.random())[1] for j in range(n)],
                        dtype=np.int32)
        u = rng.random(2 * n + 1).astype(np.float32)
        out = _run_verify(q4, target, drafts, vmap, rows, u, T, V)
        e, c = _check_verify(target, drafts, vmap, rows, u, T, out)
        n_exact, n_checks = n_exact + e, n_checks + c
        out2 = _run_verify(q4, target, drafts, vmap, rows, u, T, V)
        assert np.array_equal(out, out2)  # bitwise reproducible
    assert n_exact >= 0.6 * n_checks


@pytest.mark.gpu
@pytest.mark.parametrize("V,n_map,n", [(100, 10, 1), (1000, 1000, 3), (5000, 64, 15), (70, 3, 0), (1, 1, 2)])
def test_verify_small_and_edge_shapes(cuda_device, V, n_map, n):
    """Vocabularies smaller than a cluster's warps (empty slices), the
    identity map, the most drafts, no draft (a plain draw), one token."""
    import bit_weight_gemv_q4_b200 as q4

    rng = np.random.default_rng(V + n)
    vmap = _synthetic_map(rng, V, n_map)
    for trial in range(6):
        target = rng.normal(0, 1.5, (n + 1, V)).astype(np.float32)
        drafts = (target[:n][:, vmap] + rng.normal(0, 0.5, (n, n_map))).astype(np.float32)
        rows = np.array([OS.draft(drafts[j].astype(np.float64), vmap, 1.0, rng.random())[1] for j in range(n)],
                        dtype=np.int32)
        u = rng.random(2 * n + 1).astype(np.float32)
        out = _run_verify(q4, target, drafts, vmap, rows, u, 1.0, V)
        _check_verify(target, drafts, vmap, rows, u, 1.0, out)


@pytest.mark.gpu
def test_verify_greedy_exact(cuda_device):
    import bit_weight_gemv_q4_b200 as q4

    rng = np.random.default_rng(17)
    V, n_map, n = 248320, 65536, 3
    vmap = _synthetic_map(rng, V, n_map)
    for trial in range(8):
        target = rng.normal(0, 1, (n + 1, V)).astype(np.float32)
        rows = rng.integers(0, n_map, n).astype(np.int32)
        for j in range(n):
            if rng.random() < 0.7:  # this draft is the target's maximum (with a tie after it)
                target[j, vmap[rows[j]]] = 9.0
                target[j, V - 1 - j] = 9.0 if vmap[rows[j]] < V - 1 - j else 0.0
        drafts = rng.normal(0, 1, (n, n_map)).astype(np.float32)
        out = _run_verify(q4, target, drafts, vmap, rows, np.zeros(2 * n + 1, np.float32), 0.0, V)
        a, toks = OS.verify(target.astype(np.float64), drafts, vmap, rows, np.zeros(2 * n + 1), 0.0)
        assert out[0] == a and list(out[1: a + 2]) == toks


@pytest.mark.gpu
def test_verify_keeps_every_draft_of_an_exact_draft_head(cuda_device):
    import bit_weight_gemv_q4_b200 as q4

    rng = np.random.default_rng(23)
    V, n = 4096, 3
    vmap = np.arange(V, dtype=np.int32)
    target = rng.normal(0, 2, (n + 1, V)).astype(np.float32)
    for trial in range(6):
        rows = np.array([OS.draft(target[j].astype(np.float64), vmap, 1.0, rng.random())[1] for j in range(n)],
                        dtype=np.int32)
        u = (rng.random(2 * n + 1) * 0.99).astype(np.float32)
        out = _run_verify(q4, target, target[:n], vmap, rows, u, 1.0, V)
        assert out[0] == n and list(out[1: n + 1]) == list(rows)
        _check_draw(OS.dist(target[n].astype(np.float64), 1.0), float(u[2 * n]), int(out[n + 1]), "bonus")


@pytest.mark.gpu
def test_masked_tokens_are_never_emitted(cuda_device):
    import bit_weight_gemv_q4_b200 as q4

    rng = np.random.default_rng(29)
    V, n_map, n = 20000, 2000, 2
    vmap = _synthetic_map(rng, V, n_map)
    for trial in range(10):
        target = rng.normal(0, 1, (n + 1, V)).astype(np.float32)
        mask = rng.random(V) < 0.5
        target[:, mask] = -np.inf
        drafts = rng.normal(0, 1, (n, n_map)).astype(np.float32)
        rows = rng.integers(0, n_map, n).astype(np.int32)
        u = rng.random(2 * n + 1).astype(np.float32)
        out = _run_verify(q4, target, drafts, vmap, rows, u, 1.0, V)
        a = out[0]
        for t in out[1: a + 2]:
            assert not mask[t]
        _check_verify(target, drafts, vmap, rows, u, 1.0, out)


@pytest.mark.gpu
def test_mapped_draft_head_by_row_gather(cuda_device):
    """The vocabulary-mapped draft head: gather the mapped rows of the q8
    head's canonical codes and scales on the device, pack them, and its
    product equals the oracle's product of those rows."""
    import bit_weight_gemv_q4_b200 as q4
    import gpu_helpers as H
    from bit_weight_gemv_q4_b200 import synth

    torch = _torch()
    N, K, n_map = 6000, 1024, 1000
    rng = np.random.default_rng(31)
    vmap = _synthetic_map(rng, N, n_map)
    qh, sh = synth.tensor(8, 2, 77, N, K)
    rows_bad = np.concatenate([vmap, [-1, N]]).astype(np.int32)  # two rows out of range: zero rows
    qd, sd = _dev(qh.view(np.uint8), np.uint8), _dev(sh.view(np.uint16).view(np.int16), np.int16)
    gq = torch.empty((n_map + 2) * K, dtype=torch.uint8, device="cuda")
    gs = torch.empty((n_map + 2) * (K // 32), dtype=torch.int16, device="cuda")
    rd = _dev(rows_bad, np.int32)
    q4.q4_gather_rows_device(qd, K, N, rd, n_map + 2, gq)
    q4.q4_gather_rows_device(sd, 2 * (K // 32), N, rd, n_map + 2, gs)
    torch.cuda.synchronize()
    gqn = gq.cpu().numpy().reshape(n_map + 2, K)
    gsn = gs.cpu().numpy().view(np.uint16).reshape(n_map + 2, K // 32)
    assert np.array_equal(gqn[:n_map], qh.view(np.uint8)[vmap]) and np.array_equal(gsn[:n_map], sh[vmap])
    assert not gqn[n_map:].any() and not gsn[n_map:].any()
    packed = torch.empty(q4.q4_packed_bytes(8, n_map, K), dtype=torch.uint8, device="cuda")
    q4.q4_pack_weights_device(8, gq[: n_map * K], gs[: n_map * (K // 32)], n_map, K, packed)
    x = synth.activations(2, synth.act_stream(5), 1, K)
    y, ok = H.run_gemv(8, packed, n_map, K, H.to_device_x(x), 1)
    assert ok
    H.assert_parity(y, qh[vmap], sh[vmap], x, 8)


@pytest.mark.gpu
def test_speculative_step_end_to_end(cuda_device):
    """The whole step on the device (the mapped draft head gathered from the
    q8 output head, three drafts, the 257-product stream at M = 4, the keep /
    reject step): the draws checked against the oracle on the device's own
    logits.  The synthetic head's logits spread over ~+-300, so T = 60 keeps
    the distributions wide."""
    from bit_weight_gemv_q4_b200 import workloads

    torch = _torch()
    sp = workloads.DeviceSpec(seed=0, temperature=60.0)
    try:
        sp.run()
        sp.check()
        torch.cuda.synchronize()
        n, n_map, V = sp.n, sp.n_map, sp.V
        z = sp.z.cpu().numpy().reshape(n, n_map)
        rows = sp.rows.cpu().numpy()
        u = sp.u_host
        for j in range(n):
            _check_draw(OS.dist(z[j].astype(np.float64), sp.T), float(u[j]), int(rows[j]), f"draft {j}")
        assert np.array_equal(sp.tokens.cpu().numpy(), sp.vmap_host[rows])
        target = sp.target_logits.cpu().numpy().reshape(n + 1, V)
        out = sp.out.cpu().numpy()
        _check_verify(target, z, sp.vmap_host, rows, u[n:], sp.T, out)
        # the mapped head's outputs: row r is the output head's row at token vmap[r]
        from bit_weight_gemv_q4_b200 import synth
        import gpu_helpers as H

        rs = np.random.default_rng(1).integers(0, n_map, 6)
        for r in rs:
            qh, sh = synth.tensor(8, 0, 1023, V, sp.K, row0=int(sp.vmap_host[r]), nrows=1)
            x = sp.x_draft[0].cpu().numpy().view(np.uint16).reshape(1, sp.K)
            H.assert_parity(z[0:1, r:r + 1], qh, sh, x, 8)
    finally:
        sp.close()
        torch.cuda.empty_cache()


# ---------------------------------------------------------------- C-ABI argument checks (CPU)
def test_argument_errors_are_reported_before_any_device_work():
    """Invalid arguments are refused by the C ABI itself (no device call):
    draft count, temperature, sizes, null and misaligned pointers."""
    import ctypes

    import bit_weight_gemv_q4_b200 as q4

    L = q4.lib()
    buf = ctypes.create_string_buffer(64)
    p = ctypes.addressof(buf)
    p16 = (p + 15) // 16 * 16
    rc = L.q4_spec_verify(p16, 100, p16, 10, p16, p16, p16, 16, 1.0, p16, p16, None)
    assert rc == q4.Q4_ERR_INVALID_ARG and "n_draft" in q4.q4_last_error()
    rc = L.q4_spec_verify(p16, 100, p16, 10, p16, p16, p16, 3, -1.0, p16, p16, None)
    assert rc == q4.Q4_ERR_INVALID_ARG and "temperature" in q4.q4_last_error()
    rc = L.q4_spec_verify(p16, 100, p16, 10, p16, p16, p16, 3, float("nan"), p16, p16, None)
    assert rc == q4.Q4_ERR_INVALID_ARG
    rc = L.q4_spec_verify(p16, 0, p16, 10, p16, p16, p16, 3, 1.0, p16, p16, None)
    assert rc == q4.Q4_ERR_SHAPE
    rc = L.q4_spec_verify(p16, 100, p16, 200, p16, p16, p16, 3, 1.0, p16, p16, None)  # n_map > V
    assert rc == q4.Q4_ERR_SHAPE
    rc = L.q4_spec_verify(p16, 100, None, 10, p16, p16, p16, 3, 1.0, p16, p16, None)
    assert rc == q4.Q4_ERR_INVALID_ARG and "null" in q4.q4_last_error()
    rc = L.q4_spec_verify(p16 + 2, 100, p16, 10, p16, p16, p16, 3, 1.0, p16, p16, None)
    assert rc == q4.Q4_ERR_ALIGN
    rc = L.q4_spec_draft(p16, 0, p16, 1.0, p16, p16, p16, p16, None)
    assert rc == q4.Q4_ERR_SHAPE
    rc = L.q4_spec_draft(p16, 10, p16, float("inf"), p16, p16, p16, p16, None)
    assert rc == q4.Q4_ERR_INVALID_ARG
    rc = L.q4_gather_rows_device(p16, -1, 10, p16, 5, p16, None)
    assert rc == q4.Q4_ERR_SHAPE
    assert L.q4_gather_rows_device(p16, 16, 10, p16, 0, p16, None) == q4.Q4_OK  # nothing to copy
    rc = L.q4_gather_rows_device(p16, 16, 10, p16 + 1, 5, p16, None)
    assert rc == q4.Q4_ERR_ALIGN
