"""Pins of the CPU oracle against facts that do not come from the oracle itself.

* tangent-plane properties of log-sum-exp (exact at the reference, global
  lower bound by convexity, slope = gradient by finite differences), checked
  against scipy's logsumexp;
* closed forms (one key per chunk; zero reference; identical keys);
* the parent rule against planes computed directly from raw keys;
* append in any block size against a build from scratch;
* top-p against brute-force enumeration of every subset;
* routing and token set against the explainer figure of the page
  "Zyphra AI Introduces Zyphra Hierarchical Attention (ZHA)";
* attention against torch's scaled_dot_product_attention (fp64, CPU), and
  p = 1 routing against dense attention.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

HERE = os.path.dirname(os.path.abspath(__file__))


def rng(seed):
    return np.random.default_rng(seed)


def lse(q, K, s):
    return logsumexp(s * (K @ q))


def plane(q, mu, b, s):
    return s * float(q @ mu) + b


# ----------------------------------------------------------------- planes


@pytest.mark.parametrize("c,d", [(4, 64), (16, 128), (256, 128), (3, 8)])
def test_plane_exact_at_own_reference(orc, c, d):
    g = rng(c * 1000 + d)
    K = g.normal(size=(c, d)) + g.normal(scale=math.sqrt(0.5), size=d)
    refs = g.normal(size=(16, d)) * (3.0 / math.sqrt(d))
    s = 1.0 / math.sqrt(d)
    mu, b = orc.direct_planes(K, 0, c, refs, s)
    for r in range(16):
        assert plane(refs[r], mu[r], b[r], s) == pytest.approx(lse(refs[r], K, s), rel=1e-12, abs=1e-12)


@pytest.mark.parametrize("c", [4, 64])
def test_plane_lower_bound(orc, c):
    d = 32
    g = rng(7 + c)
    K = g.normal(size=(c, d))
    refs = g.normal(size=(8, d))
    s = 1.0 / math.sqrt(d)
    mu, b = orc.direct_planes(K, 0, c, refs, s)
    Q = g.normal(size=(2000, d)) * g.uniform(0.1, 4.0, size=(2000, 1))
    F = logsumexp(s * (Q @ K.T), axis=1)
    for r in range(8):
        est = s * (Q @ mu[r]) + b[r]
        assert np.all(est <= F + 1e-12)
    # and the estimate (max over planes) too, with equality at each reference
    for r in range(8):
        E = orc.estimate(refs[r], mu, b, s)
        assert E == pytest.approx(lse(refs[r], K, s), rel=1e-12)


def test_plane_slope_is_gradient(orc):
    d, c = 16, 8
    g = rng(11)
    K = g.normal(size=(c, d))
    r = g.normal(size=d)
    s = 0.37
    mu, b = orc.direct_planes(K, 0, c, r[None, :], s)
    h = 1e-5
    grad = np.array([(lse(r + h * e, K, s) - lse(r - h * e, K, s)) / (2 * h) for e in np.eye(d)])
    assert np.allclose(s * mu[0], grad, rtol=1e-7, atol=1e-8)


def test_closed_form_single_key_chunks_are_exact(orc):
    d = 24
    g = rng(3)
    K = g.normal(size=(1, d))
    refs = g.normal(size=(4, d))
    s = 1.0 / math.sqrt(d)
    mu, b = orc.direct_planes(K, 0, 1, refs, s)
    for q in g.normal(size=(50, d)):
        for r in range(4):
            assert plane(q, mu[r], b[r], s) == pytest.approx(s * float(q @ K[0]), abs=1e-12)


def test_closed_form_zero_reference(orc):
    d, c = 16, 12
    g = rng(4)
    K = g.normal(size=(c, d))
    mu, b = orc.direct_planes(K, 0, c, np.zeros((1, d)), 0.25)
    assert np.allclose(mu[0], K.mean(axis=0), atol=1e-14)
    assert b[0] == pytest.approx(math.log(c), abs=1e-14)


def test_closed_form_identical_keys(orc):
    d, c = 16, 8
    g = rng(5)
    k = g.normal(size=d)
    K = np.tile(k, (c, 1))
    refs = g.normal(size=(3, d))
    s = 0.25
    mu, b = orc.direct_planes(K, 0, c, refs, s)
    for q in g.normal(size=(20, d)):
        for r in range(3):
            assert plane(q, mu[r], b[r], s) == pytest.approx(s * float(q @ k) + math.log(c), abs=1e-12)


# ------------------------------------------------------------------ tree


def _keys(seed, N, d, c):
    g = rng(seed)
    off = g.normal(scale=math.sqrt(0.5), size=((N + c - 1) // c, d))
    return g.normal(size=(N, d)) + np.repeat(off, c, axis=0)[:N]


@pytest.mark.parametrize("N,c,L", [(4096, 4, 3), (1000, 4, 4), (777, 8, 3), (4096 + 3, 16, 2), (300, 256, 1)])
def test_parent_rule_equals_direct_planes(orc, N, c, L):
    """Every node, partial rightmost ones included, equals R1 over its raw keys."""
    d, R = 16, 5
    K = _keys(N, N, d, c)
    refs = rng(N + 1).normal(size=(R, d)) * 0.7
    s = 1.0 / math.sqrt(d)
    t = orc.build_tree(K, refs, N, c, L, s)
    n1 = N // c
    for level in range(1, L + 1):
        span = c ** level
        for n in range(t.n(level)):
            t0, t1 = n * span, min((n + 1) * span, n1 * c)
            mu, b = orc.direct_planes(K, t0, t1, refs, s)
            assert np.allclose(t.mu[level - 1][n], mu, rtol=1e-10, atol=1e-10), (level, n)
            assert np.allclose(t.b[level - 1][n], b, rtol=1e-10, atol=1e-10), (level, n)


def test_parent_rule_wrong_variant_would_fail(orc):
    """The same check rejects a parent that treats its children as plain keys,
    or weights them by their plane offsets (biases) instead of their log-masses."""
    d, R, c = 8, 3, 4
    K = _keys(9, 64, d, c)
    refs = rng(10).normal(size=(R, d))
    s = 0.3
    t = orc.build_tree(K, refs, 64, c, 2, s)
    mu_direct, b_direct = orc.direct_planes(K, 0, 16, refs, s)
    # a parent built from children as plain keys (no log-weights) differs
    mu_plain, b_plain = orc.direct_planes(t.mu[0][0:4, 0], 0, 4, refs[:1], s)
    assert not np.isclose(b_plain[0], b_direct[0], rtol=1e-6)
    # ... and so does one that weights them by their biases
    mu_b, b_b, _ = orc.parent_planes(t.mu[0][0:4], t.b[0][0:4], refs, s)
    assert not np.allclose(b_b, b_direct, rtol=1e-6)
    mu_f, b_f, _ = orc.parent_planes(t.mu[0][0:4], t.F[0][0:4], refs, s)
    assert np.allclose(mu_f, mu_direct, rtol=1e-10, atol=1e-10) and np.allclose(b_f, b_direct, rtol=1e-10)
    assert np.isclose(t.b[1][0, 0], b_direct[0], rtol=1e-10)


@pytest.mark.parametrize("N,c,L", [(4096, 4, 3), (777, 8, 3), (300, 256, 1)])
def test_node_logmass_is_exact_log_sum_exp(orc, N, c, L):
    """Each node's kept log-mass F_r is log sum e^{s r.k} over its raw keys
    (scipy), and equals its plane's value at its own reference."""
    from scipy.special import logsumexp
    d, R = 16, 3
    K = _keys(N + 5, N, d, c)
    refs = rng(N + 6).normal(size=(R, d)) * 0.7
    s = 1.0 / math.sqrt(d)
    t = orc.build_tree(K, refs, N, c, L, s)
    n1 = N // c
    for level in range(1, L + 1):
        span = c ** level
        for n in range(0, t.n(level), max(1, t.n(level) // 7)):
            t0, t1 = n * span, min((n + 1) * span, n1 * c)
            for r in range(R):
                exact = logsumexp(s * K[t0:t1] @ refs[r])
                assert abs(t.F[level - 1][n, r] - exact) <= 1e-11 * max(1.0, abs(exact))
                own = s * refs[r] @ t.mu[level - 1][n, r] + t.b[level - 1][n, r]
                assert abs(own - exact) <= 1e-11 * max(1.0, abs(exact))


@pytest.mark.parametrize("block", [1, 3, 4, 37, 4096])
def test_append_equals_build(orc, block):
    N, d, c, L, R = 2000, 8, 4, 4, 3
    K = _keys(21, N, d, c)
    refs = rng(22).normal(size=(R, d))
    s = 0.35
    full = orc.build_tree(K, refs, N, c, L, s)
    inc = orc.new_tree(N, c, L, R, d, s)
    n = 0
    while n < N:
        n = min(n + block, N)
        orc.tree_update(inc, K, refs, n)
    for level in range(L):
        k = full.n(level + 1)
        assert np.array_equal(full.mu[level][:k], inc.mu[level][:k])
        assert np.array_equal(full.b[level][:k], inc.b[level][:k])


def test_storage_rounding_matches_torch_bf16(orc):
    g = rng(31)
    x = g.normal(size=2000).astype(np.float32) * 10.0 ** g.integers(-6, 6, size=2000)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    mine = np.array([orc.round_storage(float(v), "bf16") for v in x])
    assert np.array_equal(mine, ref)
    assert orc.round_storage(1.0 + 2 ** -30, "f32") == 1.0


def test_bf16_storage_tree_builds_from_rounded_children(orc):
    N, d, c, L = 256, 16, 4, 3
    K = _keys(41, N, d, c)
    refs = rng(42).normal(size=(4, d))
    s = 0.25
    t = orc.build_tree(K, refs, N, c, L, s, storage="bf16")
    for level in range(L):
        m = t.mu[level][: t.n(level + 1)]
        assert np.array_equal(torch.from_numpy(m).to(torch.bfloat16).double().numpy(), m)
    ref = orc.build_tree(K, refs, N, c, L, s)
    assert np.allclose(t.mu[2][0], ref.mu[2][0], rtol=2e-2, atol=2e-2)


# ----------------------------------------------------------------- top-p


def brute_force_topp(E, p):
    """Smallest-cardinality subset with mass >= p*Z; among those the heaviest;
    among equally heavy ones the lexicographically smallest index tuple."""
    n = len(E)
    m = max(E)
    w = [math.exp(e - m) for e in E]
    Z = sum(w)
    if p >= 1.0:
        return set(range(n))
    for k in range(1, n + 1):
        best = None
        for sub in itertools.combinations(range(n), k):
            mass = sum(w[i] for i in sub)
            if mass < p * Z:
                continue
            key = (-mass, sub)
            if best is None or key < best:
                best = key
        if best is not None:
            return set(best[1])
    return set(range(n))


@pytest.mark.parametrize("seed", range(40))
def test_topp_matches_brute_force(orc, seed):
    g = rng(100 + seed)
    n = int(g.integers(1, 13))
    E = g.normal(scale=g.uniform(0.1, 3.0), size=n)
    if seed % 4 == 0 and n > 2:         # exact ties, broken by lower index
        E[g.integers(0, n)] = E[0]
        E[n - 1] = E[0]
    for p in (0.1, 0.5, 0.9, 0.95, 0.999999, 1.0):
        kept, _ = orc.topp_select(E, p)
        want = brute_force_topp(list(E), p)
        # with exact ties several heaviest subsets exist only if masses tie; the
        # brute force breaks them by index exactly like (score desc, index asc)
        assert set(np.nonzero(kept)[0]) == want, (E, p)


def test_topp_special_cases(orc):
    E = np.array([0.0, 10.0, 0.5, -3.0])
    kept, _ = orc.topp_select(E, 0.95)
    assert list(np.nonzero(kept)[0]) == [1]
    kept, _ = orc.topp_select(E, 1.0)
    assert kept.all()
    # p >= 1 keeps candidates whose mass underflows
    kept, _ = orc.topp_select(np.array([0.0, -2000.0]), 1.0)
    assert kept.all()
    kept, cum = orc.topp_select(np.array([1.0, 1.0, 1.0, 1.0]), 0.5)
    assert list(np.nonzero(kept)[0]) == [0, 1]
    assert np.allclose(cum, [0, 0.25, 0.5, 0.75])


# --------------------------------------------------------------- routing


def test_route_matches_explainer_figure(orc):
    fig = json.load(open(os.path.join(HERE, "golden", "explainer_figure_route.json")))
    c, L = fig["chunk"], fig["levels"]
    d, R = 8, 2
    N = fig["nodes_per_level"]["1"] * c
    t = orc.new_tree(N, c, L, R, d, 1.0)
    t.N = N
    kept = {int(k): v for k, v in fig["kept"].items()}
    for level in range(1, L + 1):
        assert t.n(level) == fig["nodes_per_level"][str(level)]
        t.mu[level - 1][:] = 0.0
        t.b[level - 1][:] = 0.0
        t.b[level - 1][kept[level], :] = 12.0     # the figure's kept nodes dominate
    q = np.zeros((1, d))
    r = orc.route(t, q, 0.95)
    for level in range(1, L + 1):
        assert list(np.nonzero(r.kept[level - 1][0])[0]) == kept[level]
    # candidates at each level are exactly the children of the kept parents
    for level in range(1, L):
        want = sorted(j for n in kept[level + 1] for j in range(n * c, n * c + c))
        assert list(np.nonzero(r.cand[level - 1][0])[0]) == want
    tm = orc.token_set(N, c, r.kept[0][0])
    want = {0} | {j * c + i for j in kept[1] for i in range(c)} | set(range(N - c, N))
    assert set(np.nonzero(tm)[0]) == want


def test_token_set_sink_and_current_chunk(orc):
    c = 4
    for N in (1, 2, 3, 4, 5, 8, 9, 100, 103):
        n1 = N // c
        none = np.zeros(n1, dtype=bool)
        tm = orc.token_set(N, c, none)
        cur = ((N - 1) // c) * c
        assert set(np.nonzero(tm)[0]) == {0} | set(range(cur, N))
        tt = orc.token_set(N, c, none, tail_only=True)
        assert set(np.nonzero(tt)[0]) == {0} | set(range((N // c) * c, N))


def _group(seed, N, d, c, L, R, G):
    K = _keys(seed, N, d, c)
    g = rng(seed + 1)
    V = g.normal(size=(N, d))
    refs = g.normal(size=(R, d)) / math.sqrt(d)
    q = g.normal(size=(G, d))
    return K, V, refs, q


def test_p1_routes_everything_and_equals_dense(orc):
    N, d, c, L, R, G = 1001, 16, 4, 3, 4, 3
    K, V, refs, q = _group(50, N, d, c, L, R, G)
    t = orc.build_tree(K, refs, N, c, L)
    out, r, masks = orc.decode_group(t, q, K, V, 1.0)
    for level in range(L):
        assert r.kept[level].all() and r.cand[level].all()
    assert masks.all()
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(K)[None, None].expand(1, G, N, d),
        torch.from_numpy(V)[None, None].expand(1, G, N, d), scale=t.s)[0, :, 0]
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_attend_matches_sdpa_with_mask(orc):
    N, d = 333, 32
    g = rng(61)
    q, K, V = g.normal(size=d), g.normal(size=(N, d)), g.normal(size=(N, d))
    tm = g.uniform(size=N) < 0.3
    tm[0] = True
    s = 0.2
    out = orc.attend(q, K, V, N, s, tm)
    bias = torch.full((N,), -math.inf, dtype=torch.float64)
    bias[torch.from_numpy(tm)] = 0.0
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None], torch.from_numpy(K)[None, None],
        torch.from_numpy(V)[None, None], attn_mask=bias[None, None, None], scale=s)
    assert np.allclose(out, ref.flatten().numpy(), rtol=1e-12, atol=1e-12)
    # closed forms: one token -> its value; identical keys -> mean of values
    assert np.allclose(orc.attend(q, K, V, 1, s), V[0])
    Kc = np.tile(K[5], (N, 1))
    assert np.allclose(orc.attend(q, Kc, V, N, s), V.mean(axis=0))


def test_route_invariants_random(orc):
    N, d, c, L, R, G = 4096, 16, 4, 3, 8, 4
    K, V, refs, q = _group(70, N, d, c, L, R, G)
    t = orc.build_tree(K, refs, N, c, L)
    for p in (0.5, 0.9, 0.95):
        out, r, masks = orc.decode_group(t, q, K, V, p)
        for h in range(G):
            assert masks[h, 0] and masks[h, N - c:].all()
            for level in range(L, 0, -1):
                cand = r.cand[level - 1][h]
                kept = r.kept[level - 1][h]
                assert not np.any(kept & ~cand)
                E = r.score[level - 1][h][cand]
                k2, _ = orc.topp_select(E, p)
                assert np.array_equal(k2, kept[cand])
                if level > 1:
                    kids = np.zeros_like(r.cand[level - 2][h])
                    for n in np.nonzero(kept)[0]:
                        kids[n * c:min(n * c + c, kids.shape[0])] = True
                    assert np.array_equal(kids, r.cand[level - 2][h])
                # the kept mass reaches p of the candidates' mass
                w = np.exp(E - E.max())
                assert w[kept[cand]].sum() >= p * w.sum() * (1 - 1e-12)


# ------------------------------------------------------------------ per-level p


def _uniform_tree(orc, m, d, c, L, R, G, seed):
    """Identical keys everywhere and N = m * c^L: every node of a level has the
    same planes, so all candidates of a level tie and top-p keeps the first
    ceil(p * count) of them in index order."""
    N = m * c ** L
    g = rng(seed)
    K = np.tile(g.normal(size=d), (N, 1))
    refs = g.normal(size=(R, d)) / math.sqrt(d)
    q = g.normal(size=(G, d))
    return orc.build_tree(K, refs, N, c, L), q


def _uniform_counts(m, c, p_levels):
    """Closed form of the kept count per level (level L first) on a uniform tree."""
    counts, n_cand = [], m
    for level in range(len(p_levels), 0, -1):
        k = math.ceil(p_levels[level - 1] * n_cand)
        counts.append((level, n_cand, k))
        n_cand = k * c
    return counts


def test_per_level_p_closed_form_on_uniform_tree(orc):
    """Distinct p per level: each level keeps exactly its own ceil(p_l * candidates)
    (which list entry serves which level is pinned by the distinct counts)."""
    m, d, c, L, R, G = 5, 16, 4, 3, 2, 2
    t, q = _uniform_tree(orc, m, d, c, L, R, G, 80)
    p_levels = [0.3, 0.55, 0.7]          # levels 1, 2, 3
    r = orc.route(t, q, p_levels)
    for h in range(G):
        for level, n_cand, k in _uniform_counts(m, c, p_levels):
            cand = np.nonzero(r.cand[level - 1][h])[0]
            kept = np.nonzero(r.kept[level - 1][h])[0]
            assert np.array_equal(cand, np.arange(n_cand)), (h, level)
            assert np.array_equal(kept, np.arange(k)), (h, level)
    # reversed list gives other counts: the pin separates the levels
    assert _uniform_counts(m, c, p_levels[::-1]) != _uniform_counts(m, c, p_levels)


@pytest.mark.parametrize("p", [0.6, 0.8, 0.95])
def test_depth_root_schedule_restores_coverage(orc, p):
    """On a tree with evenly spread mass the kept share of leaves is about p^L
    under one fixed p and about p under p^(1/L) per level (the depth caveat of
    the explainer, tab 5)."""
    m, d, c, L, R, G = 64, 8, 4, 3, 2, 1
    t, q = _uniform_tree(orc, m, d, c, L, R, G, 81)
    n1 = m * c ** (L - 1)
    sched = orc.depth_root_schedule(p, L)
    assert len(sched) == L and math.prod(sched) == pytest.approx(p, rel=1e-12)
    assert orc.depth_root_schedule(1.0, L) == [1.0] * L
    fixed = orc.route(t, q, p).kept[0][0].sum() / n1
    root = orc.route(t, q, sched).kept[0][0].sum() / n1
    assert fixed == pytest.approx(p ** L, abs=0.02)
    assert root == pytest.approx(p, abs=0.02)


# ------------------------------------------------------- low-precision summaries


def _e4m3_grid():
    """Every finite non-negative E4M3 value, from its bit fields (bias 7)."""
    vals = [m * 2.0 ** -9 for m in range(8)]                       # subnormals
    vals += [(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8) if not (e == 15 and m == 7)]
    return np.array(sorted(vals))


def test_e4m3_rounding_matches_torch_float8(orc):
    grid = _e4m3_grid()
    assert grid[-1] == 448.0 and grid[1] == 2.0 ** -9 and len(grid) == 127
    mids = (grid[:-1] + grid[1:]) / 2                              # exact ties
    g = rng(90)
    rnd = (g.uniform(-1, 1, size=20000) * 2.0 ** g.integers(-12, 9, size=20000)).astype(np.float32)
    rnd = rnd[np.abs(rnd) <= 448]
    x = np.concatenate([grid, -grid, mids, -mids, rnd.astype(np.float64)])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([orc.e4m3_round(v) for v in x])
    assert np.array_equal(mine, ref)
    # ties go to the even mantissa: the midpoint above 1 (= 1 + 1/16) rounds down to 1
    assert orc.e4m3_round(1.0 + 1 / 16) == 1.0 and orc.e4m3_round(1.0 + 3 / 16) == 1.25
    assert orc.e4m3_round(1000.0) == 448.0 and orc.e4m3_round(-1000.0) == -448.0


def test_mx_block_scale_closed_form(orc):
    g = rng(91)
    x = g.normal(size=(64, 128)) * 10.0 ** g.integers(-4, 4, size=(64, 1))
    x[3, 32:64] = 0.0                                             # an all-zero block
    v, e = orc.mx_round(x)
    blocks = x.reshape(64, 4, 32)
    amax = np.abs(blocks).max(axis=2)
    live = amax > 0
    scale = 2.0 ** e
    # the smallest power of two that brings the block's maximum within 448
    assert np.all(amax[live] <= 448 * scale[live]) and np.all(amax[live] > 224 * scale[live])
    assert np.all(v.reshape(64, 4, 32)[~live] == 0)
    # each element is the nearest E4M3 multiple of its block's scale
    vb, sb = v.reshape(64, 4, 32), scale[:, :, None]
    q = vb / sb
    grid = _e4m3_grid()
    assert np.all(np.isin(np.abs(q), grid))
    err = np.abs(vb - blocks)
    ulp = np.where(np.abs(blocks) / sb < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(blocks) / sb, 1e-300))) - 3))
    assert np.all(err <= 0.5 * ulp * sb * (1 + 1e-12))
    # power-of-two equivariance and idempotence
    v2, e2 = orc.mx_round(x * 8.0)
    assert np.array_equal(v2, v * 8.0) and np.array_equal(e2[live], e[live] + 3)
    v3, _ = orc.mx_round(v)
    assert np.array_equal(v3, v)


def test_mxfp8_storage_tree_builds_from_rounded_children(orc):
    N, d, c, L = 512, 64, 4, 3
    K = _keys(92, N, d, c)
    refs = rng(93).normal(size=(4, d)) / math.sqrt(d)
    s = 1 / math.sqrt(d)
    t = orc.build_tree(K, refs, N, c, L, s, storage="mxfp8")
    ref = orc.build_tree(K, refs, N, c, L, s)
    for level in range(L):
        m = t.mu[level][: t.n(level + 1)]
        again, _ = orc.mx_round(m)
        assert np.array_equal(again, m)                            # stored values are MX-FP8
        # rounding error, relative to the block's largest coordinate: half an E4M3
        # step (2^-4) per level, a parent inheriting its children's errors
        r = ref.mu[level][: t.n(level + 1)]
        bmax = np.abs(r).reshape(r.shape[:-1] + (d // 32, 32)).max(axis=-1, keepdims=True)
        err = np.abs(m - r).reshape(bmax.shape[:-1] + (32,)) / bmax
        assert err.max() <= (level + 1) * 2.0 ** -4
        b = t.b[level][: t.n(level + 1)]
        assert np.array_equal(b.astype(np.float32).astype(np.float64), b)   # bias kept in fp32
    # the parent rule on given children reproduces the tree's parents
    for level in range(1, L):
        for node in range(t.n(level + 1)):
            c0, c1 = node * c, min(node * c + c, t.n(level))
            pm, pb, pf = orc.parent_planes(t.mu[level - 1][c0:c1], t.F[level - 1][c0:c1], refs, s, "mxfp8")
            assert np.array_equal(pm, t.mu[level][node]) and np.array_equal(pb, t.b[level][node])
            assert np.array_equal(pf, t.F[level][node])
    # estimates stay close to the exact tree's (the router's purpose)
    q = rng(94).normal(size=d)
    for level in range(L):
        for n in range(t.n(level + 1)):
            e_mx = orc.estimate(q, t.mu[level][n], t.b[level][n], s)
            e_64 = orc.estimate(q, ref.mu[level][n], ref.b[level][n], s)
            # |max_r a_r - max_r b_r| <= max_r |a_r - b_r| (triangle inequality per plane)
            dmu = np.abs(t.mu[level][n] - ref.mu[level][n])
            bound = np.max(s * dmu @ np.abs(q) + np.abs(t.b[level][n] - ref.b[level][n]))
            assert abs(e_mx - e_64) <= bound + 1e-12
            assert abs(e_mx - e_64) < 0.1


# ------------------------------------------------------------ multi-query blocks


def test_block_p1_rows_equal_causal_dense(orc):
    """p = 1: every row of a block attends its whole causal prefix [0, N0 + t]."""
    N0, T, d, c, L, R, G = 517, 5, 16, 4, 3, 4, 2
    K, V, refs, _ = _group(100, N0 + T, d, c, L, R, G)
    q = rng(101).normal(size=(T, G, d))
    t = orc.build_tree(K, refs, N0, c, L)
    out, r, masks = orc.decode_block_group(t, q, K, V, 1.0)
    for tt in range(T):
        n = N0 + tt + 1
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[tt])[None, :, None, :], torch.from_numpy(K[:n])[None, None].expand(1, G, n, d),
            torch.from_numpy(V[:n])[None, None].expand(1, G, n, d), scale=t.s)[0, :, 0]
        assert np.allclose(out[tt], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_block_single_query_equals_decode_when_no_chunk_completes(orc):
    """T = 1 and N0 + 1 not a multiple of c: the tree before and after the token
    is the same, and the block's token rule is the decode rule."""
    d, c, L, R, G = 16, 4, 3, 4, 3
    for N0 in (401, 402, 1000, 4):
        K, V, refs, _ = _group(102 + N0, N0 + 1, d, c, L, R, G)
        q = rng(103).normal(size=(1, G, d))
        t = orc.build_tree(K, refs, N0, c, L)
        for p in (0.6, 0.95):
            ob, rb, mb = orc.decode_block_group(t, q, K, V, p)
            t1 = orc.build_tree(K, refs, N0 + 1, c, L)
            od, rd, md = orc.decode_group(t1, q[0], K, V, p)
            assert np.array_equal(np.stack(mb), md)
            assert np.allclose(ob[0], od, rtol=1e-12, atol=1e-12)


def test_block_rows_are_causal(orc):
    """A row's output does not depend on the block's later tokens; its token set
    is the sink, its kept leaves and [c*floor(N0/c), N0 + t]."""
    N0, T, d, c, L, R, G = 389, 6, 16, 8, 2, 4, 2
    K, V, refs, _ = _group(104, N0 + T, d, c, L, R, G)
    q = rng(105).normal(size=(T, G, d))
    t = orc.build_tree(K, refs, N0, c, L)
    out, r, masks = orc.decode_block_group(t, q, K, V, 0.8)
    K2, V2 = K.copy(), V.copy()
    K2[N0 + 2:] += 5.0
    V2[N0 + 2:] -= 3.0
    out2, _, _ = orc.decode_block_group(t, q, K2, V2, 0.8)
    assert np.array_equal(out[:2], out2[:2]) and not np.allclose(out[2:], out2[2:])
    for tt in range(T):
        for h in range(G):
            m = masks[tt * G + h]
            assert m.shape == (N0 + tt + 1,) and m[0] and m[c * (N0 // c):].all()
            kept = np.nonzero(r.kept[0][tt * G + h])[0]
            want = np.zeros_like(m)
            want[0] = True
            for j in kept:
                want[j * c:(j + 1) * c] = True
            want[c * (N0 // c):] = True
            assert np.array_equal(m, want)
