"""Parity of the MX-FP8 summary path (E4M3 blocks of 32 coordinates with a
power-of-two scale each) with the oracle's MX-FP8 storage, through the C ABI.

The GPU forms mu in fp32 and the oracle in fp64 before both round to E4M3, so
a coordinate lying within the fp32 error of a rounding boundary may land one
E4M3 step apart; such flips must be rare and at most one step."""
import numpy as np
import pytest
import torch

import zha_oracle as orc
import zha_testlib as T
from tree_indexed_sparse_02_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

CASES = T.mx_workloads()
IDS = [w.name for w in CASES]


@pytest.fixture(scope="module")
def zha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_indexed_sparse_02_b200 import zha as z
    return z


def _lens_for(w):
    if w.batch == 1:
        return None
    return [w.context] + [w.context - 3 * b - 1 for b in range(1, w.batch)]


def _flips_within_one_step(got, ref, X):
    """Coordinates where the two sides rounded to neighbouring E4M3 values:
    rare, and one step apart: 2^-3 of the magnitude in the normal range, 2^-9
    of the block scale X in the subnormal range (twice that if the two sides
    chose block exponents one apart)."""
    diff = got != ref
    assert diff.mean() <= 1e-3, diff.mean()
    if diff.any():
        step = np.maximum(np.maximum(np.abs(got), np.abs(ref)) * 2.0 ** -3, X * 2.0 ** -8)
        assert np.all(np.abs(got - ref)[diff] <= step[diff] * (1 + 1e-9)), np.abs(got - ref)[diff]


def _check_mx_level(buf, level, b, kvh, n, t, w, inp, s):
    """Level 1 against the oracle's leaves (same raw keys); a level above
    against the oracle's parent rule applied to the GPU's own stored children
    (summary keys and log-masses), so that each level is checked on its own
    inputs."""
    mu8, b_g = buf.tree_level(level)
    sc = buf.tree_level_scales(level)[b, kvh, :n]
    got = T.mx_decode(mu8[b, kvh, :n], sc)
    X = np.exp2(sc.cpu().numpy().astype(np.float64) - 127.0).repeat(32, axis=-1)
    # every stored value is on its block's E4M3 grid: decoding then re-rounding is the identity
    again, _ = orc.mx_round(got)
    assert np.array_equal(again, got)
    bg = T.np64(b_g[b, kvh, :n])
    if level == 1:
        ref, bref = t.mu[0][:n], t.b[0][:n]
    else:
        n_below = orc.level_nodes(int(inp.lens[b]), w.chunk, level - 1)
        cmu8, _ = buf.tree_level(level - 1)
        kids = T.mx_decode(cmu8[b, kvh, :n_below], buf.tree_level_scales(level - 1)[b, kvh, :n_below])
        kF = T.np64(buf.tree_level_logmass(level - 1)[b, kvh, :n_below])
        refs = T.np64(inp.refs[kvh])
        ref = np.zeros_like(got)
        bref = np.zeros_like(bg)
        Fref = np.zeros_like(bg)
        for node in range(n):
            c0, c1 = node * w.chunk, min(node * w.chunk + w.chunk, n_below)
            ref[node], bref[node], Fref[node] = orc.parent_planes(kids[c0:c1], kF[c0:c1], refs, s, "mxfp8")
        assert T.rel_err(T.np64(buf.tree_level_logmass(level)[b, kvh, :n]), Fref) <= 1e-5
    _flips_within_one_step(got, ref, X)
    eb = T.rel_err(bg, bref)
    assert eb <= 1e-4, eb
    # end to end against the oracle's own tree: flips may compound over levels, still rare
    assert (got != t.mu[level - 1][:n]).mean() <= 1e-3


@pytest.mark.parametrize("w", CASES, ids=IDS)
def test_mx_tree_build_matches_oracle(zha, w):
    cfg, inp, dev, buf = T.build_case(zha, w, lens=_lens_for(w))
    zha.tree_build(cfg, buf.tree, dev.K, dev.refs, dev.lens, buf.status)
    torch.cuda.synchronize()
    buf.check_status()
    s = T.scale_of(w)
    for b in range(w.batch):
        N = int(inp.lens[b])
        for kvh in range(w.n_kv_heads):
            t = T.oracle_tree(w, inp, b, kvh, N, s)
            for level in range(1, w.levels + 1):
                _check_mx_level(buf, level, b, kvh, orc.level_nodes(N, w.chunk, level), t, w, inp, s)


@pytest.mark.parametrize("w", CASES[:3], ids=IDS[:3])
@pytest.mark.parametrize("block", [1, 3, 1000])
def test_mx_append_equals_build_bitexact(zha, w, block):
    cfg, inp, dev, buf = T.build_case(zha, w)
    N = w.context
    ref = zha.Buffers(cfg)
    zha.tree_build(cfg, ref.tree, dev.K, dev.refs, dev.lens, ref.status)
    lens = torch.zeros_like(dev.lens)
    n = 0
    while n < N:
        step = min(block, N - n)
        n += step
        lens.fill_(n)
        zha.tree_append(cfg, buf.tree, dev.K, dev.refs, lens, step, buf.status)
    torch.cuda.synchronize()
    buf.check_status()
    for level in range(1, w.levels + 1):
        k = orc.level_nodes(N, w.chunk, level)
        assert torch.equal(buf.tree_level(level)[0][:, :, :k], ref.tree_level(level)[0][:, :, :k]), level
        assert torch.equal(buf.tree_level_scales(level)[:, :, :k], ref.tree_level_scales(level)[:, :, :k]), level
        assert torch.equal(buf.tree_level(level)[1][:, :, :k], ref.tree_level(level)[1][:, :, :k]), level


@pytest.mark.parametrize("w", CASES, ids=IDS)
def test_mx_route_matches_oracle(zha, w):
    cfg, inp, dev, buf = T.build_case(zha, w, lens=_lens_for(w))
    zha.tree_build(cfg, buf.tree, dev.K, dev.refs, dev.lens, buf.status)
    p_levels = [w.p] * w.levels
    zha.route(cfg, buf.tree, dev.q, dev.lens, p_levels, buf.sel, buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status()
    states = {l: buf.level_state(l) for l in range(1, w.levels + 1)}
    s = T.scale_of(w)
    G = w.group
    total_flipped = 0
    for b in range(w.batch):
        N = int(inp.lens[b])
        for kvh in range(w.n_kv_heads):
            t = T.oracle_tree(w, inp, b, kvh, N, s)
            q = T.np64(inp.q[b, kvh * G:(kvh + 1) * G])
            r = orc.route(t, q, w.p)
            flipped, worst = T.compare_routing(r, states, b, kvh, G, N, w, p_levels)
            assert worst <= T.TOL["bf16"], worst
            total_flipped += len(flipped)
            cnt = int(buf.sel["count"][b, kvh])
            idx = buf.sel["leaf_idx"][b, kvh, :cnt].cpu().numpy()
            hm = buf.sel["head_mask"][b, kvh, :cnt].cpu().numpy().astype(np.uint32)
            for h in range(G):
                if h in flipped:
                    continue
                got = idx[(hm >> np.uint32(h)) & 1 != 0]
                assert np.array_equal(np.sort(got), np.nonzero(r.kept[0][h])[0]), (b, kvh, h)
    assert total_flipped <= max(2, w.batch * w.n_q_heads // 8), total_flipped


@pytest.mark.parametrize("w", CASES[:3], ids=IDS[:3])
def test_mx_decode_steps_match_oracle(zha, w):
    """zha_decode with MX-FP8 summaries: each step's tree, routing and output
    match the oracle's; the appended tree equals a fresh build bit for bit."""
    steps = 9
    cap = w.context + steps + 8
    inp = make_inputs(w, capacity=cap)
    dev = T.to_device(inp)
    cfg = T.make_cfg(zha, w, cap)
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, dev.K, dev.refs, dev.lens, buf.status)
    G = w.group
    s = T.scale_of(w)
    g = torch.Generator().manual_seed(6)
    dt = w.torch_dtype()
    K_host, V_host = inp.K.clone(), inp.V.clone()
    trees = {(b, kvh): T.oracle_tree(w, inp, b, kvh, w.context, s, cap)
             for b in range(w.batch) for kvh in range(w.n_kv_heads)}
    flipped_total = 0
    for step in range(steps):
        k_new = torch.randn((w.batch, w.n_kv_heads, w.head_dim), generator=g).to(dt)
        v_new = torch.randn((w.batch, w.n_kv_heads, w.head_dim), generator=g).to(dt)
        q = torch.randn((w.batch, w.n_q_heads, w.head_dim), generator=g).to(dt)
        out = torch.zeros_like(dev.q)
        zha.decode(cfg, buf.tree, dev.K, dev.V, dev.refs, dev.lens, q.cuda(), k_new.cuda(), v_new.cuda(),
                   w.p, buf.sel, out, buf.workspace, buf.status)
        torch.cuda.synchronize()
        buf.check_status()
        states = {l: buf.level_state(l) for l in range(1, w.levels + 1)}
        for b in range(w.batch):
            N = w.context + step + 1
            K_host[b, :, N - 1] = k_new[b]
            V_host[b, :, N - 1] = v_new[b]
            for kvh in range(w.n_kv_heads):
                t = trees[(b, kvh)]
                orc.tree_update(t, T.np64(K_host[b, kvh, :N]), T.np64(inp.refs[kvh]), N)
                qg = T.np64(q[b, kvh * G:(kvh + 1) * G])
                o, r, masks = orc.decode_group(t, qg, T.np64(K_host[b, kvh, :N]), T.np64(V_host[b, kvh, :N]), w.p)
                flipped, worst = T.compare_routing(r, states, b, kvh, G, N, w, [w.p] * w.levels)
                flipped_total += len(flipped)
                got = T.np64(out[b, kvh * G:(kvh + 1) * G])
                for h in range(G):
                    if h not in flipped:
                        assert T.rel_err(got[h], o[h]) <= T.TOL["bf16"], (step, b, kvh, h)
    fresh = zha.Buffers(cfg)
    zha.tree_build(cfg, fresh.tree, dev.K, dev.refs, dev.lens, fresh.status)
    torch.cuda.synchronize()
    N = w.context + steps
    for level in range(1, w.levels + 1):
        k = orc.level_nodes(N, w.chunk, level)
        assert torch.equal(buf.tree_level(level)[0][:, :, :k], fresh.tree_level(level)[0][:, :, :k])
        assert torch.equal(buf.tree_level_scales(level)[:, :, :k], fresh.tree_level_scales(level)[:, :, :k])
        assert torch.equal(buf.tree_level(level)[1][:, :, :k], fresh.tree_level(level)[1][:, :, :k])
    assert flipped_total <= max(2, steps * w.batch * w.n_q_heads // 8)

