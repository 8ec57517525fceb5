"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle on the
same seeded inputs, at sizes the oracle finishes in seconds."""
import math

import numpy as np
import pytest
import torch

import zha_oracle as orc
import zha_testlib as T
from tree_indexed_sparse_02_b200.inputs import TINY_F32, Workload, make_inputs, random_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_indexed_sparse_02_b200 import zha as z
    return z


CASES = T.small_workloads()
IDS = [w.name for w in CASES]
# plane counts below 16 (several candidates share one MMA tile)
PACK_CASES = [Workload("R2 d64 c=4 L=3", 1, 16, 2, 64, 2047, 4, 3, 2, 0.9, 8, "bf16", 14),
              Workload("R4 G16 c=8 L=3", 1, 32, 2, 128, 3001, 8, 3, 4, 0.9, 8, "bf16", 15),
              Workload("R8 B=2 c=4 L=4", 2, 8, 1, 128, 2500, 4, 4, 8, 0.95, 8, "bf16", 16)]


def _lens_for(w):
    # a ragged batch: the second sequence (if any) a little shorter, not a multiple of c
    if w.batch == 1:
        return None
    return [w.context] + [w.context - 3 * b - 1 for b in range(1, w.batch)]


# ---------------------------------------------------------------- tree build


@pytest.mark.parametrize("w", CASES, ids=IDS)
def test_tree_build_matches_oracle(zha, w):
    cfg, inp, dev, buf = T.build_case(zha, w, lens=_lens_for(w))
    zha.tree_build(cfg, buf.tree, dev.K, dev.refs, dev.lens, buf.status)
    torch.cuda.synchronize()
    buf.check_status()
    s = T.scale_of(w)
    tol = T.TOL[w.dtype]
    for b in range(w.batch):
        N = int(inp.lens[b])
        for kvh in range(w.n_kv_heads):
            t = T.oracle_tree(w, inp, b, kvh, N, s)
            for level in range(1, w.levels + 1):
                n = orc.level_nodes(N, w.chunk, level)
                mu_g, b_g = buf.tree_level(level)
                emu = T.rel_err(T.np64(mu_g[b, kvh, :n]), t.mu[level - 1][:n])
                eb = T.rel_err(T.np64(b_g[b, kvh, :n]), t.b[level - 1][:n])
                eF = T.rel_err(T.np64(buf.tree_level_logmass(level)[b, kvh, :n]), t.F[level - 1][:n])
                assert emu <= tol and eb <= tol and eF <= tol, (b, kvh, level, emu, eb, eF)


@pytest.mark.parametrize("w", CASES, ids=IDS)
@pytest.mark.parametrize("block", [1, 3, 4, 9, 1000, 4096])
def test_append_equals_build_bitexact(zha, w, block):
    """Appending in blocks (decode-sized ones through the single-leaf path,
    larger ones through the bulk leaf kernel) equals a build at once, bit for bit."""
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
    ref.check_status()
    for level in range(1, w.levels + 1):
        k = orc.level_nodes(N, w.chunk, level)
        mu_a, b_a = buf.tree_level(level)
        mu_r, b_r = ref.tree_level(level)
        assert torch.equal(mu_a[:, :, :k], mu_r[:, :, :k]), level
        assert torch.equal(b_a[:, :, :k], b_r[:, :, :k]), level
        assert torch.equal(buf.tree_level_logmass(level)[:, :, :k], ref.tree_level_logmass(level)[:, :, :k]), level


# ------------------------------------------------------------- top-p select


def _score_sets(seed, n_sets, stride):
    g = torch.Generator().manual_seed(seed)
    scores = torch.randn((n_sets, stride), generator=g) * torch.rand((n_sets, 1), generator=g) * 4
    counts = torch.randint(0, stride + 1, (n_sets,), generator=g, dtype=torch.int32)
    counts[0], counts[1], counts[2] = 0, 1, stride
    # exact ties: repeat values inside some sets
    scores[3, 1::2] = scores[3, 0::2][: scores[3, 1::2].shape[0]]
    scores[4, :] = 0.25
    scores[5, : stride // 2] = -1.5
    # a crossing among many exactly equal scores below a distinct maximum (more
    # equal members than the value-bucket path holds: the radix path decides)
    scores[6, :] = -3.0 + torch.rand(stride, generator=g) * 0.5
    scores[6, ::2] = 1.0
    scores[6, 0] = 2.0
    counts[6] = stride
    # a crossing inside a dense cluster of close but distinct scores
    scores[7, :] = 0.5 + torch.arange(stride, dtype=torch.float32) * 1e-6
    counts[7] = stride
    return scores, counts


@pytest.mark.parametrize("p", [0.3, 0.9, 0.95, 0.99, 1.0])
@pytest.mark.parametrize("stride", [7, 300, 5000, 70000])
def test_topp_select_matches_oracle(zha, p, stride):
    scores, counts = _score_sets(stride, 12, stride)
    kept = torch.zeros((12, stride), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    zha.topp_select(scores.cuda(), counts.cuda(), p, kept, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kept = kept.cpu().numpy().astype(bool)
    boundary = 0
    for i in range(12):
        n = int(counts[i])
        E = scores[i, :n].double().numpy()
        ko, cb = orc.topp_select(E, p)
        kg = kept[i, :n]
        assert not kept[i, n:].any()
        diff = np.nonzero(ko != kg)[0]
        for j in diff:
            assert abs(cb[j] - p) <= 1e-5, (i, j, cb[j], p)
        boundary += diff.size
    assert boundary <= 2


def test_topp_select_many_near_equal_masses(zha):
    """Sets of more than 2^17 candidates at p = 0.99, where the fixed-point
    mass sum's error bound (n 2^-32 of the largest mass) matters most: close
    but distinct scores, exactly equal scores, and a few large masses over a
    sea of near-equal small ones. Differences from the oracle are allowed only
    within 1e-5 + n 2^-32 / Z of p."""
    n = 140_000
    g = torch.Generator().manual_seed(9)
    scores = torch.empty((4, n))
    scores[0] = 0.5 + torch.rand(n, generator=g) * 1e-4
    scores[1] = -2.0
    scores[2] = torch.rand(n, generator=g) * 1e-3 - 12.0
    scores[2, torch.randint(0, n, (8,), generator=g)] = 0.0
    scores[3] = torch.randn(n, generator=g) * 0.01
    counts = torch.full((4,), n, dtype=torch.int32)
    kept = torch.zeros((4, n), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    zha.topp_select(scores.cuda(), counts.cuda(), 0.99, kept, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kept = kept.cpu().numpy().astype(bool)
    for i in range(4):
        E = scores[i].double().numpy()
        ko, cb = orc.topp_select(E, 0.99)
        band = 1e-5 + T.fixed_point_band(E)
        diff = np.nonzero(ko != kept[i])[0]
        for j in diff:
            assert abs(cb[j] - 0.99) <= band, (i, j, cb[j])
        assert diff.size <= 2, (i, diff.size)


# ------------------------------------------------------------------ routing


@pytest.mark.parametrize("w", CASES + PACK_CASES, ids=IDS + [w.name for w in PACK_CASES])
def test_route_matches_oracle(zha, w):
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
            assert worst <= T.TOL[w.dtype], worst
            total_flipped += len(flipped)
            # the selection is the union of the level-1 kept sets, ascending
            cnt = int(buf.sel["count"][b, kvh])
            idx = buf.sel["leaf_idx"][b, kvh, :cnt].cpu().numpy()
            assert np.all(np.diff(idx) > 0)
            hm = buf.sel["head_mask"][b, kvh, :cnt].cpu().numpy().astype(np.uint32)
            for h in range(G):
                if h in flipped:
                    continue
                want = np.nonzero(r.kept[0][h])[0]
                got = idx[(hm >> np.uint32(h)) & 1 != 0]
                assert np.array_equal(np.sort(got), want), (b, kvh, h)
                lk = buf.sel["level_kept"][b, kvh * G + h].cpu().numpy()
                for level in range(1, w.levels + 1):
                    assert lk[level - 1] == r.kept[level - 1][h].sum()
    heads = w.batch * w.n_q_heads
    if w.dtype == "f32":
        assert total_flipped == 0
    else:
        assert total_flipped <= max(2, heads // 8), total_flipped


@pytest.mark.parametrize("w", CASES[1:4], ids=IDS[1:4])
def test_route_depth_schedule_matches_oracle(zha, w):
    """Routing with the depth-root schedule p^(1/L) per level (from zha_p_schedule)
    equals the oracle's routing with the same per-level fractions."""
    cfg, inp, dev, buf = T.build_case(zha, w, lens=_lens_for(w))
    zha.tree_build(cfg, buf.tree, dev.K, dev.refs, dev.lens, buf.status)
    p_levels = zha.p_schedule(w.p, w.levels, "root")
    assert all(p > w.p for p in p_levels)
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
            r = orc.route(t, q, p_levels)
            flipped, worst = T.compare_routing(r, states, b, kvh, G, N, w, p_levels)
            assert worst <= T.TOL[w.dtype], worst
            total_flipped += len(flipped)
            for h in range(G):
                if h in flipped:
                    continue
                lk = buf.sel["level_kept"][b, kvh * G + h].cpu().numpy()
                for level in range(1, w.levels + 1):
                    assert lk[level - 1] == r.kept[level - 1][h].sum()
    assert total_flipped <= max(2, w.batch * w.n_q_heads // 8), total_flipped


# ------------------------------------------------------------------ attention


def _oracle_attn(inp, b, kvh, G, N, s, masks):
    K = T.np64(inp.K[b, kvh, :N])
    V = T.np64(inp.V[b, kvh, :N])
    q = T.np64(inp.q[b, kvh * G:(kvh + 1) * G])
    return np.stack([orc.attend(q[h], K, V, N, s, masks[h]) for h in range(G)])


def _random_sel(zha, cfg, w, inp, frac, seed, force=()):
    """A generator-made selection per group (ascending leaves, non-zero head masks)."""
    G = w.group
    cap1 = zha.level_nodes(cfg, cfg.max_len, 1)
    sel = {"leaf_idx": torch.zeros((w.batch, w.n_kv_heads, cap1), dtype=torch.int32),
           "head_mask": torch.zeros((w.batch, w.n_kv_heads, cap1), dtype=torch.int32),
           "count": torch.zeros((w.batch, w.n_kv_heads), dtype=torch.int32), "level_kept": None}
    for b in range(w.batch):
        n1 = int(inp.lens[b]) // w.chunk
        for kvh in range(w.n_kv_heads):
            idx, m = random_selection(n1, G, frac, seed + 17 * b + kvh)
            idx, m = idx.tolist(), m.tolist()
            for f in force:          # e.g. leaf 0 or the last leaf, for some heads
                j = f if f >= 0 else n1 + f
                if 0 <= j < n1 and j not in idx:
                    pos = int(np.searchsorted(idx, j))
                    idx.insert(pos, j)
                    m.insert(pos, 1)
            sel["leaf_idx"][b, kvh, :len(idx)] = torch.tensor(idx, dtype=torch.int32)
            sel["head_mask"][b, kvh, :len(idx)] = torch.tensor(m, dtype=torch.int64).to(torch.int32)
            sel["count"][b, kvh] = len(idx)
    return {k: (v.cuda() if v is not None else None) for k, v in sel.items()}


SEL_CASES = [(0.0, ()), (0.05, ()), (0.3, (0, -1)), (0.9, (0,)), (1.0, ())]


@pytest.mark.parametrize("w", CASES, ids=IDS)
@pytest.mark.parametrize("frac,force", SEL_CASES, ids=[f"{f}-{c}" for f, c in SEL_CASES])
def test_sparse_attn_on_given_selection(zha, w, frac, force):
    cfg, inp, dev, buf = T.build_case(zha, w, lens=_lens_for(w))
    sel = _random_sel(zha, cfg, w, inp, frac, 100 + int(frac * 100), force)
    out = torch.zeros_like(dev.q)
    zha.sparse_attn(cfg, dev.q, dev.K, dev.V, dev.lens, sel, out, buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status()
    s = T.scale_of(w)
    G = w.group
    for b in range(w.batch):
        N = int(inp.lens[b])
        for kvh in range(w.n_kv_heads):
            masks = T.selection_to_masks(sel, b, kvh, G, N, w.chunk)
            ref = _oracle_attn(inp, b, kvh, G, N, s, masks)
            got = T.np64(out[b, kvh * G:(kvh + 1) * G])
            assert T.rel_err(got, ref) <= T.TOL[w.dtype], (b, kvh)


@pytest.mark.parametrize("w", CASES, ids=IDS)
def test_dense_decode_matches_oracle(zha, w):
    cfg, inp, dev, buf = T.build_case(zha, w, lens=_lens_for(w))
    out = torch.zeros_like(dev.q)
    zha.dense_decode(cfg, dev.q, dev.K, dev.V, dev.lens, out, buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status()
    s = T.scale_of(w)
    G = w.group
    for b in range(w.batch):
        N = int(inp.lens[b])
        for kvh in range(w.n_kv_heads):
            ref = _oracle_attn(inp, b, kvh, G, N, s, [None] * G)
            got = T.np64(out[b, kvh * G:(kvh + 1) * G])
            assert T.rel_err(got, ref) <= T.TOL[w.dtype]


@pytest.mark.parametrize("N", [1, 2, 3, 4, 5, 7, 8, 64, 65, 1001])
@pytest.mark.parametrize("tail_only", [False, True])
def test_sparse_attn_edge_lengths(zha, N, tail_only):
    """Short caches (N < c, N = c, ragged) with empty, full and sink/tail-overlapping selections."""
    w = Workload("edge", 1, 8, 1, 128, N, 4, 3, 16, 0.9, 0, "bf16", 21)
    flags = zha.ZHA_FLAG_TAIL_ONLY if tail_only else 0
    cap = N + 16
    inp = make_inputs(w, capacity=cap)
    dev = T.to_device(inp)
    cfg = T.make_cfg(zha, w, cap, flags=flags)
    buf = zha.Buffers(cfg)
    for frac, force in [(0.0, ()), (1.0, ()), (0.5, (0, -1))]:
        sel = _random_sel(zha, cfg, w, inp, frac, 7, force)
        out = torch.zeros_like(dev.q)
        zha.sparse_attn(cfg, dev.q, dev.K, dev.V, dev.lens, sel, out, buf.workspace, buf.status)
        torch.cuda.synchronize()
        buf.check_status()
        masks = T.selection_to_masks(sel, 0, 0, 8, N, 4, tail_only)
        ref = _oracle_attn(inp, 0, 0, 8, N, T.scale_of(w), masks)
        assert T.rel_err(T.np64(out[0]), ref) <= 2e-2, (N, frac)


def test_p1_routes_all_and_equals_dense(zha):
    w = CASES[1]
    cfg, inp, dev, buf = T.build_case(zha, w, lens=_lens_for(w))
    zha.tree_build(cfg, buf.tree, dev.K, dev.refs, dev.lens, buf.status)
    zha.route(cfg, buf.tree, dev.q, dev.lens, 1.0, buf.sel, buf.workspace, buf.status)
    out = torch.zeros_like(dev.q)
    dense = torch.zeros_like(dev.q)
    zha.sparse_attn(cfg, dev.q, dev.K, dev.V, dev.lens, buf.sel, out, buf.workspace, buf.status)
    zha.dense_decode(cfg, dev.q, dev.K, dev.V, dev.lens, dense, buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status()
    full = (1 << w.group) - 1
    for b in range(w.batch):
        n1 = int(inp.lens[b]) // w.chunk
        for kvh in range(w.n_kv_heads):
            assert int(buf.sel["count"][b, kvh]) == n1
            assert torch.all(buf.sel["head_mask"][b, kvh, :n1] == full)
    assert T.rel_err(T.np64(out), T.np64(dense)) <= 1e-2


# ------------------------------------------------------------------- decode


@pytest.mark.parametrize("w", CASES[:4], ids=IDS[:4])
def test_decode_steps_match_oracle(zha, w):
    """zha_decode appends, routes and attends; the oracle repeats each step."""
    steps = 9
    cap = w.context + steps + 8
    inp = make_inputs(w, capacity=cap)
    dev = T.to_device(inp)
    cfg = T.make_cfg(zha, w, cap)
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, dev.K, dev.refs, dev.lens, buf.status)
    G = w.group
    s = T.scale_of(w)
    g = torch.Generator().manual_seed(5)
    dt = w.torch_dtype()
    K_host = inp.K.clone()
    V_host = inp.V.clone()
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
            assert int(dev.lens[b]) == N
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
                        assert T.rel_err(got[h], o[h]) <= T.TOL[w.dtype], (step, b, kvh, h)
    # after the steps the incrementally extended tree equals a fresh build
    fresh = zha.Buffers(cfg)
    zha.tree_build(cfg, fresh.tree, dev.K, dev.refs, dev.lens, fresh.status)
    torch.cuda.synchronize()
    N = w.context + steps
    for level in range(1, w.levels + 1):
        k = orc.level_nodes(N, w.chunk, level)
        assert torch.equal(buf.tree_level(level)[0][:, :, :k], fresh.tree_level(level)[0][:, :, :k])
        assert torch.equal(buf.tree_level(level)[1][:, :, :k], fresh.tree_level(level)[1][:, :, :k])
    assert flipped_total <= max(2, steps * w.batch * w.n_q_heads // 8)


# -------------------------------------------------------------- error paths


def test_device_errors_are_reported_not_trapped(zha):
    w = TINY_F32
    cfg, inp, dev, buf = T.build_case(zha, w, extra_cap=0)
    # lens beyond max_len -> capacity error, nothing read out of bounds
    lens = torch.full_like(dev.lens, cfg.max_len + 5)
    zha.tree_build(cfg, buf.tree, dev.K, dev.refs, lens, buf.status)
    torch.cuda.synchronize()
    assert int(buf.status.item()) == 3
    buf.status.zero_()
    # a leaf index out of range in a caller selection -> invalid argument
    sel = _random_sel(zha, cfg, w, inp, 0.1, 3)
    sel["leaf_idx"][0, 0, 0] = 10 ** 6
    out = torch.zeros_like(dev.q)
    zha.sparse_attn(cfg, dev.q, dev.K, dev.V, dev.lens, sel, out, buf.workspace, buf.status)
    torch.cuda.synchronize()
    assert int(buf.status.item()) == 1
    buf.status.zero_()
    # decode on a full cache -> capacity error, lens unchanged
    full = torch.full_like(dev.lens, cfg.max_len)
    z = torch.zeros((1, 1, 64), dtype=torch.float32, device="cuda")
    zha.decode(cfg, buf.tree, dev.K, dev.V, dev.refs, full, dev.q, z, z, 0.9, buf.sel, out,
               buf.workspace, buf.status)
    torch.cuda.synchronize()
    assert int(buf.status.item()) == 3
    assert int(full.item()) == cfg.max_len
    with pytest.raises(zha.ZhaError):
        zha.route(cfg, buf.tree, dev.q, dev.lens, -0.5, buf.sel, buf.workspace, buf.status)
