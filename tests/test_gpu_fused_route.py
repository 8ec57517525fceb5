"""The fused route (ZHA_FLAG_FUSED_ROUTE: one launch, one thread-block cluster
per (sequence, KV head) walking every level) against the fp64 oracle, and
against the default per-level launches, whose scores and selections it must
reproduce bit for bit: few kept nodes (aligned references), many (random
references: more candidates per level than the cluster's shared memory
holds), a ragged batch, head_dim 64, many groups (8-CTA clusters), fewer
query rows than CTAs, a cache shorter than one chunk, and decode steps
(against the default path and against the oracle repeating each step)."""
import dataclasses

import numpy as np
import pytest
import torch

import zha_testlib as T
from tree_indexed_sparse_02_b200.inputs import WIDE_32K, Workload, decode_stream, make_inputs

pytestmark = pytest.mark.gpu

CASES = [Workload("deep bf16 B=2 c=4 L=4", 2, 16, 2, 128, 3001, 4, 4, 16, 0.95, 16, "bf16", 11),
         Workload("deep aligned N=65536 L=6", 1, 32, 4, 128, 65536, 4, 6, 16, 0.95, 64, "bf16", 5,
                  refs_mode="aligned"),
         Workload("deep random N=65536 L=6", 1, 32, 4, 128, 65536, 4, 6, 16, 0.95, 64, "bf16", 6),
         Workload("d64 aligned B=2 c=4 L=5", 2, 16, 2, 64, 20000, 4, 5, 16, 0.9, 16, "bf16", 31,
                  refs_mode="aligned"),
         dataclasses.replace(WIDE_32K, name="wide aligned N=32768 c=256", refs_mode="aligned"),
         # many groups (clusters of 8 CTAs: the 16-CTA clusters of 20 groups do not all fit at once)
         Workload("20 groups B=5 aligned c=4 L=5", 5, 32, 4, 128, 6000, 4, 5, 16, 0.9, 16, "bf16", 41,
                  refs_mode="aligned"),
         # four query rows per group (CTAs that own no row)
         Workload("G=4 d64 B=2 c=4 L=4", 2, 16, 4, 64, 9000, 4, 4, 16, 0.9, 16, "bf16", 43)]
IDS = [w.name for w in CASES]


@pytest.fixture(scope="module")
def zha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_indexed_sparse_02_b200 import zha as z
    return z


def _lens(w):
    return None if w.batch == 1 else [w.context] + [w.context - 7 * b - 2 for b in range(1, w.batch)]


def _routed(zha, w, inp, flags):
    cap = w.context + 64
    cfg = T.make_cfg(zha, w, cap, flags=flags)
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, inp.K, inp.refs, inp.lens, buf.status)
    zha.route(cfg, buf.tree, inp.q, inp.lens, w.p, buf.sel, buf.workspace, buf.status)
    out = torch.zeros_like(inp.q)
    zha.sparse_attn(cfg, inp.q, inp.K, inp.V, inp.lens, buf.sel, out, buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status()
    return cfg, buf, out


@pytest.mark.parametrize("w", CASES, ids=IDS)
def test_fused_route_matches_oracle_and_default(zha, w):
    inp = make_inputs(w, capacity=w.context + 64, lens=_lens(w))
    dev = T.to_device(inp)
    cfg, fused, out_f = _routed(zha, w, dev, zha.ZHA_FLAG_FUSED_ROUTE)
    _, ref, out_r = _routed(zha, w, dev, 0)
    # the oracle, group by group (level by level, selections, outputs)
    flipped = 0
    for b in range(w.batch):
        for kvh in range(w.n_kv_heads):
            flipped += len(T.check_group_vs_oracle(w, inp, fused, b, kvh, [w.p] * w.levels, out=out_f))
    assert flipped <= max(2, w.batch * w.n_q_heads // 8), flipped
    # the default launches: same candidates, scores, kept masks, selection and output
    for level in range(1, w.levels + 1):
        a, r = fused.level_state(level), ref.level_state(level)
        assert torch.equal(a["count"], r["count"]), level
        for b in range(w.batch):
            for kvh in range(w.n_kv_heads):
                n = int(r["count"][b, kvh])
                for key in ("cand_idx", "cand_mask", "kept_mask"):
                    assert torch.equal(a[key][b, kvh, :n], r[key][b, kvh, :n]), (level, key)
                assert torch.equal(a["scores"][b, kvh, :, :n], r["scores"][b, kvh, :, :n]), level
    assert torch.equal(fused.sel["count"], ref.sel["count"])
    for b in range(w.batch):
        for kvh in range(w.n_kv_heads):
            n = int(ref.sel["count"][b, kvh])
            assert torch.equal(fused.sel["leaf_idx"][b, kvh, :n], ref.sel["leaf_idx"][b, kvh, :n])
            assert torch.equal(fused.sel["head_mask"][b, kvh, :n], ref.sel["head_mask"][b, kvh, :n])
    assert torch.equal(fused.sel["level_kept"], ref.sel["level_kept"])
    assert torch.equal(out_f, out_r)


@pytest.mark.parametrize("N", [1, 3, 5, 17])
def test_fused_route_short_caches(zha, N):
    """Caches shorter than a few chunks: an empty or tiny tree still routes."""
    w = Workload("short", 1, 8, 1, 128, N, 4, 3, 16, 0.9, 0, "bf16", 23)
    inp = make_inputs(w, capacity=N + 16)
    dev = T.to_device(inp)
    cfg, fused, out_f = _routed(zha, w, dev, zha.ZHA_FLAG_FUSED_ROUTE)
    _, ref, out_r = _routed(zha, w, dev, 0)
    assert torch.equal(fused.sel["count"], ref.sel["count"])
    assert torch.equal(out_f, out_r)


def test_fused_decode_steps_equal_default(zha):
    """zha_decode with the fused route: the same outputs and selections as the
    default launches, step after step (tokens appended, chunks completing)."""
    w = dataclasses.replace(CASES[1], name="decode aligned")
    steps = 9
    cap = w.context + steps + 8
    inp = T.to_device(make_inputs(w, capacity=cap))
    k_new, v_new, qs = decode_stream(w, steps, device="cuda")
    runs = []
    for flags in (zha.ZHA_FLAG_FUSED_ROUTE, 0):
        cfg = T.make_cfg(zha, w, cap, flags=flags)
        buf = zha.Buffers(cfg)
        K, V, lens = inp.K.clone(), inp.V.clone(), inp.lens.clone()
        zha.tree_build(cfg, buf.tree, K, inp.refs, lens, buf.status)
        outs, sels = [], []
        for i in range(steps):
            out = torch.zeros_like(qs[i])
            zha.decode(cfg, buf.tree, K, V, inp.refs, lens, qs[i], k_new[i], v_new[i], w.p, buf.sel, out,
                       buf.workspace, buf.status)
            outs.append(out)
            sels.append(buf.sel["count"].clone())
        torch.cuda.synchronize()
        buf.check_status()
        runs.append((outs, sels))
    for (of, sf), (orr, sr) in zip(zip(*runs[0]), zip(*runs[1])):
        assert torch.equal(of, orr)
        assert torch.equal(sf, sr)
    assert np.isfinite(runs[0][0][-1].float().cpu().numpy()).all()


DECODE_CASES = [CASES[0], CASES[4], CASES[5], CASES[6],
                Workload("short N=3 c=4 L=3", 1, 8, 1, 128, 3, 4, 3, 16, 0.9, 0, "bf16", 29)]


@pytest.mark.parametrize("w", DECODE_CASES, ids=[w.name for w in DECODE_CASES])
def test_fused_decode_steps_match_oracle(zha, w):
    """zha_decode with the fused route against the oracle repeating each step
    (append, route, exact attention): ragged batch, the wide tree, 8-CTA
    clusters, four query rows per group, and a cache that starts shorter than
    one chunk (sink, kept leaves and current chunk overlapping)."""
    import zha_oracle as orc
    steps = 6
    cap = w.context + steps + 8
    inp = make_inputs(w, capacity=cap, lens=_lens(w))
    dev = T.to_device(inp)
    cfg = T.make_cfg(zha, w, cap, flags=zha.ZHA_FLAG_FUSED_ROUTE)
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, dev.K, dev.refs, dev.lens, buf.status)
    G = w.group
    s = T.scale_of(w)
    g = torch.Generator().manual_seed(7)
    dt = w.torch_dtype()
    K_host, V_host = inp.K.clone(), inp.V.clone()
    lens0 = [int(x) for x in inp.lens]
    trees = {(b, kvh): T.oracle_tree(w, inp, b, kvh, lens0[b], s, cap)
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
            N = lens0[b] + step + 1
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
    assert flipped_total <= max(2, steps * w.batch * w.n_q_heads // 8)


@pytest.mark.parametrize("p", [1.0, 0.5])
def test_fused_route_p_edges(zha, p):
    """p = 1 keeps every member (the selection's shortcut); p = 0.5 keeps few:
    both equal the per-level launches bit for bit."""
    w = dataclasses.replace(CASES[0], name=f"p={p}", p=p)
    inp = make_inputs(w, capacity=w.context + 64, lens=_lens(w))
    dev = T.to_device(inp)
    _, fused, out_f = _routed(zha, w, dev, zha.ZHA_FLAG_FUSED_ROUTE)
    _, ref, out_r = _routed(zha, w, dev, 0)
    assert torch.equal(fused.sel["count"], ref.sel["count"])
    assert torch.equal(fused.sel["level_kept"], ref.sel["level_kept"])
    assert torch.equal(out_f, out_r)


@pytest.mark.parametrize("noise", [0.0, 1e-3])
def test_fused_route_equal_scores(zha, noise):
    """Keys that are all equal (every node of a level scores the same: one
    bucket holding every candidate, more than the ranked list takes, so the
    warp selection decides, ties by node index) and keys a hair apart (a
    crowded crossing bucket): the fused route equals the per-level launches
    bit for bit, level by level."""
    w = Workload(f"equal keys noise={noise}", 1, 16, 2, 128, 65536, 4, 4, 16, 0.9, 0, "bf16", 47)
    inp = make_inputs(w, capacity=w.context + 64)
    g = torch.Generator().manual_seed(3)
    base = torch.randn(w.head_dim, generator=g)
    K = base.expand_as(inp.K).clone() + noise * torch.randn(inp.K.shape, generator=g)
    inp = dataclasses.replace(inp, K=K.to(inp.K.dtype))
    dev = T.to_device(inp)
    _, fused, out_f = _routed(zha, w, dev, zha.ZHA_FLAG_FUSED_ROUTE)
    _, ref, out_r = _routed(zha, w, dev, 0)
    for level in range(1, w.levels + 1):
        a, r = fused.level_state(level), ref.level_state(level)
        assert torch.equal(a["count"], r["count"]), level
        for kvh in range(w.n_kv_heads):
            n = int(r["count"][0, kvh])
            assert torch.equal(a["kept_mask"][0, kvh, :n], r["kept_mask"][0, kvh, :n]), level
    assert torch.equal(fused.sel["count"], ref.sel["count"])
    assert torch.equal(out_f, out_r)


def test_fused_flag_with_other_options(zha):
    """The fused flag next to the tcgen05 scorer flag (the fused route runs)
    and with MX-FP8 summaries (outside the fused route's scope: the per-level
    route runs): each equals the per-level route of the same configuration
    bit for bit."""
    w = CASES[0]
    inp = make_inputs(w, capacity=w.context + 64, lens=_lens(w))
    dev = T.to_device(inp)
    _, a, out_a = _routed(zha, w, dev, zha.ZHA_FLAG_FUSED_ROUTE | zha.ZHA_FLAG_TCGEN05)
    _, r, out_r = _routed(zha, w, dev, 0)
    assert torch.equal(a.sel["count"], r.sel["count"])
    assert torch.equal(out_a, out_r)
    wm = dataclasses.replace(w, name="mx", summary="mxfp8")
    _, a, out_a = _routed(zha, wm, dev, zha.ZHA_FLAG_FUSED_ROUTE)
    _, r, out_r = _routed(zha, wm, dev, 0)
    assert torch.equal(a.sel["count"], r.sel["count"])
    assert torch.equal(out_a, out_r)


@pytest.mark.parametrize("flags,dtype,max_len,fused", [(4, "bf16", 16384, True), (0, "bf16", 16384, False),
                                                       (4, "f32", 16384, False), (4, "bf16", 16400, False)])
def test_route_fused_query_names_the_launch(zha, flags, dtype, max_len, fused):
    """zha_route_fused says which routing zha_route runs: the fused kernel
    appears in the launch record exactly when it answers 1 (a two-level tree
    of 4-token chunks has 1,024 top-level nodes at 16,384 tokens and 1,025 at
    16,400, where it routes per level)."""
    w = Workload("query", 1, 32, 4, 128, 3000, 4, 2, 16, 0.95, 16, dtype, 13, refs_mode="aligned")
    inp = T.to_device(make_inputs(w, capacity=max_len))
    cfg = T.make_cfg(zha, w, max_len, flags=flags)
    assert zha.route_fused(cfg) == fused
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, inp.K, inp.refs, inp.lens, buf.status)
    torch.cuda.synchronize()
    zha.profile_read()
    zha.profile_enable(True)
    try:
        zha.route(cfg, buf.tree, inp.q, inp.lens, w.p, buf.sel, buf.workspace, buf.status)
        torch.cuda.synchronize()
        names = zha.profile_read()
    finally:
        zha.profile_enable(False)
    buf.check_status()
    assert ("route_fused" in names) == fused, sorted(names)
