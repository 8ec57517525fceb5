"""Parity at the benchmark's full size: the 256K deep-tree workload (B=4,
Hq=32/Hkv=4, d=128, N=262,144, c=4, L=6, R=16, p=0.95), built and decoded on
the GPU in the launch configuration bench.py times, checked on outputs the
oracle can compute one by one: sampled tree nodes (against planes computed
straight from their raw keys), one whole group's routing and attention, and
dense attention for sampled heads."""
import numpy as np
import pytest
import torch

import zha_oracle as orc
import zha_testlib as T
from tree_indexed_sparse_02_b200.inputs import DEEP_256K, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def case():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_indexed_sparse_02_b200 import zha
    w = DEEP_256K
    cap = w.context + 64
    inp = make_inputs(w, device="cuda", capacity=cap)
    cfg = T.make_cfg(zha, w, cap)
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, inp.K, inp.refs, inp.lens, buf.status)
    zha.route(cfg, buf.tree, inp.q, inp.lens, w.p, buf.sel, buf.workspace, buf.status)
    out = torch.zeros_like(inp.q)
    zha.sparse_attn(cfg, inp.q, inp.K, inp.V, inp.lens, buf.sel, out, buf.workspace, buf.status)
    dense = torch.zeros_like(inp.q)
    zha.dense_decode(cfg, inp.q, inp.K, inp.V, inp.lens, dense, buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status("full-size build/route/attend")
    return zha, w, cfg, inp, buf, out, dense


def test_sampled_nodes_match_planes_from_raw_keys(case):
    zha, w, cfg, inp, buf, out, dense = case
    s = T.scale_of(w)
    g = np.random.default_rng(0)
    N = w.context
    n1 = N // w.chunk
    for b, kvh in [(0, 0), (1, 3), (3, 2)]:
        refs = T.np64(inp.refs[kvh])
        for level in range(1, w.levels + 1):
            n_l = orc.level_nodes(N, w.chunk, level)
            mu_g, b_g = buf.tree_level(level)
            span = w.chunk ** level
            for node in sorted(set(g.integers(0, n_l, size=3).tolist()) | {n_l - 1}):
                t0, t1 = node * span, min((node + 1) * span, n1 * w.chunk)
                mu, bias = orc.direct_planes(T.np64(inp.K[b, kvh, t0:t1]), 0, t1 - t0, refs, s)
                assert T.rel_err(T.np64(mu_g[b, kvh, node]), mu) <= 2e-2, (b, kvh, level, node)
                assert T.rel_err(T.np64(b_g[b, kvh, node]), bias) <= 2e-2, (b, kvh, level, node)


def test_one_group_routes_and_attends_like_the_oracle(case):
    zha, w, cfg, inp, buf, out, dense = case
    b, kvh = 2, 1
    G, N, s = w.group, w.context, T.scale_of(w)
    t = T.oracle_tree(w, inp, b, kvh, N, s)
    K = T.np64(inp.K[b, kvh, :N])
    V = T.np64(inp.V[b, kvh, :N])
    q = T.np64(inp.q[b, kvh * G:(kvh + 1) * G])
    o, r, masks = orc.decode_group(t, q, K, V, w.p)
    states = {l: buf.level_state(l) for l in range(1, w.levels + 1)}
    flipped, worst = T.compare_routing(r, states, b, kvh, G, N, w, [w.p] * w.levels)
    assert worst <= 2e-2
    assert len(flipped) <= 2
    got = T.np64(out[b, kvh * G:(kvh + 1) * G])
    for h in range(G):
        if h not in flipped:
            assert T.rel_err(got[h], o[h]) <= 2e-2, h


def test_sampled_dense_heads_match_oracle(case):
    zha, w, cfg, inp, buf, out, dense = case
    s = T.scale_of(w)
    G = w.group
    for b, hq in [(0, 0), (1, 17), (3, 31)]:
        kvh = hq // G
        ref = orc.attend(T.np64(inp.q[b, hq]), T.np64(inp.K[b, kvh, :w.context]),
                         T.np64(inp.V[b, kvh, :w.context]), w.context, s)
        assert T.rel_err(T.np64(dense[b, hq]), ref) <= 2e-2, (b, hq)


def test_decode_step_at_full_size(case):
    """One zha_decode step on the full workload: the cache grows by one token
    and the step's output equals sparse attention over its own selection."""
    zha, w, cfg, inp, buf, out, dense = case
    k_new = torch.randn((w.batch, w.n_kv_heads, w.head_dim), device="cuda").to(torch.bfloat16)
    v_new = torch.randn((w.batch, w.n_kv_heads, w.head_dim), device="cuda").to(torch.bfloat16)
    q = torch.randn((w.batch, w.n_q_heads, w.head_dim), device="cuda").to(torch.bfloat16)
    o1 = torch.zeros_like(q)
    zha.decode(cfg, buf.tree, inp.K, inp.V, inp.refs, inp.lens, q, k_new, v_new, w.p, buf.sel, o1,
               buf.workspace, buf.status)
    o2 = torch.zeros_like(q)
    zha.sparse_attn(cfg, q, inp.K, inp.V, inp.lens, buf.sel, o2, buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status("full-size decode")
    assert torch.all(inp.lens == w.context + 1)
    assert torch.equal(o1, o2)
    # the new token is attended by every head (it is in the current chunk)
    b, kvh = 0, 0
    N = w.context + 1
    masks = T.selection_to_masks(buf.sel, b, kvh, w.group, N, w.chunk)
    assert all(m[N - 1] and m[0] for m in masks)
