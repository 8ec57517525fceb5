"""Parity at the 1M deep-tree size (B=1, Hq=32/Hkv=4, d=128, N=1,048,576,
c=4, L=6, R=16): the tree built by zha_tree_append in 4,096-token blocks
equals zha_tree_build bit for bit; sampled nodes equal planes computed
straight from their raw keys; and one whole group routes (256 top nodes,
262,144 level-1 candidates per query row, which the selection spreads over
many CTAs per row) and attends like the oracle at p = 0.9, 0.95 and 0.99."""
import numpy as np
import pytest
import torch

import zha_oracle as orc
import zha_testlib as T
from tree_indexed_sparse_02_b200.inputs import DEEP_1M, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def case():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_indexed_sparse_02_b200 import zha
    w = DEEP_1M
    cap = w.context + 64
    inp = make_inputs(w, device="cuda", capacity=cap)
    cfg = T.make_cfg(zha, w, cap)
    buf = zha.Buffers(cfg)
    lens = torch.zeros_like(inp.lens)
    block = 4096
    for start in range(0, w.context, block):
        lens.fill_(min(start + block, w.context))
        zha.tree_append(cfg, buf.tree, inp.K, inp.refs, lens, min(block, w.context - start), buf.status)
    torch.cuda.synchronize()
    buf.check_status("1M appends")
    return zha, w, cfg, inp, buf


def test_appended_tree_equals_build(case):
    zha, w, cfg, inp, buf = case
    ref = zha.Buffers(cfg, level_kept=False)
    zha.tree_build(cfg, ref.tree, inp.K, inp.refs, inp.lens, ref.status)
    torch.cuda.synchronize()
    ref.check_status("1M build")
    for level in range(1, w.levels + 1):
        k = orc.level_nodes(w.context, w.chunk, level)
        mu_a, b_a = buf.tree_level(level)
        mu_r, b_r = ref.tree_level(level)
        assert torch.equal(mu_a[:, :, :k], mu_r[:, :, :k]), level
        assert torch.equal(b_a[:, :, :k], b_r[:, :, :k]), level
    del ref
    torch.cuda.empty_cache()


def test_sampled_nodes_match_planes_from_raw_keys(case):
    zha, w, cfg, inp, buf = case
    s = T.scale_of(w)
    g = np.random.default_rng(1)
    N = w.context
    n1 = N // w.chunk
    for kvh in (0, 3):
        refs = T.np64(inp.refs[kvh])
        for level in range(1, w.levels + 1):
            n_l = orc.level_nodes(N, w.chunk, level)
            mu_g, b_g = buf.tree_level(level)
            span = w.chunk ** level
            for node in sorted(set(g.integers(0, n_l, size=2).tolist()) | {n_l - 1}):
                t0, t1 = node * span, min((node + 1) * span, n1 * w.chunk)
                mu, bias = orc.direct_planes(T.np64(inp.K[0, kvh, t0:t1]), 0, t1 - t0, refs, s)
                assert T.rel_err(T.np64(mu_g[0, kvh, node]), mu) <= 2e-2, (kvh, level, node)
                assert T.rel_err(T.np64(b_g[0, kvh, node]), bias) <= 2e-2, (kvh, level, node)


@pytest.mark.parametrize("p", [0.9, 0.95, 0.99])
def test_one_group_routes_and_attends_like_the_oracle(case, p):
    zha, w, cfg, inp, buf = case
    zha.route(cfg, buf.tree, inp.q, inp.lens, p, buf.sel, buf.workspace, buf.status)
    out = torch.zeros_like(inp.q)
    zha.sparse_attn(cfg, inp.q, inp.K, inp.V, inp.lens, buf.sel, out, buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status("1M route/attend")
    # the level-1 rows are large enough for the multi-CTA selection
    assert int(buf.level_state(1)["count"][0, 1]) > 65536
    T.check_group_vs_oracle(w, inp, buf, 0, 1, [p] * w.levels, out=out)
