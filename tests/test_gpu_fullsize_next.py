"""Parity at the benchmark's full size (256K deep tree, B=4, Hq=32/Hkv=4,
d=128, N=262,144, c=4, L=6, R=16, p=0.95) for the extensions: MX-FP8
summaries and a multi-query block of 4 positions, each checked on one whole
group against the oracle (routing level by level, then the outputs)."""
import dataclasses

import numpy as np
import pytest
import torch

import zha_oracle as orc
import zha_testlib as T
from tree_indexed_sparse_02_b200.inputs import DEEP_256K, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_indexed_sparse_02_b200 import zha as z
    return z


def test_mx_fullsize_group_matches_oracle(zha):
    w = dataclasses.replace(DEEP_256K, summary="mxfp8")
    cap = w.context + 64
    inp = make_inputs(w, device="cuda", capacity=cap)
    cfg = T.make_cfg(zha, w, cap)
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, inp.K, inp.refs, inp.lens, buf.status)
    zha.route(cfg, buf.tree, inp.q, inp.lens, w.p, buf.sel, buf.workspace, buf.status)
    out = torch.zeros_like(inp.q)
    zha.sparse_attn(cfg, inp.q, inp.K, inp.V, inp.lens, buf.sel, out, buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status("mx full-size")
    b, kvh = 1, 2
    G, N, s = w.group, w.context, T.scale_of(w)
    t = T.oracle_tree(w, inp, b, kvh, N, s)
    o, r, masks = orc.decode_group(t, T.np64(inp.q[b, kvh * G:(kvh + 1) * G]), T.np64(inp.K[b, kvh, :N]),
                                   T.np64(inp.V[b, kvh, :N]), w.p)
    states = {l: buf.level_state(l) for l in range(1, w.levels + 1)}
    flipped, worst = T.compare_routing(r, states, b, kvh, G, N, w, [w.p] * w.levels)
    assert worst <= 2e-2 and len(flipped) <= 2
    got = T.np64(out[b, kvh * G:(kvh + 1) * G])
    for h in range(G):
        if h not in flipped:
            assert T.rel_err(got[h], o[h]) <= 2e-2, h


def test_block_fullsize_group_matches_oracle(zha):
    w = DEEP_256K
    Tb = 4
    cap = w.context + Tb + 64
    inp = make_inputs(w, device="cuda", capacity=cap)
    cfg = zha.config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.levels, w.n_refs, w.dtype, cap,
                     queries=Tb)
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, inp.K, inp.refs, inp.lens, buf.status)
    g = torch.Generator(device="cuda").manual_seed(9)
    q = torch.randn((w.batch, Tb, w.n_q_heads, w.head_dim), generator=g, device="cuda").to(torch.bfloat16)
    kn = torch.randn((w.batch, Tb, w.n_kv_heads, w.head_dim), generator=g, device="cuda").to(torch.bfloat16)
    vn = torch.randn((w.batch, Tb, w.n_kv_heads, w.head_dim), generator=g, device="cuda").to(torch.bfloat16)
    out = torch.zeros_like(q)
    zha.decode_block(cfg, Tb, buf.tree, inp.K, inp.V, inp.refs, inp.lens, q, kn, vn, w.p, buf.sel, out,
                     buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status("block full-size")
    b, kvh = 3, 1
    G, N0, s = w.group, w.context, T.scale_of(w)
    assert int(inp.lens[b]) == N0 + Tb
    t = T.oracle_tree(w, inp, b, kvh, N0, s)
    K = T.np64(inp.K[b, kvh, :N0 + Tb])           # the block's tokens were written by the call
    V = T.np64(inp.V[b, kvh, :N0 + Tb])
    assert np.array_equal(K[N0:], T.np64(kn[b, :, kvh]))
    o, r, masks = orc.decode_block_group(t, T.np64(q[b, :, kvh * G:(kvh + 1) * G]), K, V, w.p)
    states = {l: buf.level_state(l, T=Tb) for l in range(1, w.levels + 1)}
    flipped, worst = T.compare_routing(r, states, b, kvh, Tb * G, N0, w, [w.p] * w.levels)
    assert worst <= 2e-2 and len(flipped) <= 4
    got = T.np64(out[b, :, kvh * G:(kvh + 1) * G])
    for tt in range(Tb):
        for h in range(G):
            if tt * G + h not in flipped:
                assert T.rel_err(got[tt, h], o[tt, h]) <= 2e-2, (tt, h)
