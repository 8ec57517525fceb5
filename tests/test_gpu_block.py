"""zha_decode_block (T query positions per sequence sharing every summary and
KV read) against the oracle's block reading, through the C ABI: consecutive
blocks, each routed over the tree before it and attended causally, then the
tree extended; blocks of several sizes, crossing chunk boundaries."""
import numpy as np
import pytest
import torch

import zha_oracle as orc
import zha_testlib as T
from tree_indexed_sparse_02_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

BASE = T.small_workloads()
# (workload, block sizes of the consecutive calls); T * G <= 32
CASES = [(BASE[1], [4, 1, 3, 4, 2]),          # deep-small bf16 B=2 ragged, G=8
         (BASE[2], [2, 1, 2, 2]),             # G=16 R=32 d=64 c=8
         (BASE[3], [3, 4, 1, 4]),             # R=1 c=8 p=0.75
         (BASE[0], [4, 3, 4]),                # tiny fp32, G=2
         (Workload("MHA G=1 c=4 L=3", 1, 4, 4, 64, 1500, 4, 3, 8, 0.9, 4, "bf16", 17), [32, 5, 17])]
IDS = [w.name for w, _ in CASES]


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


@pytest.mark.parametrize("w,blocks", CASES, ids=IDS)
def test_decode_block_matches_oracle(zha, w, blocks):
    Tmax = max(blocks)
    cap = w.context + sum(blocks) + 8
    lens0 = _lens_for(w) or [w.context] * w.batch
    inp = make_inputs(w, capacity=cap, lens=lens0)
    dev = T.to_device(inp)
    cfg = zha.config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.levels, w.n_refs, w.dtype,
                     cap, queries=Tmax)
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, dev.K, dev.refs, dev.lens, buf.status)
    G = w.group
    s = T.scale_of(w)
    g = torch.Generator().manual_seed(7)
    dt = w.torch_dtype()
    K_host, V_host = inp.K.clone(), inp.V.clone()
    trees = {(b, kvh): T.oracle_tree(w, inp, b, kvh, lens0[b], s, cap)
             for b in range(w.batch) for kvh in range(w.n_kv_heads)}
    tol = T.TOL[w.dtype]
    flipped_total = rows_total = 0
    n_done = 0
    for Tb in blocks:
        k_new = torch.randn((w.batch, Tb, w.n_kv_heads, w.head_dim), generator=g).to(dt)
        v_new = torch.randn((w.batch, Tb, w.n_kv_heads, w.head_dim), generator=g).to(dt)
        q = torch.randn((w.batch, Tb, w.n_q_heads, w.head_dim), generator=g).to(dt)
        out = torch.zeros_like(q).cuda()
        zha.decode_block(cfg, Tb, buf.tree, dev.K, dev.V, dev.refs, dev.lens, q.cuda(), k_new.cuda(),
                         v_new.cuda(), w.p, buf.sel, out, buf.workspace, buf.status)
        torch.cuda.synchronize()
        buf.check_status()
        states = {l: buf.level_state(l, T=Tb) for l in range(1, w.levels + 1)}
        for b in range(w.batch):
            N0 = lens0[b] + n_done
            assert int(dev.lens[b]) == N0 + Tb
            for t in range(Tb):
                K_host[b, :, N0 + t] = k_new[b, t]
                V_host[b, :, N0 + t] = v_new[b, t]
            for kvh in range(w.n_kv_heads):
                tr = trees[(b, kvh)]
                assert tr.N == N0
                qg = T.np64(q[b, :, kvh * G:(kvh + 1) * G])                  # [Tb, G, d]
                Kb = T.np64(K_host[b, kvh, :N0 + Tb])
                Vb = T.np64(V_host[b, kvh, :N0 + Tb])
                o, r, masks = orc.decode_block_group(tr, qg, Kb, Vb, w.p)
                flipped, worst = T.compare_routing(r, states, b, kvh, Tb * G, N0, w, [w.p] * w.levels)
                assert worst <= tol, worst
                flipped_total += len(flipped)
                rows_total += Tb * G
                got = T.np64(out[b, :, kvh * G:(kvh + 1) * G])
                for t in range(Tb):
                    for h in range(G):
                        if t * G + h not in flipped:
                            assert T.rel_err(got[t, h], o[t, h]) <= tol, (Tb, b, kvh, t, h)
                orc.tree_update(tr, Kb, T.np64(inp.refs[kvh]), N0 + Tb)
        n_done += Tb
    assert flipped_total <= max(2, rows_total // 8), (flipped_total, rows_total)
    # the tree extended block by block equals a fresh build of the final cache
    fresh = zha.Buffers(cfg)
    zha.tree_build(cfg, fresh.tree, dev.K, dev.refs, dev.lens, fresh.status)
    torch.cuda.synchronize()
    for level in range(1, w.levels + 1):
        for b in range(w.batch):
            k = orc.level_nodes(lens0[b] + n_done, w.chunk, level)
            assert torch.equal(buf.tree_level(level)[0][b, :, :k], fresh.tree_level(level)[0][b, :, :k])
            assert torch.equal(buf.tree_level(level)[1][b, :, :k], fresh.tree_level(level)[1][b, :, :k])


def test_decode_block_single_query_equals_decode(zha):
    """T = 1 with no chunk completed by the token: the same output as zha_decode."""
    w = BASE[1]
    cap = w.context + 16
    inp = make_inputs(w, capacity=cap)
    dev_a, dev_b = T.to_device(inp), T.to_device(inp)
    cfg = zha.config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.levels, w.n_refs, w.dtype,
                     cap, queries=4)
    assert (w.context + 1) % w.chunk != 0
    ba, bb = zha.Buffers(cfg), zha.Buffers(cfg)
    zha.tree_build(cfg, ba.tree, dev_a.K, dev_a.refs, dev_a.lens, ba.status)
    zha.tree_build(cfg, bb.tree, dev_b.K, dev_b.refs, dev_b.lens, bb.status)
    g = torch.Generator().manual_seed(8)
    k_new = torch.randn((w.batch, 1, w.n_kv_heads, w.head_dim), generator=g).to(torch.bfloat16).cuda()
    v_new = torch.randn((w.batch, 1, w.n_kv_heads, w.head_dim), generator=g).to(torch.bfloat16).cuda()
    q = torch.randn((w.batch, 1, w.n_q_heads, w.head_dim), generator=g).to(torch.bfloat16).cuda()
    out_a = torch.zeros_like(q)
    out_b = torch.zeros_like(q[:, 0])
    zha.decode_block(cfg, 1, ba.tree, dev_a.K, dev_a.V, dev_a.refs, dev_a.lens, q, k_new, v_new, w.p, ba.sel,
                     out_a, ba.workspace, ba.status)
    zha.decode(cfg, bb.tree, dev_b.K, dev_b.V, dev_b.refs, dev_b.lens, q[:, 0].contiguous(),
               k_new[:, 0].contiguous(), v_new[:, 0].contiguous(), w.p, bb.sel, out_b, bb.workspace, bb.status)
    torch.cuda.synchronize()
    ba.check_status()
    bb.check_status()
    assert torch.equal(dev_a.lens, dev_b.lens)
    assert torch.equal(ba.sel["count"], bb.sel["count"])
    assert torch.equal(out_a[:, 0], out_b)


def test_decode_block_rejects_bad_sizes(zha):
    w = BASE[1]
    cfg = zha.config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.levels, w.n_refs, w.dtype,
                     w.context + 16, queries=2)
    buf = zha.Buffers(cfg)
    z = torch.zeros((w.batch, 3, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    lens = torch.full((w.batch,), w.context, dtype=torch.int32, device="cuda")
    with pytest.raises(zha.ZhaError):   # T above cfg.queries
        zha.decode_block(cfg, 3, buf.tree, z, z, z, lens, z, z, z, 0.9, buf.sel, z, buf.workspace, buf.status)
    with pytest.raises(zha.ZhaError):   # T * G above 32
        zha.config(1, 16, 1, 64, 4, 3, 16, "bf16", 4096, queries=3)
