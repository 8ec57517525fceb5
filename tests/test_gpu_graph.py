"""Decode steps replayed from one captured CUDA graph give bit-identical
outputs, selections and trees to ordinary zha_decode calls."""
import pytest
import torch

import zha_testlib as T
from tree_indexed_sparse_02_b200.inputs import decode_stream, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("idx", [0, 1, 3], ids=["tiny-f32", "deep-bf16", "r1-c8"])
def test_graph_replay_equals_direct_calls(idx):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_indexed_sparse_02_b200 import zha
    w = T.small_workloads()[idx]
    steps = 7
    cap = w.context + steps + 8
    k_new, v_new, qs = decode_stream(w, steps)
    runs = []
    for use_graph in (False, True):
        inp = T.to_device(make_inputs(w, capacity=cap))
        cfg = T.make_cfg(zha, w, cap)
        buf = zha.Buffers(cfg)
        zha.tree_build(cfg, buf.tree, inp.K, inp.refs, inp.lens, buf.status)
        graph = zha.DecodeGraph(cfg, buf, inp.K, inp.V, inp.refs, inp.lens, w.p) if use_graph else None
        outs = []
        for i in range(steps):
            if graph is not None:
                outs.append(graph.step(qs[i].cuda(), k_new[i].cuda(), v_new[i].cuda()).clone())
            else:
                out = torch.zeros_like(inp.q)
                zha.decode(cfg, buf.tree, inp.K, inp.V, inp.refs, inp.lens, qs[i].cuda(), k_new[i].cuda(),
                           v_new[i].cuda(), w.p, buf.sel, out, buf.workspace, buf.status)
                outs.append(out)
        torch.cuda.synchronize()
        buf.check_status()
        assert torch.all(inp.lens == w.context + steps)
        runs.append((outs, buf, inp))
        if graph is not None:
            assert graph.kernels_per_step > 0
    (o0, b0, i0), (o1, b1, i1) = runs
    for a, b in zip(o0, o1):
        assert torch.equal(a, b)
    assert torch.equal(b0.sel["count"], b1.sel["count"])
    N = w.context + steps
    for level in range(1, w.levels + 1):       # every live node of the tree
        k = zha.level_nodes(b0.cfg, N, level)
        assert torch.equal(b0.tree_level(level)[0][:, :, :k], b1.tree_level(level)[0][:, :, :k])
        assert torch.equal(b0.tree_level(level)[1][:, :, :k], b1.tree_level(level)[1][:, :, :k])
    assert torch.equal(i0.K, i1.K) and torch.equal(i0.V, i1.V)
