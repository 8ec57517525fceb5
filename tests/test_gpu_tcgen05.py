"""The tcgen05 (tensor-memory) scoring kernel: routing with it against the
fp64 oracle on the same inputs (level by level, the selection and the
attention outputs), and, as an extra check, against the mma.sync scorer (same
tree, same queries, scores within fp32 summation-order rounding, the same
routing except at exact-score boundary ties)."""
import numpy as np
import pytest
import torch

import zha_testlib as T
from tree_indexed_sparse_02_b200.inputs import DEEP_256K, Workload, make_inputs

pytestmark = pytest.mark.gpu

CASES = [Workload("deep bf16 B=2 c=4 L=4", 2, 16, 2, 128, 3001, 4, 4, 16, 0.95, 16, "bf16", 11),
         Workload("deep bf16 B=1 G=16 c=4 L=5", 1, 32, 2, 128, 20000, 4, 5, 16, 0.9, 32, "bf16", 41),
         Workload("wide bf16 c=256 L=1", 1, 32, 4, 128, 32768, 256, 1, 16, 0.95, 64, "bf16", 1),
         Workload("deep bf16 aligned", 1, 32, 4, 128, 65536, 4, 6, 16, 0.95, 64, "bf16", 5, refs_mode="aligned"),
         Workload("c=2 L=8", 1, 16, 2, 128, 3001, 2, 8, 16, 0.9, 8, "bf16", 6),
         Workload("c=8 L=3", 2, 16, 2, 128, 2999, 8, 3, 16, 0.9, 8, "bf16", 7),
         Workload("c=16 L=2", 1, 16, 1, 128, 5000, 16, 2, 16, 0.9, 8, "bf16", 8)]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_tcgen05_scores_match_mma_sync(w):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_indexed_sparse_02_b200 import zha
    cap = w.context + 64
    inp = T.to_device(make_inputs(w, capacity=cap))
    runs = []
    for flags in (zha.ZHA_FLAG_TCGEN05, 0):
        cfg = T.make_cfg(zha, w, cap, flags=flags)
        buf = zha.Buffers(cfg)
        zha.tree_build(cfg, buf.tree, inp.K, inp.refs, inp.lens, buf.status)
        zha.route(cfg, buf.tree, inp.q, inp.lens, w.p, buf.sel, buf.workspace, buf.status)
        torch.cuda.synchronize()
        buf.check_status()
        runs.append(buf)
    tc, ref = runs
    for level in range(w.levels, 0, -1):
        a, b = tc.level_state(level), ref.level_state(level)
        for bb in range(w.batch):
            for kvh in range(w.n_kv_heads):
                n = int(b["count"][bb, kvh])
                assert int(a["count"][bb, kvh]) == n
                same = (a["cand_idx"][bb, kvh, :n] == b["cand_idx"][bb, kvh, :n]).cpu().numpy()
                if level == w.levels:
                    assert same.all()
                real = same & (b["cand_mask"][bb, kvh, :n] != 0).cpu().numpy()
                sa = a["scores"][bb, kvh, :, :n].cpu().numpy()[:, real]
                sb = b["scores"][bb, kvh, :, :n].cpu().numpy()[:, real]
                assert np.allclose(sa, sb, rtol=1e-5, atol=1e-5), (level, bb, kvh, np.abs(sa - sb).max())
    # the final selections agree (a boundary tie could flip one leaf; none expected here)
    assert torch.equal(tc.sel["count"], ref.sel["count"])


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_tcgen05_route_matches_oracle(w):
    """ZHA_FLAG_TCGEN05 routing and attention of every group against the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_indexed_sparse_02_b200 import zha
    cap = w.context + 64
    inp = make_inputs(w, capacity=cap)
    dev = T.to_device(inp)
    cfg = T.make_cfg(zha, w, cap, flags=zha.ZHA_FLAG_TCGEN05)
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, dev.K, dev.refs, dev.lens, buf.status)
    zha.route(cfg, buf.tree, dev.q, dev.lens, w.p, buf.sel, buf.workspace, buf.status)
    out = torch.zeros_like(dev.q)
    zha.sparse_attn(cfg, dev.q, dev.K, dev.V, dev.lens, buf.sel, out, buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status()
    flipped = 0
    for b in range(w.batch):
        for kvh in range(w.n_kv_heads):
            flipped += len(T.check_group_vs_oracle(w, inp, buf, b, kvh, [w.p] * w.levels, out=out))
    assert flipped <= max(2, w.batch * w.n_q_heads // 8), flipped
