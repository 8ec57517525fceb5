"""Failure detection on the GPU without a fault: every wait inside the
library's kernels is bounded. zha_wait_expiry_check runs those waits (the
counter barrier of the selection spread over several CTAs per row, with one
CTA that never arrives; an mbarrier wait that nothing completes) with a short
limit: the call must come back, with ZHA_ERR_TIMEOUT in the device status,
and the context must stay usable -- the next route and attention on the same
stream are checked against the oracle."""
import time

import pytest
import torch

import zha_testlib as T
from tree_indexed_sparse_02_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

W = Workload("expiry then route B=1 N=3001 c=4 L=4", 1, 16, 2, 128, 3001, 4, 4, 16, 0.95, 16, "bf16", 61)


@pytest.fixture(scope="module")
def zha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_indexed_sparse_02_b200 import zha as z
    return z


@pytest.mark.parametrize("kind", ["ZHA_WAIT_ROW_BARRIER", "ZHA_WAIT_MBARRIER"])
def test_wait_runs_out_and_the_next_call_is_correct(zha, kind):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    zha.wait_expiry_check(getattr(zha, kind), 2_000_000, status)   # about a millisecond of SM cycles
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 10.0
    assert int(status.item()) == 5, zha.STATUS_NAMES.get(int(status.item()))   # ZHA_ERR_TIMEOUT
    # the context is usable: a full route and attention, against the oracle
    inp = make_inputs(W, capacity=W.context + 64)
    dev = T.to_device(inp)
    cfg = T.make_cfg(zha, W, W.context + 64)
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, dev.K, dev.refs, dev.lens, buf.status)
    zha.route(cfg, buf.tree, dev.q, dev.lens, W.p, buf.sel, buf.workspace, buf.status)
    out = torch.zeros_like(dev.q)
    zha.sparse_attn(cfg, dev.q, dev.K, dev.V, dev.lens, buf.sel, out, buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status()
    for kvh in range(W.n_kv_heads):
        T.check_group_vs_oracle(W, inp, buf, 0, kvh, [W.p] * W.levels, out=out)


def test_a_longer_limit_still_returns(zha):
    """About 0.1 s of SM cycles: the wait gives up on its own clock, not at once."""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    zha.wait_expiry_check(zha.ZHA_WAIT_ROW_BARRIER, 200_000_000, status)
    end.record()
    torch.cuda.synchronize()
    assert int(status.item()) == 5
    ms = start.elapsed_time(end)
    assert 20.0 < ms < 2000.0, ms   # 2e8 cycles at 0.1-2 GHz
