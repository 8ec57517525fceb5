"""zha_dense_decode_noalloc: dense decode for callers that cannot allocate
device memory (a host framework that owns every allocation, or a loop that
must not pay for cudaMalloc). It keeps its split-K scratch in a fixed array
inside the library. Checked through the C ABI against zha_dense_decode, on
two calls in a row (the second call reuses the scratch the first one left),
and against the oracle's exact attention after a larger call, with shorter
caches and other split counts (splits with no tokens)."""
import ctypes

import numpy as np
import pytest
import torch

import zha_oracle as orc
import zha_testlib as T
from tree_indexed_sparse_02_b200.inputs import TINY_F32, Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zha():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from tree_indexed_sparse_02_b200 import zha as z
    fn = z.lib().zha_dense_decode_noalloc
    P = ctypes.c_void_p
    fn.argtypes = [ctypes.POINTER(z.Config), P, P, P, P, P, P, P]
    fn.restype = ctypes.c_int32
    return z


def _noalloc(zha, cfg, q, K, V, lens, out, status):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return zha.lib().zha_dense_decode_noalloc(ctypes.byref(cfg), q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                              lens.data_ptr(), out.data_ptr(), status.data_ptr(), stream)


@pytest.mark.parametrize("w", [TINY_F32, Workload("noalloc bf16 B=2", 2, 16, 2, 128, 5000, 4, 3, 16, 0.9, 8,
                                                  "bf16", 31)], ids=["f32", "bf16"])
def test_noalloc_matches_dense_decode_twice(zha, w):
    cap = w.context + 16
    inp = make_inputs(w, capacity=cap)
    dev = T.to_device(inp)
    cfg = T.make_cfg(zha, w, cap)
    buf = zha.Buffers(cfg)
    ref = torch.zeros_like(dev.q)
    zha.dense_decode(cfg, dev.q, dev.K, dev.V, dev.lens, ref, buf.workspace, buf.status)
    q2 = torch.flip(dev.q, dims=[1]).contiguous()        # a different query for the second call
    ref2 = torch.zeros_like(dev.q)
    zha.dense_decode(cfg, q2, dev.K, dev.V, dev.lens, ref2, buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status()
    for q, want in ((dev.q, ref), (q2, ref2)):
        out = torch.full_like(dev.q, float("nan"))
        assert _noalloc(zha, cfg, q, dev.K, dev.V, dev.lens, out, buf.status) == 0
        torch.cuda.synchronize()
        buf.check_status()
        assert T.rel_err(T.np64(out), T.np64(want)) <= T.TOL[w.dtype]


def test_noalloc_rejects_configs_beyond_its_scratch(zha):
    # 16 groups x 4096 splits x 8 heads x 130 floats is far more than the fixed scratch
    cfg = zha.config(4, 32, 4, 128, 4, 3, 16, "bf16", 1 << 20, attn_splits=4096)
    z = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    lens = torch.zeros(4, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _noalloc(zha, cfg, z, z, z, lens, z, status) == 3   # ZHA_ERR_CAPACITY, nothing launched


def test_noalloc_after_a_larger_call_matches_the_oracle(zha):
    """A call over long caches fills many partials; the next calls, over
    shorter ragged caches and with other split counts, leave some splits
    without tokens (they write an empty partial). Every output is checked
    against the oracle's exact softmax attention."""
    w = Workload("noalloc ragged B=3", 3, 16, 2, 128, 6000, 4, 3, 16, 0.9, 8, "bf16", 37)
    cap = w.context + 16
    inp = make_inputs(w, capacity=cap)
    dev = T.to_device(inp)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    big = zha.config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.levels, w.n_refs, w.dtype, cap,
                     attn_splits=32)
    out = torch.zeros_like(dev.q)
    assert _noalloc(zha, big, dev.q, dev.K, dev.V, dev.lens, out, status) == 0
    s = T.scale_of(w)
    G = w.group
    for splits, lens in ((32, [700, 1, 0]), (7, [5999, 33, 2]), (64, [64, 3, 4096])):
        cfg = zha.config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.levels, w.n_refs, w.dtype,
                         cap, attn_splits=splits)
        dlens = torch.tensor(lens, dtype=torch.int32, device="cuda")
        out = torch.full_like(dev.q, float("nan"))
        assert _noalloc(zha, cfg, dev.q, dev.K, dev.V, dlens, out, status) == 0
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for b in range(w.batch):
            N = lens[b]
            for kvh in range(w.n_kv_heads):
                got = T.np64(out[b, kvh * G:(kvh + 1) * G])
                if N == 0:
                    assert np.all(got == 0.0), (splits, b)   # no token: a zero output
                    continue
                K = T.np64(inp.K[b, kvh, :N])
                V = T.np64(inp.V[b, kvh, :N])
                q = T.np64(inp.q[b, kvh * G:(kvh + 1) * G])
                ref = np.stack([orc.attend(q[h], K, V, N, s) for h in range(G)])
                assert T.rel_err(got, ref) <= T.TOL[w.dtype], (splits, b, kvh)
