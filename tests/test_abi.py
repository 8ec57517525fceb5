"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/zha.h declares, and its layout queries agree with the
rules they document (and with the oracle's level sizes)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "zha.h")).read()
    return sorted(set(re.findall(r"^ZHA_API\s+[\w\s\*]+?\b(zha_\w+)\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def zha():
    from tree_indexed_sparse_02_b200 import build
    build.build()
    from tree_indexed_sparse_02_b200 import zha as z
    return z


def test_header_declares_the_hot_path(zha):
    names = declared_functions()
    for required in ("zha_tree_build", "zha_tree_append", "zha_route", "zha_sparse_attn", "zha_decode",
                     "zha_dense_decode", "zha_topp_select"):
        assert required in names


def test_library_exports_every_declared_symbol(zha):
    lib = ctypes.CDLL(zha.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_config_checks(zha):
    zha.config(1, 2, 1, 64, 4, 3, 16, "f32", 4096)
    bad = [dict(head_dim=96), dict(chunk=3), dict(chunk=512), dict(levels=9), dict(n_refs=33),
           dict(n_q_heads=34, n_kv_heads=2), dict(n_q_heads=3, n_kv_heads=2)]
    for kw in bad:
        args = dict(batch=1, n_q_heads=2, n_kv_heads=1, head_dim=64, chunk=4, levels=3, n_refs=16,
                    dtype="f32", max_len=4096)
        args.update(kw)
        with pytest.raises(zha.ZhaError):
            zha.config(**args)


def test_level_sizes_match_oracle(zha, orc):
    cfg = zha.config(1, 8, 1, 128, 4, 6, 16, "bf16", 1 << 20)
    for n in (0, 1, 3, 4, 5, 4095, 4096, 4097, 262144, 262147, 1 << 20):
        for level in range(1, 7):
            assert zha.level_nodes(cfg, n, level) == orc.level_nodes(n, 4, level)


def test_tree_and_workspace_layout(zha):
    cfg = zha.config(4, 32, 4, 128, 4, 6, 16, "bf16", 262144 + 512)
    total = zha.tree_bytes(cfg)
    prev_end = 0
    for level in range(1, 7):
        mu_off, b_off = zha.tree_level_offsets(cfg, level)
        cap = zha.level_nodes(cfg, cfg.max_len, level)
        assert mu_off % 256 == 0 and b_off % 256 == 0
        assert mu_off >= prev_end
        assert b_off >= mu_off + 4 * 4 * cap * 16 * 128 * 2
        prev_end = b_off + 4 * 4 * cap * 16 * 4
    assert total >= prev_end
    ws = zha.workspace_bytes(cfg)
    for level in range(1, 7):
        v = zha.workspace_level_view(cfg, level)
        assert v.cap == (zha.level_nodes(cfg, cfg.max_len, level) + cfg.chunk + 7) // 8 * 8
        for off in (v.cand_idx, v.cand_mask, v.scores, v.kept_mask, v.count):
            assert off % 256 == 0 and off < ws


def test_invalid_arguments_are_rejected_before_launch(zha):
    """Argument errors come back synchronously; these calls launch nothing."""
    cfg = zha.config(1, 2, 1, 64, 4, 3, 16, "f32", 4096)
    L = zha.lib()
    assert L.zha_tree_build(ctypes.byref(cfg), None, None, None, None, None, None) == 1
    p = (ctypes.c_float * 3)(0.9, 0.0, 0.9)       # p <= 0 at one level
    sel = zha.Selection(16, 16, 16, None)
    assert L.zha_route(ctypes.byref(cfg), ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), p,
                       ctypes.byref(sel), ctypes.c_void_p(16), None, None) == 1
    p = (ctypes.c_float * 3)(0.9, float("nan"), 0.9)
    assert L.zha_route(ctypes.byref(cfg), ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), p,
                       ctypes.byref(sel), ctypes.c_void_p(16), None, None) == 1
    assert L.zha_topp_select(None, None, 1, 8, ctypes.c_float(0.5), None, None, None) == 1
    assert L.zha_topp_select(None, None, 0, 8, ctypes.c_float(0.5), None, None, None) == 0
    # misaligned pointer
    assert L.zha_dense_decode(ctypes.byref(cfg), ctypes.c_void_p(18), ctypes.c_void_p(16), ctypes.c_void_p(16),
                              ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), None, None) == 1
    assert L.zha_status_string(3).decode().startswith("capacity")
    # the bounded-wait expiry check: unknown kind, limit out of range, no status
    assert L.zha_wait_expiry_check(7, 1000, ctypes.c_void_p(16), None) == 1
    assert L.zha_wait_expiry_check(zha.ZHA_WAIT_MBARRIER, 0, ctypes.c_void_p(16), None) == 1
    assert L.zha_wait_expiry_check(zha.ZHA_WAIT_MBARRIER, (1 << 31) + 1, ctypes.c_void_p(16), None) == 1
    assert L.zha_wait_expiry_check(zha.ZHA_WAIT_ROW_BARRIER, 1000, None, None) == 1


def test_p_schedule_host_rule(zha, orc):
    """zha_p_schedule is host-only: fixed = p everywhere; depth-root = the
    oracle's p^(1/L) rounded once to fp32; invalid arguments are refused."""
    import numpy as np
    for p in (0.5, 0.75, 0.95, 0.999):
        for L in (1, 3, 6, 8):
            assert zha.p_schedule(p, L, "fixed") == [float(np.float32(p))] * L
            want = [float(np.float32(v)) for v in orc.depth_root_schedule(float(np.float32(p)), L)]
            assert zha.p_schedule(p, L, "root") == want
    assert zha.p_schedule(1.5, 4, "root") == [1.0] * 4
    out = (ctypes.c_float * 8)()
    L = zha.lib()
    for args in ((0.0, 3, 1), (float("nan"), 3, 1), (0.9, 0, 1), (0.9, 9, 1), (0.9, 3, 7)):
        assert L.zha_p_schedule(ctypes.c_float(args[0]), args[1], args[2], out) == 1
    assert L.zha_p_schedule(ctypes.c_float(0.9), 3, 1, None) == 1


def test_mx_summary_config_and_layout(zha):
    """MX-FP8 summaries need bf16 KV; their records take R*d + R*d/32 + 4R bytes
    (2,176 at R=16, d=128) instead of R*2d + 4R (4,160), plus 4R bytes of each
    plane's value at its own reference in both formats, and the block scales
    have their own offset, which the native format refuses."""
    with pytest.raises(zha.ZhaError):
        zha.config(1, 2, 1, 64, 4, 3, 16, "f32", 4096, summary="mxfp8")
    with pytest.raises(zha.ZhaError):
        zha.config(1, 2, 1, 64, 4, 3, 16, "bf16", 4096, summary=7)
    mx = zha.config(1, 8, 1, 128, 4, 1, 16, "bf16", 4096, summary="mxfp8")
    nat = zha.config(1, 8, 1, 128, 4, 1, 16, "bf16", 4096)
    n1 = zha.level_nodes(mx, 4096, 1)
    mu_off, b_off = zha.tree_level_offsets(mx, 1)
    off = ctypes.c_size_t()
    assert zha.lib().zha_tree_level_scales(ctypes.byref(mx), 1, ctypes.byref(off)) == 0
    assert mu_off == 0 and off.value >= n1 * 16 * 128 and b_off >= off.value + n1 * 16 * 4
    assert zha.tree_bytes(mx) == pytest.approx(n1 * (2176 + 64), rel=0.01)
    assert zha.tree_bytes(nat) == pytest.approx(n1 * (4160 + 64), rel=0.01)
    assert zha.lib().zha_tree_level_scales(ctypes.byref(nat), 1, ctypes.byref(off)) == 1


def test_route_fused_query(zha):
    """The fused launch runs only with its flag on a bf16 tree with native
    summaries, 16 planes, at most 8 query rows per group, single queries and
    a top level of at most 1,024 nodes at max_len; everything else routes per
    level."""
    F = zha.ZHA_FLAG_FUSED_ROUTE
    base = dict(batch=1, n_q_heads=32, n_kv_heads=4, head_dim=128, chunk=4, levels=6, n_refs=16, dtype="bf16",
                max_len=(1 << 18) + 64, flags=F)

    def fused(T=1, **kw):
        args = dict(base)
        args.update(kw)
        return zha.route_fused(zha.config(**args), T)

    assert fused()                                   # 256K deep: 64 top-level nodes
    assert fused(head_dim=64)
    assert fused(n_q_heads=16)                       # 4 rows per group
    assert not fused(flags=0)
    assert not fused(dtype="f32")
    assert not fused(summary="mxfp8")
    assert not fused(n_refs=8)
    assert not fused(n_q_heads=64)                   # 16 rows per group
    assert not fused(T=2)
    # top level at max_len: 1,024 nodes fused, one more per level below is not
    assert fused(max_len=4 * 1024 * 4 ** 5)
    assert not fused(max_len=4 * 1024 * 4 ** 5 + 4 ** 6 * 4)
    assert not fused(max_len=4 * 1024 * 4 ** 5 + 4 ** 6)
    # a one-level tree of 256-token chunks outgrows 1,024 nodes past 256K tokens
    assert fused(chunk=256, levels=1, max_len=1 << 18)
    assert not fused(chunk=256, levels=1, max_len=(1 << 18) + 256)
    cfg = zha.config(**base)
    with pytest.raises(zha.ZhaError):
        zha.route_fused(cfg, 0)
    assert zha.lib().zha_route_fused(ctypes.byref(cfg), 1, None) == 1
