"""Thin Python binding of libzha's C ABI (``include/zha.h``).

Argument marshalling only: every function forwards device pointers of torch
tensors and a CUDA stream to the library, and raises ``ZhaError`` on a
non-zero status. Nothing here computes any step of the method; if libzha.so
is missing the import fails loudly (there is no fallback path).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzha.so")

ZHA_BF16, ZHA_F32 = 0, 1
ZHA_FLAG_TAIL_ONLY = 1
ZHA_FLAG_TCGEN05 = 2
ZHA_FLAG_FUSED_ROUTE = 4
ZHA_P_FIXED, ZHA_P_DEPTH_ROOT = 0, 1
ZHA_WAIT_ROW_BARRIER, ZHA_WAIT_MBARRIER = 0, 1
ZHA_SUMMARY_NATIVE, ZHA_SUMMARY_MXFP8 = 0, 1
ZHA_MAX_LEVELS = 8
STATUS_NAMES = {0: "ZHA_OK", 1: "ZHA_ERR_INVALID_ARG", 2: "ZHA_ERR_UNSUPPORTED",
                3: "ZHA_ERR_CAPACITY", 4: "ZHA_ERR_CUDA", 5: "ZHA_ERR_TIMEOUT"}


class ZhaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({_lib.zha_status_string(code).decode()})")


class Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("chunk", ctypes.c_int32), ("levels", ctypes.c_int32),
                ("n_refs", ctypes.c_int32), ("dtype", ctypes.c_int32), ("max_len", ctypes.c_int64),
                ("scale", ctypes.c_float), ("flags", ctypes.c_int32), ("attn_splits", ctypes.c_int32),
                ("summary", ctypes.c_int32), ("queries", ctypes.c_int32), ("reserved", ctypes.c_int32)]

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == ZHA_BF16 else torch.float32


class Selection(ctypes.Structure):
    _fields_ = [("leaf_idx", ctypes.c_void_p), ("head_mask", ctypes.c_void_p), ("count", ctypes.c_void_p),
                ("level_kept", ctypes.c_void_p)]


class LevelView(ctypes.Structure):
    _fields_ = [("cap", ctypes.c_int64), ("cand_idx", ctypes.c_size_t), ("cand_mask", ctypes.c_size_t),
                ("scores", ctypes.c_size_t), ("kept_mask", ctypes.c_size_t), ("count", ctypes.c_size_t)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libzha.so not built at {LIB_PATH}; run tree_indexed_sparse_02_b200/build.py")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    CP = ctypes.POINTER(Config)
    SP = ctypes.POINTER(Selection)
    sig = {
        "zha_status_string": ([i32], ctypes.c_char_p),
        "zha_check_config": ([CP], i32),
        "zha_level_nodes": ([CP, i64, i32], i64),
        "zha_route_fused": ([CP, i32, ctypes.POINTER(i32)], i32),
        "zha_tree_bytes": ([CP], sz),
        "zha_tree_level_offsets": ([CP, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)], i32),
        "zha_tree_level_scales": ([CP, i32, ctypes.POINTER(sz)], i32),
        "zha_tree_level_logmass": ([CP, i32, ctypes.POINTER(sz)], i32),
        "zha_workspace_bytes": ([CP], sz),
        "zha_workspace_level_view": ([CP, i32, ctypes.POINTER(LevelView)], i32),
        "zha_workspace_level_view_block": ([CP, i32, i32, ctypes.POINTER(LevelView)], i32),
        "zha_tree_build": ([CP, P, P, P, P, P, P], i32),
        "zha_tree_append": ([CP, P, P, P, P, i32, P, P], i32),
        "zha_route": ([CP, P, P, P, P, SP, P, P, P], i32),
        "zha_sparse_attn": ([CP, P, P, P, P, SP, P, P, P, P], i32),
        "zha_decode": ([CP, P, P, P, P, P, P, P, P, P, SP, P, P, P, P], i32),
        "zha_decode_block": ([CP, i32, P, P, P, P, P, P, P, P, P, SP, P, P, P, P], i32),
        "zha_dense_decode": ([CP, P, P, P, P, P, P, P, P], i32),
        "zha_topp_select": ([P, P, i32, i64, f32, P, P, P], i32),
        "zha_p_schedule": ([f32, i32, i32, ctypes.POINTER(f32)], i32),
        "zha_wait_expiry_check": ([i32, i64, P, P], i32),
        "zha_launch_count": ([], ctypes.c_uint64),
        "zha_profile_enable": ([i32], i32),
        "zha_profile_read": ([ctypes.c_char_p, i32, ctypes.POINTER(ctypes.c_double),
                              ctypes.POINTER(ctypes.c_int64), i32], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


_lib = _load()


def lib():
    return _lib


def config(batch, n_q_heads, n_kv_heads, head_dim, chunk, levels, n_refs, dtype="bf16", max_len=4096,
           scale=0.0, flags=0, attn_splits=0, summary="native", queries=0) -> Config:
    dt = {"bf16": ZHA_BF16, "f32": ZHA_F32}.get(dtype, dtype)
    sm = {"native": ZHA_SUMMARY_NATIVE, "mxfp8": ZHA_SUMMARY_MXFP8}.get(summary, summary)
    c = Config(batch, n_q_heads, n_kv_heads, head_dim, chunk, levels, n_refs, dt, max_len, scale, flags,
               attn_splits, sm, queries)
    check(_lib.zha_check_config(ctypes.byref(c)), "zha_check_config")
    return c


def check(code: int, where: str):
    if code != 0:
        raise ZhaError(code, where)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def level_nodes(cfg: Config, n_tokens: int, level: int) -> int:
    return int(_lib.zha_level_nodes(ctypes.byref(cfg), int(n_tokens), int(level)))


def route_fused(cfg: Config, T: int = 1) -> bool:
    """True if routing with cfg (T query positions) runs the fused launch."""
    out = ctypes.c_int32(0)
    check(_lib.zha_route_fused(ctypes.byref(cfg), int(T), ctypes.byref(out)), "zha_route_fused")
    return bool(out.value)


def tree_bytes(cfg: Config) -> int:
    return int(_lib.zha_tree_bytes(ctypes.byref(cfg)))


def workspace_bytes(cfg: Config) -> int:
    return int(_lib.zha_workspace_bytes(ctypes.byref(cfg)))


def tree_level_offsets(cfg: Config, level: int):
    mu, b = ctypes.c_size_t(), ctypes.c_size_t()
    check(_lib.zha_tree_level_offsets(ctypes.byref(cfg), level, ctypes.byref(mu), ctypes.byref(b)),
          "zha_tree_level_offsets")
    return mu.value, b.value


def workspace_level_view(cfg: Config, level: int, T: int = 1) -> LevelView:
    v = LevelView()
    check(_lib.zha_workspace_level_view_block(ctypes.byref(cfg), int(T), level, ctypes.byref(v)),
          "zha_workspace_level_view_block")
    return v


def _plevels(cfg: Config, p):
    if isinstance(p, (int, float)):
        p = [float(p)] * cfg.levels
    arr = (ctypes.c_float * cfg.levels)(*[float(x) for x in p])
    return arr


def p_schedule(p: float, levels: int, schedule=ZHA_P_FIXED) -> list[float]:
    """Per-level fractions (index l-1 is level l) from libzha's schedule rule."""
    schedule = {"fixed": ZHA_P_FIXED, "root": ZHA_P_DEPTH_ROOT}.get(schedule, schedule)
    out = (ctypes.c_float * max(int(levels), 1))()
    check(_lib.zha_p_schedule(float(p), int(levels), int(schedule), out), "zha_p_schedule")
    return [float(x) for x in out[:levels]]


def _sel(sel) -> Selection:
    return Selection(sel["leaf_idx"].data_ptr(), sel["head_mask"].data_ptr(), sel["count"].data_ptr(),
                     None if sel.get("level_kept") is None else sel["level_kept"].data_ptr())


def tree_build(cfg, tree, K, refs, lens, dev_status=None, stream=None):
    check(_lib.zha_tree_build(ctypes.byref(cfg), _p(tree), _p(K), _p(refs), _p(lens), _p(dev_status),
                              _stream(stream)), "zha_tree_build")


def tree_append(cfg, tree, K, refs, lens, n_new, dev_status=None, stream=None):
    check(_lib.zha_tree_append(ctypes.byref(cfg), _p(tree), _p(K), _p(refs), _p(lens), int(n_new),
                               _p(dev_status), _stream(stream)), "zha_tree_append")


def route(cfg, tree, q, lens, p, sel, workspace, dev_status=None, stream=None):
    s = _sel(sel)
    check(_lib.zha_route(ctypes.byref(cfg), _p(tree), _p(q), _p(lens), _plevels(cfg, p), ctypes.byref(s),
                         _p(workspace), _p(dev_status), _stream(stream)), "zha_route")


def sparse_attn(cfg, q, K, V, lens, sel, out, workspace, dev_status=None, stream=None):
    s = _sel(sel)
    check(_lib.zha_sparse_attn(ctypes.byref(cfg), _p(q), _p(K), _p(V), _p(lens), ctypes.byref(s), _p(out),
                               _p(workspace), _p(dev_status), _stream(stream)), "zha_sparse_attn")


def decode(cfg, tree, K, V, refs, lens, q, k_new, v_new, p, sel, out, workspace, dev_status=None,
           stream=None):
    s = _sel(sel)
    check(_lib.zha_decode(ctypes.byref(cfg), _p(tree), _p(K), _p(V), _p(refs), _p(lens), _p(q), _p(k_new),
                          _p(v_new), _plevels(cfg, p), ctypes.byref(s), _p(out), _p(workspace),
                          _p(dev_status), _stream(stream)), "zha_decode")


def decode_block(cfg, T, tree, K, V, refs, lens, q, k_new, v_new, p, sel, out, workspace, dev_status=None,
                 stream=None):
    """T query positions per sequence: q, out [B, T, Hq, d]; k_new, v_new [B, T, Hkv, d]."""
    s = _sel(sel)
    check(_lib.zha_decode_block(ctypes.byref(cfg), int(T), _p(tree), _p(K), _p(V), _p(refs), _p(lens), _p(q),
                                _p(k_new), _p(v_new), _plevels(cfg, p), ctypes.byref(s), _p(out),
                                _p(workspace), _p(dev_status), _stream(stream)), "zha_decode_block")


def dense_decode(cfg, q, K, V, lens, out, workspace, dev_status=None, stream=None):
    check(_lib.zha_dense_decode(ctypes.byref(cfg), _p(q), _p(K), _p(V), _p(lens), _p(out), _p(workspace),
                                _p(dev_status), _stream(stream)), "zha_dense_decode")


def topp_select(scores, counts, p, kept, dev_status=None, stream=None):
    n_sets, stride = scores.shape
    check(_lib.zha_topp_select(_p(scores), _p(counts), int(n_sets), int(stride), float(p), _p(kept),
                               _p(dev_status), _stream(stream)), "zha_topp_select")


def wait_expiry_check(kind: int, limit_cycles: int, dev_status, stream=None):
    """Run one of the library's bounded device waits on a condition nothing
    satisfies (ZHA_WAIT_ROW_BARRIER or ZHA_WAIT_MBARRIER), giving up after
    limit_cycles SM cycles with ZHA_ERR_TIMEOUT in dev_status."""
    check(_lib.zha_wait_expiry_check(int(kind), int(limit_cycles), _p(dev_status), _stream(stream)),
          "zha_wait_expiry_check")


def launch_count() -> int:
    """Kernels libzha has launched since it was loaded."""
    return int(_lib.zha_launch_count())


def profile_enable(on: bool = True):
    check(_lib.zha_profile_enable(1 if on else 0), "zha_profile_enable")


def profile_read(max_kernels: int = 64) -> dict:
    """{kernel name: (total ms, launches)} of the launches recorded since the last read."""
    names = ctypes.create_string_buffer(8192)
    ms = (ctypes.c_double * max_kernels)()
    ln = (ctypes.c_int64 * max_kernels)()
    n = _lib.zha_profile_read(names, 8192, ms, ln, max_kernels)
    if n < 0:
        raise ZhaError(4, "zha_profile_read")
    keys = names.value.decode().split("\n")[:n]
    return {k: (ms[i], ln[i]) for i, k in enumerate(keys)}


class DecodeGraph:
    """zha_decode captured once into a CUDA graph and replayed per step.

    Every pointer, grid size and p is fixed at capture; the cache lengths live
    on the device, so one graph serves every later step. Inputs are copied into
    the graph's own q / k_new / v_new buffers before each replay."""

    def __init__(self, cfg, buf, K, V, refs, lens, p):
        B, Hq, Hkv, d = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
        dt = cfg.torch_dtype
        dev = K.device
        self.q = torch.zeros((B, Hq, d), dtype=dt, device=dev)
        self.k_new = torch.zeros((B, Hkv, d), dtype=dt, device=dev)
        self.v_new = torch.zeros((B, Hkv, d), dtype=dt, device=dev)
        self.out = torch.zeros((B, Hq, d), dtype=dt, device=dev)
        # one ordinary (state-free) launch first, so per-device kernel attributes
        # are set outside the capture
        dense_decode(cfg, self.q, K, V, lens, self.out, buf.workspace, buf.status)
        before = launch_count()
        self.graph = torch.cuda.CUDAGraph()
        torch.cuda.synchronize()
        with torch.cuda.graph(self.graph):
            decode(cfg, buf.tree, K, V, refs, lens, self.q, self.k_new, self.v_new, p, buf.sel, self.out,
                   buf.workspace, buf.status)
        self.kernels_per_step = launch_count() - before

    def stage(self, q, k_new, v_new):
        """Put a step's inputs into the graph's own buffers (one multi-tensor
        copy); a caller that produces them there directly skips this."""
        torch._foreach_copy_([self.q, self.k_new, self.v_new], [q, k_new, v_new], non_blocking=True)

    def replay(self):
        """One decode step on the inputs in the graph's buffers."""
        self.graph.replay()
        return self.out

    def step(self, q, k_new, v_new):
        self.stage(q, k_new, v_new)
        return self.replay()


class Buffers:
    """Device buffers one configuration needs: tree, workspace, selection, status."""

    def __init__(self, cfg: Config, device="cuda", level_kept: bool = True):
        self.cfg = cfg
        cap1 = max(level_nodes(cfg, cfg.max_len, 1), 1)
        G = cfg.n_kv_heads * cfg.batch
        self.tree = torch.empty(tree_bytes(cfg), dtype=torch.uint8, device=device)
        self.workspace = torch.zeros(workspace_bytes(cfg), dtype=torch.uint8, device=device)
        self.sel = {
            "leaf_idx": torch.zeros((cfg.batch, cfg.n_kv_heads, cap1), dtype=torch.int32, device=device),
            "head_mask": torch.zeros((cfg.batch, cfg.n_kv_heads, cap1), dtype=torch.int32, device=device),
            "count": torch.zeros((cfg.batch, cfg.n_kv_heads), dtype=torch.int32, device=device),
            # [B, Hq, L] for single queries; a block call writes [B, Hkv, T, G, L]
            "level_kept": (torch.zeros((cfg.batch, cfg.n_q_heads * max(cfg.queries, 1), cfg.levels),
                                       dtype=torch.int32, device=device) if level_kept else None),
        }
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        del G

    def check_status(self, where="device"):
        code = int(self.status.item())
        if code:
            self.status.zero_()
            raise ZhaError(code, where)

    # views of the tree buffer (for inspection and tests)
    def tree_level(self, level: int):
        """(mu, bias) views of one level; with MX-FP8 summaries mu is the E4M3
        byte array and tree_level_scales() gives the block scales."""
        cfg = self.cfg
        mu_off, b_off = tree_level_offsets(cfg, level)
        cap = level_nodes(cfg, cfg.max_len, level)
        shape = (cfg.batch, cfg.n_kv_heads, cap, cfg.n_refs, cfg.head_dim)
        n_mu = cfg.batch * cfg.n_kv_heads * cap * cfg.n_refs * cfg.head_dim
        if cfg.summary == ZHA_SUMMARY_MXFP8:
            mu = self.tree[mu_off:mu_off + n_mu].view(*shape)
        else:
            es = 2 if cfg.dtype == ZHA_BF16 else 4
            mu = self.tree[mu_off:mu_off + n_mu * es].view(cfg.torch_dtype).view(*shape)
        n_b = cfg.batch * cfg.n_kv_heads * cap * cfg.n_refs
        bias = self.tree[b_off:b_off + n_b * 4].view(torch.float32).view(cfg.batch, cfg.n_kv_heads, cap, cfg.n_refs)
        return mu, bias

    def tree_level_scales(self, level: int):
        """Block-scale bytes [B, Hkv, cap, R, d/32] of an MX-FP8 level (2^(byte-127))."""
        cfg = self.cfg
        off = ctypes.c_size_t()
        check(_lib.zha_tree_level_scales(ctypes.byref(cfg), level, ctypes.byref(off)), "zha_tree_level_scales")
        cap = level_nodes(cfg, cfg.max_len, level)
        n = cfg.batch * cfg.n_kv_heads * cap * cfg.n_refs * (cfg.head_dim // 32)
        return self.tree[off.value:off.value + n].view(cfg.batch, cfg.n_kv_heads, cap, cfg.n_refs,
                                                        cfg.head_dim // 32)

    def tree_level_logmass(self, level: int):
        """Log-masses F [B, Hkv, cap, R] of one level (each plane's log attention
        mass at its own reference)."""
        cfg = self.cfg
        off = ctypes.c_size_t()
        check(_lib.zha_tree_level_logmass(ctypes.byref(cfg), level, ctypes.byref(off)), "zha_tree_level_logmass")
        cap = level_nodes(cfg, cfg.max_len, level)
        n = cfg.batch * cfg.n_kv_heads * cap * cfg.n_refs
        return self.tree[off.value:off.value + n * 4].view(torch.float32).view(cfg.batch, cfg.n_kv_heads, cap,
                                                                               cfg.n_refs)

    def level_state(self, level: int, T: int = 1):
        """Routing state of one level from the last route/decode call (T: query
        positions of the last decode_block call; its rows are t * G + head)."""
        cfg = self.cfg
        v = workspace_level_view(cfg, level, T)
        cap = v.cap
        BG = cfg.batch * cfg.n_kv_heads
        G = cfg.group * T
        ws = self.workspace

        def arr(off, n, dt):
            return ws[off:off + n * 4].view(dt)

        return {
            "cap": cap,
            "cand_idx": arr(v.cand_idx, BG * cap, torch.int32).view(cfg.batch, cfg.n_kv_heads, cap),
            "cand_mask": arr(v.cand_mask, BG * cap, torch.int32).view(cfg.batch, cfg.n_kv_heads, cap),
            "scores": arr(v.scores, BG * G * cap, torch.float32).view(cfg.batch, cfg.n_kv_heads, G, cap),
            "kept_mask": arr(v.kept_mask, BG * cap, torch.int32).view(cfg.batch, cfg.n_kv_heads, cap),
            "count": arr(v.count, BG, torch.int32).view(cfg.batch, cfg.n_kv_heads),
        }
