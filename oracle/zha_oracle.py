"""Python face of the fp64 CPU oracle of the ZHA decode path (``zha_oracle.c``).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this module. It never imports the
product package, and the product package never imports it.

Every function works on ONE (sequence, KV head) pair -- one summary tree and
the G query heads that share it -- with numpy float64 arrays. Inputs stored in
bf16 or fp32 on the GPU are handed over already widened to float64, so both
sides see the same values.

The method (page "Zyphra AI Introduces Zyphra Hierarchical Attention (ZHA)",
sections "Building the tree" and "How does top-p routing pick tokens", plus the
explainer widget's step-5 caption) and the readings taken where those pages
are loose are listed at the top of ``zha_oracle.c``.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zha_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libzha_oracle.so")

STORE_F64, STORE_F32, STORE_BF16, STORE_MXFP8 = 0, 1, 2, 3
_STORAGE = {"f64": STORE_F64, "f32": STORE_F32, "bf16": STORE_BF16, "mxfp8": STORE_MXFP8}


def build_library(force: bool = False) -> str:
    """Compile zha_oracle.c with gcc (plain -O2, IEEE arithmetic, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build_library())
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.orc_round_storage.argtypes = [f64, i32]
        L.orc_round_storage.restype = f64
        L.orc_e4m3_round.argtypes = [f64]
        L.orc_e4m3_round.restype = f64
        L.orc_mx_round.argtypes = [P, i32, P]
        L.orc_parent_planes.argtypes = [P, P, i64, i32, P, i32, f64, i32, P, P, P]
        L.orc_num_threads.restype = i32
        L.orc_level_nodes.argtypes = [i64, i32, i32]
        L.orc_level_nodes.restype = i64
        L.orc_direct_planes.argtypes = [P, i64, i64, i32, P, i32, f64, P, P]
        L.orc_tree_update.argtypes = [P, i64, i64, i32, P, i32, i32, i32, f64, i32, P, P, P]
        L.orc_estimate.argtypes = [P, P, P, i32, i32, f64]
        L.orc_estimate.restype = f64
        L.orc_topp_select.argtypes = [i64, P, f64, P, P]
        L.orc_topp_select.restype = i64
        L.orc_route.argtypes = [P, i32, i32, f64, i32, i32, i32, i64, P, P, P, P, P, P, P]
        L.orc_token_set.argtypes = [i64, i32, i64, P, i32, P]
        L.orc_attend.argtypes = [P, P, P, i64, i32, f64, P, P]
        _lib = L
    return _lib


def num_threads() -> int:
    return lib().orc_num_threads()


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def round_storage(x: float, storage: str) -> float:
    return lib().orc_round_storage(float(x), _STORAGE[storage])


def e4m3_round(x: float) -> float:
    """Nearest FP8 E4M3 value (ties to even, saturating at 448)."""
    return lib().orc_e4m3_round(float(x))


def mx_round(x: np.ndarray):
    """MX-FP8 value of planes x [..., d] (blocks of 32 coordinates) -> (values, block exponents)."""
    x = np.array(x, dtype=np.float64, order="C", copy=True)
    d = x.shape[-1]
    flat = x.reshape(-1, d)
    exps = np.zeros((flat.shape[0], d // 32), dtype=np.int32)
    for i in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[i])
        lib().orc_mx_round(_ptr(row), d, exps[i].ctypes.data)
        flat[i] = row
    return flat.reshape(x.shape), exps.reshape(x.shape[:-1] + (d // 32,))


def level_nodes(N: int, c: int, level: int) -> int:
    """Nodes at `level` (1 = leaf chunks) for N cached tokens: floor(N/c), then ceil(./c)."""
    return int(lib().orc_level_nodes(int(N), int(c), int(level)))


@dataclass
class Tree:
    """Summary tree of one (sequence, KV head): mu[l-1] [cap_l, R, d], b[l-1] [cap_l, R],
    F[l-1] [cap_l, R] (each plane's log-mass at its reference, which parents weight
    their children by)."""
    c: int
    L: int
    R: int
    d: int
    s: float
    storage: str
    N: int = 0
    mu: list = field(default_factory=list)
    b: list = field(default_factory=list)
    F: list = field(default_factory=list)

    def n(self, level: int) -> int:
        return level_nodes(self.N, self.c, level)


def new_tree(cap_tokens: int, c: int, L: int, R: int, d: int, s: float | None = None,
             storage: str = "f64") -> Tree:
    s = default_scale(d) if s is None else s
    t = Tree(c=c, L=L, R=R, d=d, s=s, storage=storage)
    for level in range(1, L + 1):
        n = max(level_nodes(cap_tokens, c, level), 1)
        t.mu.append(np.zeros((n, R, d)))
        t.b.append(np.zeros((n, R)))
        t.F.append(np.zeros((n, R)))
    return t


def tree_update(tree: Tree, K: np.ndarray, refs: np.ndarray, new_N: int) -> Tree:
    """Extend the tree from tree.N to new_N tokens of K ([>=new_N, d])."""
    K = _f64(K)
    refs = _f64(refs)
    assert refs.shape == (tree.R, tree.d) and K.shape[1] == tree.d and K.shape[0] >= new_N
    assert tree.mu[0].shape[0] >= level_nodes(new_N, tree.c, 1) or level_nodes(new_N, tree.c, 1) == 0
    mus = (ctypes.c_void_p * tree.L)(*[m.ctypes.data for m in tree.mu])
    bs = (ctypes.c_void_p * tree.L)(*[b.ctypes.data for b in tree.b])
    Fs = (ctypes.c_void_p * tree.L)(*[f.ctypes.data for f in tree.F])
    lib().orc_tree_update(_ptr(K), int(tree.N), int(new_N), tree.d, _ptr(refs), tree.R, tree.c,
                          tree.L, tree.s, _STORAGE[tree.storage], mus, bs, Fs)
    tree.N = int(new_N)
    return tree


def build_tree(K: np.ndarray, refs: np.ndarray, N: int, c: int, L: int, s: float | None = None,
               storage: str = "f64", cap_tokens: int | None = None) -> Tree:
    refs = _f64(refs)
    R, d = refs.shape
    t = new_tree(cap_tokens or N, c, L, R, d, s, storage)
    return tree_update(t, K, refs, N)


def direct_planes(K: np.ndarray, t0: int, t1: int, refs: np.ndarray, s: float):
    """Planes of every reference straight from the raw keys K[t0:t1] (no tree)."""
    K = _f64(K)
    refs = _f64(refs)
    R, d = refs.shape
    mu = np.zeros((R, d))
    b = np.zeros(R)
    lib().orc_direct_planes(_ptr(K), int(t0), int(t1), d, _ptr(refs), R, float(s), _ptr(mu), _ptr(b))
    return mu, b


def parent_planes(child_mu: np.ndarray, child_F: np.ndarray, refs: np.ndarray, s: float,
                  storage: str = "f64"):
    """Planes of one parent from given children (child_mu [n, R, d] and their
    log-masses child_F [n, R]) -> (mu [R, d], b [R], F [R])."""
    cm, cf, refs = _f64(child_mu), _f64(child_F), _f64(refs)
    n, R, d = cm.shape
    mu = np.zeros((R, d))
    b = np.zeros(R)
    F = np.zeros(R)
    lib().orc_parent_planes(_ptr(cm), _ptr(cf), n, d, _ptr(refs), R, float(s), _STORAGE[storage], _ptr(mu),
                            _ptr(b), _ptr(F))
    return mu, b, F


def estimate(q: np.ndarray, mu: np.ndarray, b: np.ndarray, s: float) -> float:
    q, mu, b = _f64(q), _f64(mu), _f64(b)
    R, d = mu.shape
    return lib().orc_estimate(_ptr(q), _ptr(mu), _ptr(b), R, d, float(s))


def topp_select(E: np.ndarray, p: float):
    """Top-p over candidates in ascending node order -> (kept bool[n], cum_before float[n])."""
    E = _f64(E)
    n = E.shape[0]
    kept = np.zeros(n, dtype=np.uint8)
    cumb = np.zeros(n)
    lib().orc_topp_select(n, _ptr(E), float(p), _ptr(kept), _ptr(cumb))
    return kept.astype(bool), cumb


@dataclass
class Route:
    """Per level l (index l-1) arrays [G, n_l]: cand, kept (bool), score, cum_before."""
    cand: list
    kept: list
    score: list
    cumb: list

    def kept_leaves(self, h: int) -> np.ndarray:
        return np.nonzero(self.kept[0][h])[0]


def route(tree: Tree, q: np.ndarray, p) -> Route:
    """Route the G queries q [G, d] through the tree; p is one float or one per level."""
    q = _f64(q)
    G, d = q.shape
    L = tree.L
    p_level = np.full(L, float(p)) if np.isscalar(p) else _f64(p)
    assert p_level.shape == (L,)
    n1 = tree.n(1)
    nl = [level_nodes(tree.N, tree.c, l) for l in range(1, L + 1)]
    tot = sum(nl)
    cand = np.zeros((G, max(tot, 1)), dtype=np.uint8)
    kept = np.zeros((G, max(tot, 1)), dtype=np.uint8)
    score = np.full((G, max(tot, 1)), -np.inf)
    cumb = np.full((G, max(tot, 1)), np.nan)
    mus = (ctypes.c_void_p * L)(*[m.ctypes.data for m in tree.mu])
    bs = (ctypes.c_void_p * L)(*[b.ctypes.data for b in tree.b])
    lib().orc_route(_ptr(q), G, d, tree.s, tree.R, tree.c, L, n1, mus, bs, _ptr(p_level),
                    _ptr(cand), _ptr(kept), _ptr(score), _ptr(cumb))
    out = Route([], [], [], [])
    off = 0
    for l in range(L):
        sl = slice(off, off + nl[l])
        out.cand.append(cand[:, sl].astype(bool))
        out.kept.append(kept[:, sl].astype(bool))
        out.score.append(score[:, sl])
        out.cumb.append(cumb[:, sl])
        off += nl[l]
    return out


def depth_root_schedule(p: float, L: int) -> list:
    """Per-level fractions p^(1/L) (level 1 first), so that their product over the
    L levels is p. The explainer's caveat cards (MarkTechPost, tab 5) warn that
    one fixed p per level shrinks coverage with depth; the pages name no
    schedule, and this is the plainest one that undoes the p^L shrinkage."""
    v = 1.0 if p >= 1.0 else float(p) ** (1.0 / L)
    return [v] * L


def token_set(N: int, c: int, kept_leaf: np.ndarray, tail_only: bool = False) -> np.ndarray:
    """Attended tokens: sink, kept leaf chunks, current chunk -> bool[N]."""
    kl = np.ascontiguousarray(kept_leaf, dtype=np.uint8)
    tm = np.zeros(max(N, 1), dtype=np.uint8)
    lib().orc_token_set(int(N), int(c), int(kl.shape[0]), _ptr(kl), int(bool(tail_only)), _ptr(tm))
    return tm[:N].astype(bool)


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, N: int, s: float, tmask=None) -> np.ndarray:
    """Exact softmax attention of one query over tokens [0, N) (optionally masked)."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    d = q.shape[0]
    out = np.zeros(d)
    tm = None if tmask is None else np.ascontiguousarray(tmask, dtype=np.uint8)
    lib().orc_attend(_ptr(q), _ptr(K), _ptr(V), int(N), d, float(s),
                     None if tm is None else _ptr(tm), _ptr(out))
    return out


def decode_group(tree: Tree, q: np.ndarray, K: np.ndarray, V: np.ndarray, p, tail_only=False):
    """Route the G heads of one group, then attend each over its token set.

    Returns (out [G, d], route, token masks [G, N]).
    """
    q = _f64(q)
    G = q.shape[0]
    N = tree.N
    r = route(tree, q, p)
    outs = np.zeros((G, tree.d))
    masks = np.zeros((G, N), dtype=bool)
    for h in range(G):
        kept_leaf = r.kept[0][h] if tree.n(1) > 0 else np.zeros(0, dtype=bool)
        masks[h] = token_set(N, tree.c, kept_leaf, tail_only)
        outs[h] = attend(q[h], K, V, N, tree.s, masks[h])
    return outs, r, masks


# ----------------------------------------------------------- multi-query blocks
#
# T consecutive query positions of one sequence at once (a multi-query decode
# or a chunked-prefill block). The pages describe routing for one decoding
# query ("How does top-p routing pick tokens"); the reading taken for a block:
# every query routes over the tree of the N0 tokens cached before the block,
# and query t attends {0} U its kept leaf chunks U [c*floor(N0/c), N0 + t],
# i.e. the cached tail after the tree's last complete chunk and the block's
# own tokens up to its position (causal).


def block_token_set(N0: int, t: int, c: int, kept_leaf: np.ndarray) -> np.ndarray:
    """Tokens query t of a block attends -> bool[N0 + t + 1]."""
    n = N0 + t + 1
    m = np.zeros(n, dtype=bool)
    m[0] = True
    for j in np.nonzero(np.asarray(kept_leaf, dtype=bool))[0]:
        m[j * c:(j + 1) * c] = True
    m[c * (N0 // c):n] = True
    return m


def decode_block_group(tree: Tree, q: np.ndarray, K: np.ndarray, V: np.ndarray, p):
    """One group's block: q [T, G, d], K/V hold at least tree.N + T tokens.

    Returns (out [T, G, d], route over the T*G rows (row t*G + h), token masks
    per row [T*G] of bool arrays)."""
    q = _f64(q)
    T, G, d = q.shape
    N0 = tree.N
    r = route(tree, q.reshape(T * G, d), p)
    out = np.zeros((T, G, d))
    masks = []
    for t in range(T):
        for h in range(G):
            row = t * G + h
            kept_leaf = r.kept[0][row] if tree.n(1) > 0 else np.zeros(0, dtype=bool)
            m = block_token_set(N0, t, tree.c, kept_leaf)
            masks.append(m)
            out[t, h] = attend(q[t, h], K, V, N0 + t + 1, tree.s, m)
    return out, r, masks
