"""Shared helpers of the GPU parity tests: run the oracle on the same inputs
the CUDA path gets, and compare the two the way the method allows."""
from __future__ import annotations

import math
import os

import numpy as np
import torch

import zha_oracle as orc
from tree_indexed_sparse_02_b200.inputs import Workload, make_inputs

# tolerances, err = max|gpu - oracle| / max(max|oracle|, 1)
TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(gpu, ref) -> float:
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    if r.size == 0:
        return 0.0
    return float(np.max(np.abs(g - r)) / max(float(np.max(np.abs(r))), 1.0))


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def storage(w: Workload) -> str:
    if w.summary == "mxfp8":
        return "mxfp8"
    return "bf16" if w.dtype == "bf16" else "f32"


def mx_byte_offsets(d: int) -> np.ndarray:
    """Byte position of each coordinate in a stored MX-FP8 row (the order
    include/zha.h gives): block b = k // 32, w = k % 32 sits at
    64 (b // 2) + 16 ((w % 16) // 4) + 8 (b % 2) + 4 (w // 16) + w % 4."""
    k = np.arange(d)
    b, w = k // 32, k % 32
    return 64 * (b // 2) + 16 * ((w % 16) // 4) + 8 * (b % 2) + 4 * (w // 16) + w % 4


def mx_decode(mu8: torch.Tensor, scales: torch.Tensor) -> np.ndarray:
    """Values of MX-FP8 planes read back from the device: E4M3 bytes [..., d]
    (stored in the permuted order) times 2^(scale byte - 127) per 32
    coordinates, in float64, in coordinate order."""
    d = mu8.shape[-1]
    perm = torch.from_numpy(mx_byte_offsets(d)).to(mu8.device)
    v = mu8.contiguous()[..., perm].contiguous().view(torch.float8_e4m3fn).to(torch.float64)
    sc = torch.exp2(scales.to(torch.float64) - 127.0).repeat_interleave(32, dim=-1)
    return (v * sc).cpu().numpy()


def mx_workloads():
    """The bf16 parity cases with MX-FP8 summaries."""
    import dataclasses
    return [dataclasses.replace(w, name=w.name + " mxfp8", summary="mxfp8")
            for w in small_workloads() if w.dtype == "bf16"]


def make_cfg(zha, w: Workload, cap: int, flags: int = 0, splits: int = 0):
    return zha.config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.levels, w.n_refs,
                      w.dtype, cap, flags=flags, attn_splits=splits, summary=w.summary)


def to_device(inp, device="cuda"):
    from tree_indexed_sparse_02_b200.inputs import Inputs
    return Inputs(K=inp.K.to(device), V=inp.V.to(device), q=inp.q.to(device), refs=inp.refs.to(device),
                  lens=inp.lens.to(device), needle_pos=inp.needle_pos)


def oracle_tree(w: Workload, inp, b: int, kvh: int, N: int, s: float, cap_tokens: int | None = None):
    K = np64(inp.K[b, kvh, :max(N, 1)])
    refs = np64(inp.refs[kvh])
    return orc.build_tree(K, refs, N, w.chunk, w.levels, s, storage=storage(w),
                          cap_tokens=max(cap_tokens or N, 1))


def gpu_level_candidates(state, b, kvh, h, n_l):
    """GPU candidates / kept / scores of query head h (within its group) as arrays over nodes."""
    cnt = int(state["count"][b, kvh])
    idx = state["cand_idx"][b, kvh, :cnt].cpu().numpy().astype(np.int64)
    cm = state["cand_mask"][b, kvh, :cnt].cpu().numpy().astype(np.uint32)
    km = state["kept_mask"][b, kvh, :cnt].cpu().numpy().astype(np.uint32)
    sc = state["scores"][b, kvh, h, :cnt].cpu().numpy().astype(np.float64)
    assert np.all(np.diff(idx) > 0), "candidate list must be strictly ascending"
    # entries with an empty head mask are padding (children past the level's end)
    real = cm != 0
    assert not np.any(km[~real]), "padding entry kept"
    idx, cm, km, sc = idx[real], cm[real], km[real], sc[real]
    bit = np.uint32(1 << h)
    cand = np.zeros(n_l, dtype=bool)
    kept = np.zeros(n_l, dtype=bool)
    score = np.full(n_l, -np.inf)
    member = (cm & bit) != 0
    assert idx.size == 0 or (idx.min() >= 0 and idx.max() < n_l)
    cand[idx[member]] = True
    kept[idx[member & ((km & bit) != 0)]] = True
    assert not np.any((km & ~cm) != 0), "kept by a head that did not have it as a candidate"
    score[idx] = sc
    return cand, kept, score


def fixed_point_band(E) -> float:
    """Bound on the error of a running-mass fraction that the GPU's selection
    sums in fixed point: each candidate's mass e^(E - max) is rounded to a
    multiple of 2^-31 (error <= 2^-32), so a running sum of up to n of them is
    off by at most n 2^-32, and a fraction of the total Z = sum e^(E - max)
    (>= 1) by at most n 2^-32 / Z."""
    E = np.asarray(E, dtype=np.float64)
    E = E[np.isfinite(E)]
    if E.size == 0:
        return 0.0
    Z = float(np.sum(np.exp(E - E.max())))
    return E.size * 2.0 ** -32 / Z


# Every boundary flip the routing comparisons meet, reported at the end of
# the pytest run (tests/conftest.py): which test, level, query head and node,
# the oracle's running mass before the node and its distance from p.
FLIPS: list = []
ROUTES_COMPARED = {"heads": 0}


def _current_test() -> str:
    return os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]


def compare_routing(route_o, states, b, kvh, G, N, w: Workload, p_levels):
    """Level-by-level comparison of one group's routing. Flips (nodes kept by
    one side only) are allowed only where the oracle's running mass before the
    node is within the band of p that the score error and the fixed-point mass
    sum allow (4 x score error + 1e-5 + fixed_point_band), widened by the
    mass of candidates whose scores are within twice the score error of the
    node's (near ties the two sides may order differently); each one is
    recorded in FLIPS. A head is compared down to its first flip: below it
    the two sides route over different candidate sets (scores of the common
    candidates are still compared).
    Returns (flipped_heads, max score err)."""
    L = w.levels
    flipped = set()
    worst = 0.0
    ROUTES_COMPARED["heads"] += G
    for h in range(G):
        diverged = False
        for level in range(L, 0, -1):
            n_l = orc.level_nodes(N, w.chunk, level)
            cand_g, kept_g, score_g = gpu_level_candidates(states[level], b, kvh, h, n_l)
            cand_o = route_o.cand[level - 1][h]
            kept_o = route_o.kept[level - 1][h]
            if not diverged:
                assert np.array_equal(cand_g, cand_o), (h, level)
            common = cand_g & cand_o
            if not common.any():
                continue
            so = route_o.score[level - 1][h][common]
            sg = score_g[common]
            err = float(np.max(np.abs(sg - so)))
            worst = max(worst, err / max(1.0, float(np.max(np.abs(so)))))
            if diverged:
                # after a flip above, the two sides score different candidate
                # sets at this level: their running masses are not comparable
                continue
            flips = np.nonzero((kept_g != kept_o) & common)[0]
            if flips.size:
                p = float(p_levels[level - 1])
                Eo = route_o.score[level - 1][h]
                band = 4.0 * err + 1e-5 + fixed_point_band(Eo[cand_o])
                cb = route_o.cumb[level - 1][h]
                # normalised masses of the head's candidates at this level
                mass = np.zeros(n_l)
                mass[cand_o] = np.exp(Eo[cand_o] - np.max(Eo[cand_o]))
                mass /= mass.sum()
                for n in flips:
                    # candidates whose scores lie within twice the score error of
                    # this one may sit on either side of it in the GPU's order,
                    # moving its running mass by theirs
                    near = cand_o & (np.abs(Eo - Eo[n]) <= 2.0 * err + 1e-12)
                    near[n] = False
                    slack = float(mass[near].sum())
                    FLIPS.append({"test": _current_test(), "group": (int(b), int(kvh)), "level": level,
                                  "head": h, "node": int(n), "cum_before": float(cb[n]), "p": p,
                                  "dist": float(abs(cb[n] - p)), "band": band, "near_tie_mass": slack,
                                  "kept_by": "gpu" if kept_g[n] else "oracle"})
                    assert abs(cb[n] - p) <= band + slack, (
                        f"head {h} level {level} node {n}: cum {cb[n]:.6f} vs p {p} "
                        f"(band {band:.2e}, near-tie mass {slack:.2e})")
                diverged = True
                flipped.add(h)
    return flipped, worst


def selection_to_masks(sel, b, kvh, G, N, c, tail_only=False):
    """Per-head attended-token masks implied by a selection (via the oracle's token rule)."""
    cnt = int(sel["count"][b, kvh])
    idx = sel["leaf_idx"][b, kvh, :cnt].cpu().numpy().astype(np.int64)
    hm = sel["head_mask"][b, kvh, :cnt].cpu().numpy().astype(np.uint32)
    n1 = N // c
    out = []
    for h in range(G):
        kl = np.zeros(n1, dtype=bool)
        kl[idx[(hm >> np.uint32(h)) & np.uint32(1) != 0]] = True
        out.append(orc.token_set(N, c, kl, tail_only))
    return out


def scale_of(w: Workload) -> float:
    return 1.0 / math.sqrt(w.head_dim)


def small_workloads():
    """Parity cases small enough for the oracle: several tiles and ragged tails."""
    from tree_indexed_sparse_02_b200.inputs import TINY_F32, WIDE_32K
    deep = Workload("deep-small bf16 B=2 c=4 L=4", 2, 16, 2, 128, 3001, 4, 4, 16, 0.95, 16, "bf16", 11)
    g16 = Workload("G16 R32 d64 c=8 L=3", 1, 32, 2, 64, 2500, 8, 3, 32, 0.9, 8, "bf16", 12)
    r1 = Workload("R1 c=8 p=0.75", 1, 8, 1, 128, 5003, 8, 4, 1, 0.75, 4, "bf16", 13)
    return [TINY_F32, deep, g16, r1, WIDE_32K]


def build_case(zha, w: Workload, extra_cap: int = 64, lens=None, device="cuda", gen_device="cpu"):
    cap = w.context + extra_cap
    inp = make_inputs(w, device=gen_device, capacity=cap, lens=lens)
    dev = to_device(inp, device)
    cfg = make_cfg(zha, w, cap)
    buf = zha.Buffers(cfg, device=device)
    return cfg, inp, dev, buf


def check_group_vs_oracle(w: Workload, inp, buf, b: int, kvh: int, p_levels, out=None, tol=None,
                          max_flipped: int = 2):
    """One (sequence, KV head) group of a routed (and optionally attended) call
    against the oracle on the same inputs: routing level by level
    (compare_routing), the selection's per-head leaf sets and kept counts for
    every head without a boundary flip, and -- if `out` is given -- each such
    head's attention output. Returns the set of flipped heads."""
    G, s = w.group, scale_of(w)
    N = int(inp.lens[b])
    t = oracle_tree(w, inp, b, kvh, N, s)
    K = np64(inp.K[b, kvh, :N])
    V = np64(inp.V[b, kvh, :N])
    q = np64(inp.q[b, kvh * G:(kvh + 1) * G])
    o, r, _ = orc.decode_group(t, q, K, V, p_levels)
    states = {l: buf.level_state(l) for l in range(1, w.levels + 1)}
    flipped, worst = compare_routing(r, states, b, kvh, G, N, w, p_levels)
    tol = TOL[w.dtype] if tol is None else tol
    assert worst <= tol, worst
    assert len(flipped) <= max_flipped, flipped
    cnt = int(buf.sel["count"][b, kvh])
    idx = buf.sel["leaf_idx"][b, kvh, :cnt].cpu().numpy()
    assert np.all(np.diff(idx) > 0)
    hm = buf.sel["head_mask"][b, kvh, :cnt].cpu().numpy().astype(np.uint32)
    got = None if out is None else np64(out[b, kvh * G:(kvh + 1) * G])
    for h in range(G):
        if h in flipped:
            continue
        assert np.array_equal(np.sort(idx[(hm >> np.uint32(h)) & 1 != 0]), np.nonzero(r.kept[0][h])[0]), h
        if buf.sel.get("level_kept") is not None:
            lk = buf.sel["level_kept"][b, kvh * G + h].cpu().numpy()
            for level in range(1, w.levels + 1):
                assert lk[level - 1] == r.kept[level - 1][h].sum(), (h, level)
        if got is not None:
            assert rel_err(got[h], o[h]) <= tol, h
    return flipped
