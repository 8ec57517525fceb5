"""Seeded synthetic inputs for the ZHA decode path.

This module draws random tensors and places planted "needle" keys; it holds
none of the method's arithmetic. Both the CUDA path and the CPU oracle are fed
from it (the oracle after widening the same rounded values to float64).

Recipe (all draws from one seeded ``torch.Generator`` on the chosen device;
fp32 draws are rounded once, round-to-nearest-even, to the storage dtype):

* keys    k_t = z_t + m_{floor(t/c)},  z ~ N(0, I_d),  per-chunk offset
  m ~ N(0, 0.5 I_d) (variance 0.5), c = the tree's chunk size;
* values  ~ N(0, I_d); queries q_{b,h} ~ N(0, I_d);
* reference queries ("random" mode) ~ N(0, I_d / d); in "aligned" mode (a
  training-free stand-in for learned references, which serve every sequence)
  each query head h has one direction u_h ~ N(0, I_d) shared by the whole
  batch, sequence b's query is q_{b,h} = u_h + 0.1 e_{b,h} (e ~ N(0, I_d)),
  and the first min(G, R) references of KV head g are its query heads' u_h
  (the rest drawn as in "random" mode);
* decode steps: query of step i = q_{b,h} + 0.1 N(0, I_d), so every step asks
  for what the needles of its head were planted for;
* needles: ``needles`` per sequence, assigned round-robin to the query heads;
  needle j of head h sits at a position drawn without replacement from
  [1, N - c) in KV head h // G, with key 3 sqrt(d) q_h/|q_h| + z;
* diffuse heads (optional): the last query head of every KV group gets
  ``diffuse_nodes`` extra needles, one in each of that many distinct top
  nodes (spans of c**L tokens) drawn at random.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass
class Workload:
    """Shapes and generator settings of one synthetic decode workload."""
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    context: int          # N tokens already in the cache when decoding starts
    chunk: int            # c
    levels: int           # L
    n_refs: int           # R
    p: float
    needles: int          # per sequence
    dtype: str            # "bf16" or "f32"
    seed: int
    diffuse_nodes: int = 0
    refs_mode: str = "random"
    p_schedule: str = "fixed"   # "fixed": p per level; "root": p^(1/L) per level
    summary: str = "native"     # "native": mu in the KV dtype; "mxfp8": E4M3 blocks of 32 + scales

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


# The workloads the method is exercised on (head_dim 128 unless noted).
TINY_F32 = Workload("tiny-f32 N=4096 c=4 L=3", 1, 2, 1, 64, 4096, 4, 3, 16, 0.95, 8, "f32", 0)
WIDE_32K = Workload("wide N=32768 c=256 L=1", 1, 32, 4, 128, 32768, 256, 1, 16, 0.95, 64, "bf16", 1)
DEEP_256K = Workload("deep N=262144 c=4 L=6 B=4", 4, 32, 4, 128, 262144, 4, 6, 16, 0.95, 256, "bf16", 2,
                     diffuse_nodes=32)
DEEP_1M = Workload("deep N=1048576 c=4 L=6", 1, 32, 4, 128, 1048576, 4, 6, 16, 0.95, 256, "bf16", 3)
# The geometry of the pages' latency model (MarkTechPost, "How fast is ZHA" and the
# explainer's tab 4): one reference per tree, chunks of 8, p = 0.75, batch 1.
# Four levels give 4,096 tokens per top node, as in the deep tree.
SPEED_256K = Workload("speed-model N=262144 c=8 L=4 R=1 p=0.75", 1, 32, 4, 128, 262144, 8, 4, 1, 0.75, 64,
                      "bf16", 5)


def sweep_workload(N: int, tree: str) -> Workload:
    """Context-sweep workload (batch 1, 32/4 heads, d 128) with the deep, wide or
    speed-model (R=1, c=8, L=4, p=0.75) tree."""
    c, L, R, p = {"deep": (4, 6, 16, 0.95), "wide": (256, 1, 16, 0.95), "speed": (8, 4, 1, 0.75)}[tree]
    return Workload(f"sweep-{tree} N={N}", 1, 32, 4, 128, N, c, L, R, p, 64, "bf16", 4)


@dataclass
class Inputs:
    K: torch.Tensor        # [B, Hkv, cap, d]
    V: torch.Tensor        # [B, Hkv, cap, d]
    q: torch.Tensor        # [B, Hq, d]
    refs: torch.Tensor     # [Hkv, R, d]
    lens: torch.Tensor     # [B] int32 (tokens in the cache)
    needle_pos: list       # per sequence: list of (query head, position)


def _randn(gen, shape, device, std=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return x * std if std != 1.0 else x


def _draw_queries(w: Workload, gen, device):
    """Queries [B, Hq, d] and references [Hkv, R, d] (fp32), the generator's
    first draws."""
    B, Hq, Hkv, d, G = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.group
    q = _randn(gen, (B, Hq, d), device)
    refs = _randn(gen, (Hkv, w.n_refs, d), device, std=1.0 / math.sqrt(d))
    if w.refs_mode == "aligned":
        # one direction per query head for the whole batch (sequence 0's draws),
        # which is what references trained on many sequences would point at
        u = q[0].clone()
        for g in range(Hkv):
            for r in range(min(G, w.n_refs)):
                refs[g, r] = u[g * G + r]
        q = u.unsqueeze(0) + 0.1 * _randn(gen, (B, Hq, d), device)
    return q, refs


def make_inputs(w: Workload, device="cpu", capacity: int | None = None, lens=None) -> Inputs:
    """Draw K, V (for `capacity` >= N slots), q, refs and place the needles.

    `lens` (list of ints, default N for every sequence) lets sequences of a
    batch hold different numbers of tokens; keys beyond a sequence's length
    are still drawn (they are the tokens later appends write).
    """
    B, Hq, Hkv, d, c = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk
    G = w.group
    N = w.context
    cap = max(capacity or N, N)
    lens = [N] * B if lens is None else list(lens)
    dt = w.torch_dtype()
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)

    q, refs = _draw_queries(w, gen, device)
    K = torch.empty((B, Hkv, cap, d), dtype=dt, device=device)
    V = torch.empty((B, Hkv, cap, d), dtype=dt, device=device)
    n_chunks = (cap + c - 1) // c
    for b in range(B):
        for g in range(Hkv):
            off = _randn(gen, (n_chunks, d), device, std=math.sqrt(0.5))
            z = _randn(gen, (cap, d), device)
            z += off.repeat_interleave(c, dim=0)[:cap]
            K[b, g] = z.to(dt)
            V[b, g] = _randn(gen, (cap, d), device).to(dt)

    needle_pos = []
    span_top = c ** w.levels
    for b in range(B):
        Nb = lens[b]
        placed = []
        hi = max(Nb - c, 2)
        perm = torch.randperm(hi - 1, generator=gen, device=device)[: max(w.needles, 0)] + 1
        for j in range(min(w.needles, perm.numel())):
            h = j % Hq
            placed.append((h, int(perm[j])))
        if w.diffuse_nodes:
            n_top = max(Nb // span_top, 1)
            for g in range(Hkv):
                h = g * G + G - 1
                k = min(w.diffuse_nodes, n_top)
                tops = torch.randperm(n_top, generator=gen, device=device)[:k]
                for t in tops.tolist():
                    lo, hi_t = t * span_top + 1, min((t + 1) * span_top, Nb - c)
                    if hi_t <= lo:
                        continue
                    pos = lo + int(torch.randint(hi_t - lo, (1,), generator=gen, device=device))
                    placed.append((h, pos))
        for h, pos in placed:
            qh = q[b, h]
            key = 3.0 * math.sqrt(d) * qh / qh.norm() + _randn(gen, (d,), device)
            K[b, h // G, pos] = key.to(dt)
        needle_pos.append(placed)

    lens_t = torch.tensor(lens, dtype=torch.int32, device=device)
    return Inputs(K=K, V=V, q=q.to(dt), refs=refs.to(dt), lens=lens_t, needle_pos=needle_pos)


def decode_stream(w: Workload, steps: int, device="cpu", seed_offset: int = 1000):
    """New tokens and queries for `steps` decode steps.

    Returns (k_new [steps, B, Hkv, d], v_new [steps, B, Hkv, d], q [steps, B, Hq, d]);
    new keys follow the key recipe with fresh per-chunk offsets; the queries
    are the workload's queries (those the needles were planted for) plus
    0.1 N(0, I) noise per step.
    """
    B, Hq, Hkv, d = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim
    dt = w.torch_dtype()
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed + seed_offset)
    k_new = (_randn(gen, (steps, B, Hkv, d), device)
             + _randn(gen, (1, B, Hkv, d), device, std=math.sqrt(0.5))).to(dt)
    v_new = _randn(gen, (steps, B, Hkv, d), device).to(dt)
    base = make_query_base(w, device)
    q = (base.unsqueeze(0) + 0.1 * _randn(gen, (steps, B, Hq, d), device)).to(dt)
    return k_new, v_new, q


def make_query_base(w: Workload, device="cpu") -> torch.Tensor:
    """The fp32 queries make_inputs draws first (same seed, same order)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    return _draw_queries(w, gen, device)[0]


def random_selection(n_leaves: int, G: int, frac: float, seed: int, device="cpu"):
    """A synthetic routed selection for one (sequence, KV head): sorted unique leaf
    indices and a non-zero G-bit head mask per index (each head keeps ~frac)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    bits = torch.rand((n_leaves, G), generator=gen, device=device) < frac
    weights = (1 << torch.arange(G, device=device, dtype=torch.int64))
    masks = (bits.to(torch.int64) * weights).sum(dim=1)
    idx = torch.nonzero(masks != 0).flatten()
    return idx.to(torch.int32), masks[idx].to(torch.int32)
