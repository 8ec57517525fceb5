#!/usr/bin/env python
"""Decode benchmark of the ZHA hot path on B200: one step = append the new
token to the cache and the summary tree, route every query head top-down with
top-p, and attend over the routed tokens (zha_decode), for every sequence of
the batch. Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload deep256k]
  python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Multi-GPU (torchrun): each rank decodes its own independent replica of the
workload (the path shards by sequence and KV head with no exchange), timed on
the device; the slowest rank's time is used.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/s per layer & µs/step vs context; HBM GB/s on touched bytes"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="zha", choices=["zha", "reference"])
    ap.add_argument("--workload", default="deep256k",
                    choices=["deep256k", "deep1m", "wide32k", "tiny", "small", "medium", "speed256k"])
    ap.add_argument("--refs", default="random", choices=["random", "aligned"])
    ap.add_argument("--p", type=float, default=None)
    ap.add_argument("--summary", default="native", choices=["native", "mxfp8"],
                    help="summary storage: mu in the KV dtype, or MX-FP8 (E4M3 blocks of 32 + scales)")
    ap.add_argument("--p-schedule", default="fixed", choices=["fixed", "root"],
                    help="per-level p: fixed p, or p^(1/L) at every level")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-profile", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the 1M incremental-build record and the crossover summary of the default line")
    ap.add_argument("--scorer", default="mma", choices=["tcgen05", "mma"],
                    help="node-scoring kernel: tcgen05 (tensor memory) where it applies, or mma.sync")
    ap.add_argument("--route", default="levels", choices=["levels", "fused"],
                    help="routing launches: per level (default), or one fused launch (ZHA_FLAG_FUSED_ROUTE)")
    ap.add_argument("--graph", action=argparse.BooleanOptionalAction, default=True,
                    help="replay each decode step from a captured CUDA graph (default on)")
    ap.add_argument("--sweep", action="store_true",
                    help="context sweep vs dense (deep and wide trees, random and aligned references)")
    ap.add_argument("--sweep-n", default="8192,32768,65536,131072,524288,2097152,4194304")
    ap.add_argument("--sweep-trees", default="deep,wide", help="comma list of deep, wide, speed")
    ap.add_argument("--block", default=None,
                    help="comma list of query positions per call: time zha_decode_block at each")
    ap.add_argument("--incremental", action="store_true",
                    help="build the tree by 4,096-token appends, then decode at p = 0.9, 0.95, 0.99")
    return ap.parse_args()


def workload(args):
    import dataclasses

    from tree_indexed_sparse_02_b200 import inputs as I
    w = {"deep256k": I.DEEP_256K, "deep1m": I.DEEP_1M, "wide32k": I.WIDE_32K, "tiny": I.TINY_F32,
         "speed256k": I.SPEED_256K,
         # a reduced deep-tree case (same kernels, B=1, N=64K) for detailed profiler captures
         "small": dataclasses.replace(I.DEEP_256K, name="deep N=65536 c=4 L=6 B=1", batch=1,
                                      context=65536, needles=64, diffuse_nodes=8),
         # one sequence of the 256K deep workload (a quarter of its bytes)
         "medium": dataclasses.replace(I.DEEP_256K, name="deep N=262144 c=4 L=6 B=1", batch=1)}[args.workload]
    w = dataclasses.replace(w, refs_mode=args.refs, p_schedule=args.p_schedule, summary=args.summary)
    if args.p is not None:
        w = dataclasses.replace(w, p=args.p)
    return w


# ----------------------------------------------------------------- helpers


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, enabled: bool = True):
        self.index, self.enabled, self.proc, self.path = index, enabled, None, None

    def __enter__(self):
        if not self.enabled:
            return self
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]), f[5], f[6], f[7], f[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[3 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": reasons}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "zha":
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    import torch
    if world > 1:
        torch.distributed.barrier()


def _all_reduce(x: float, world: int, op) -> float:
    import torch
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float, world: int) -> float:
    import torch
    return _all_reduce(x, world, torch.distributed.ReduceOp.MAX)


def sum_over_ranks(x: float, world: int) -> float:
    import torch
    return _all_reduce(x, world, torch.distributed.ReduceOp.SUM)


def job_throughput(tokens_local: float, ms_local: float, world: int):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    ms = max_over_ranks(ms_local, world)
    return sum_over_ranks(tokens_local, world) / (ms / 1e3), ms


def replica(w, rank: int):
    """The workload a rank decodes: the same shapes, its own seed."""
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + 1000 * rank) if rank else w


# --------------------------------------------------------------- CPU oracle


def _oracle():
    sys.path.insert(0, os.path.join(ROOT, "oracle"))
    import zha_oracle as orc
    orc.build_library()
    return orc


def oracle_batch_steps(w, inp, qs, k_new, v_new, first: int, steps: int, warmup: int = 0):
    """Time the oracle on whole-batch decode steps: for EVERY (sequence, KV
    head) group of the batch, append the step's token to the group's oracle
    tree, route its query heads and attend each over its token set -- the
    same work as one zha_decode call. Groups run concurrently on the host's
    cores (one task per group for the append and the routing, whose head loop
    the oracle spreads over its OpenMP threads; one task per query head for
    the attention); as many groups are held at once as half the free host
    memory allows (their fp64 caches and trees), the rest in later rounds,
    each round's time added to the step. Returns (seconds of each timed
    whole-batch step, threads used, sample description)."""
    import concurrent.futures as cf

    import numpy as np
    import psutil
    import torch

    orc = _oracle()
    B, Hkv, G, N, d, c = w.batch, w.n_kv_heads, w.group, w.context, w.head_dim, w.chunk
    s = 1.0 / math.sqrt(d)
    n_steps = warmup + steps
    cap = N + n_steps
    storage = "mxfp8" if w.summary == "mxfp8" else ("bf16" if w.dtype == "bf16" else "f32")
    p = oracle_p(orc, w)
    groups = [(b, g) for b in range(B) for g in range(Hkv)]
    nodes = sum(orc.level_nodes(cap, c, l) for l in range(1, w.levels + 1))
    per_group = 8 * d * (2 * cap + w.n_refs * nodes)
    at_once = max(1, min(len(groups), int(0.5 * psutil.virtual_memory().available // per_group)))
    cores = len(os.sched_getaffinity(0))
    pool = cf.ThreadPoolExecutor(max_workers=max(cores, at_once))
    step_s = [0.0] * steps
    build_s = 0.0

    def prep(bg):
        b, g = bg
        K = np.empty((cap, d))
        V = np.empty((cap, d))
        K[:N] = inp.K[b, g, :N].to("cpu", torch.float64).numpy()
        V[:N] = inp.V[b, g, :N].to("cpu", torch.float64).numpy()
        K[N:] = k_new[first:first + n_steps, b, g].to("cpu", torch.float64).numpy()
        V[N:] = v_new[first:first + n_steps, b, g].to("cpu", torch.float64).numpy()
        refs = inp.refs[g].to("cpu", torch.float64).numpy()
        q = qs[first:first + n_steps, b, g * G:(g + 1) * G].to("cpu", torch.float64).numpy()
        tree = orc.build_tree(K, refs, N, c, w.levels, s, storage=storage, cap_tokens=cap)
        return {"K": K, "V": V, "refs": refs, "q": q, "tree": tree, "route": None}

    def append_route(st, i):
        orc.tree_update(st["tree"], st["K"], st["refs"], N + i + 1)
        st["route"] = orc.route(st["tree"], st["q"][i], p)

    def attend(st, i, h):
        kept = st["route"].kept[0][h] if st["tree"].n(1) > 0 else np.zeros(0, dtype=bool)
        n = N + i + 1
        orc.attend(st["q"][i][h], st["K"], st["V"], n, s, orc.token_set(n, c, kept))

    for lo in range(0, len(groups), at_once):
        t0 = time.perf_counter()
        part = list(pool.map(prep, groups[lo:lo + at_once]))
        build_s += time.perf_counter() - t0
        for i in range(n_steps):
            t0 = time.perf_counter()
            list(pool.map(lambda st: append_route(st, i), part))
            list(pool.map(lambda a: attend(*a), [(st, i, h) for st in part for h in range(G)]))
            if i >= warmup:
                step_s[i - warmup] += time.perf_counter() - t0
        del part
    pool.shutdown()
    sample = (f"whole batch: all {len(groups)} (sequence, KV head) groups of every step (token append to the "
              f"oracle tree, routing of every query head, exact attention over each head's token set), "
              f"{steps} timed steps after {warmup} untimed, {at_once} groups held at once; oracle trees built "
              f"beforehand in {build_s:.1f} s (untimed)")
    return step_s, max(cores, orc.num_threads()), sample


def reference_arm(args, w, world, rank):
    import torch
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    from tree_indexed_sparse_02_b200.inputs import decode_stream, make_inputs
    inp = make_inputs(w, device=dev)
    k_new, v_new, qs = decode_stream(w, args.warmup + args.steps, device=dev)
    times, cores, sample = oracle_batch_steps(w, inp, qs, k_new, v_new, 0, args.steps, args.warmup)
    step_s = sum(times) / len(times)
    value = w.batch / step_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def oracle_p(orc, w):
    """Per-level p of the workload, by the oracle's own schedule rule."""
    return w.p if w.p_schedule == "fixed" else orc.depth_root_schedule(w.p, w.levels)


def config_of(w):
    return {"workload": w.name, "batch": w.batch, "context": w.context, "n_q_heads": w.n_q_heads,
            "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "chunk": w.chunk, "levels": w.levels,
            "n_refs": w.n_refs, "p": w.p, "p_schedule": w.p_schedule, "summary": w.summary, "refs": w.refs_mode,
            "needles_per_seq": w.needles,
            "l2": "flushed (256 MiB write) before every timed step, outside the timed region"}


# -------------------------------------------------------------- ZHA arm


def zha_arm(args, w, world, rank, local):
    import dataclasses

    import torch

    from tree_indexed_sparse_02_b200 import zha
    from tree_indexed_sparse_02_b200.inputs import decode_stream, make_inputs

    K_steps, W_steps = args.steps, args.warmup
    w = replica(w, rank)   # independent replica per rank
    n_total = W_steps + 2 * K_steps + (K_steps if not args.no_e2e else 0) + 1   # + the quality step
    cap = w.context + n_total + 8
    inp = make_inputs(w, device="cuda", capacity=cap)
    flags = (zha.ZHA_FLAG_TCGEN05 if args.scorer == "tcgen05" else 0) | \
        (zha.ZHA_FLAG_FUSED_ROUTE if args.route == "fused" else 0)
    cfg = zha.config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.levels, w.n_refs, w.dtype,
                     cap, flags=flags, summary=w.summary)
    buf = zha.Buffers(cfg)
    K, V, refs, lens = inp.K, inp.V, inp.refs, inp.lens
    k_new, v_new, qs = decode_stream(w, n_total, device="cuda")
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=w.torch_dtype(), device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    p = zha.p_schedule(w.p, w.levels, w.p_schedule)

    zha.tree_build(cfg, buf.tree, K, refs, lens, buf.status)
    torch.cuda.synchronize()
    buf.check_status("tree build")
    peak, peak_kind = read_peaks()
    tree_timing = build_append_timing(zha, cfg, w, K, refs, w.context, flush, peak)

    count_views = [buf.level_state(l)["count"].view(-1) for l in range(1, w.levels + 1)]
    sel_count = buf.sel["count"].view(-1)
    step_i = 0

    graph = zha.DecodeGraph(cfg, buf, K, V, refs, lens, p) if args.graph else None
    use_graph = [graph is not None]

    # A graph reads its inputs from its own buffers: a step's query and token
    # are put there before the step (as a model layer would write them there),
    # outside the timed region; direct calls take them where they are.
    def stage_step(i):
        if use_graph[0]:
            graph.stage(qs[i], k_new[i], v_new[i])

    def decode_step(i):
        if use_graph[0]:
            graph.replay()
        else:
            zha.decode(cfg, buf.tree, K, V, refs, lens, qs[i], k_new[i], v_new[i], p, buf.sel, out,
                       buf.workspace, buf.status)

    # warm-up
    for _ in range(W_steps):
        stage_step(step_i)
        decode_step(step_i)
        step_i += 1
    torch.cuda.synchronize()
    buf.check_status("warm-up")

    def timed_pass(n, hist):
        nonlocal step_i
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for j in range(n):
            flush.fill_(float(j))
            stage_step(step_i)
            ev[j][0].record(stream)
            decode_step(step_i)
            ev[j][1].record(stream)
            step_i += 1
            for l in range(w.levels):
                hist[j, l].copy_(count_views[l], non_blocking=True)
            hist[j, w.levels].copy_(sel_count, non_blocking=True)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    G_groups = w.batch * w.n_kv_heads
    hist_a = torch.zeros((K_steps, w.levels + 1, G_groups), dtype=torch.int32, device="cuda")
    barrier(world)
    torch.cuda.synchronize()
    launches0 = zha.launch_count()
    with Clocks(local, enabled=not args.no_clocks) as clk:
        times_a = timed_pass(K_steps, hist_a)
    launches = zha.launch_count() - launches0
    if graph is not None:   # replays launch the captured kernels without going through the library
        launches = graph.kernels_per_step * K_steps
    barrier(world)
    buf.check_status("timed steps")
    clocks = clk.summary()

    value, total_ms = job_throughput(float(w.batch * K_steps), sum(times_a), world)
    ms_per_step = total_ms / K_steps

    # bytes the step must move (algorithmic), from the routed counts of each step
    es = 2 if w.dtype == "bf16" else 4
    node_bytes = summary_node_bytes(w)                              # summary keys + plane offsets
    cand_bytes = node_bytes                                         # algorithmic bytes per scored node
    tok_bytes = 2 * w.head_dim * es                                 # K + V row
    h = hist_a.double().cpu()
    cand_per_step = h[:, : w.levels, :].sum(dim=(1, 2))             # all levels, all groups
    leaves_per_step = h[:, w.levels, :].sum(dim=1)
    extra_tokens = G_groups * (w.chunk + 1)                          # sink + current chunk, upper bound
    attn_tokens = leaves_per_step * w.chunk + extra_tokens
    qo_bytes = G_groups * 2 * w.group * w.head_dim * es
    touched = cand_per_step * cand_bytes + attn_tokens * tok_bytes + qo_bytes
    touched_mean = float(touched.mean())
    keys_share = float(attn_tokens.mean()) / (G_groups * (w.context + W_steps + K_steps))

    res = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K_steps,
           "warmup": W_steps, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": w.dtype, "data": "synthetic", "config": config_of(w),
           "us_per_step": ms_per_step * 1e3, "tree_build_ms": tree_timing["build"]["ms"],
           "tree_build": tree_timing["build"], "tree_append": tree_timing["append"],
           "touched_bytes_per_step": touched_mean,
           "touched_gbs": touched_mean / (ms_per_step / 1e3) / 1e9,
           "touched_frac_of_hbm": touched_mean / (ms_per_step / 1e3) / 1e9 / peak,
           "keys_attended": keys_share,
           "candidates_per_step": float(cand_per_step.mean()),
           "candidates_per_level": [float(h[:, l, :].sum(dim=1).mean()) for l in range(w.levels)],
           "attended_tokens_per_step": float(attn_tokens.mean()),
           "gpu_launches": int(launches), "cuda_graph": graph is not None, "scorer": args.scorer,
           "route": args.route, "route_run": "fused" if zha.route_fused(cfg) else "levels",
           "clocks": clocks}

    # per-kernel CUDA-event timing: a second pass of K steps, every launch bracketed
    if not args.no_profile:
        hist_b = torch.zeros_like(hist_a)
        use_graph[0] = False   # per-launch events need ordinary launches
        zha.profile_enable(True)
        times_b = timed_pass(K_steps, hist_b)
        zha.profile_enable(False)
        prof = zha.profile_read()
        buf.check_status("profiled steps")
        hb = hist_b.double().cpu()
        tot = sum(v[0] for v in prof.values())
        top = max(prof, key=lambda k: prof[k][0])
        res["kernels"] = {k: {"ms_per_step": v[0] / K_steps, "launches_per_step": v[1] / K_steps,
                              "share": v[0] / tot} for k, v in sorted(prof.items(), key=lambda kv: -kv[1][0])}
        res["profiled_ms_per_step"] = sum(times_b) / K_steps
        # algorithmic bytes of the dominant kernel over the profiled pass
        if top.startswith("score[l"):
            lvl = int(top[len("score[l"):-1])
            alg = float(hb[:, lvl - 1, :].sum()) * cand_bytes
            unit_desc = f"{cand_bytes} B per candidate node at level {lvl} (its summary record)"
        elif top == "attn_sparse":
            toks = hb[:, w.levels, :].sum() * w.chunk + K_steps * extra_tokens
            alg = float(toks) * tok_bytes
            unit_desc = f"{tok_bytes} B per attended (union) token"
        else:
            alg = None
            unit_desc = "not an HBM-streaming kernel"
        ms_top, n_top = prof[top]
        if alg is not None:
            achieved = alg / n_top / (ms_top / n_top / 1e3) / 1e9
            res["roofline"] = {"kernel": top, "bound": "hbm", "achieved": achieved, "peak": peak,
                               "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                               "traffic": traffic_for(top, alg / n_top), "bytes_per_launch": alg / n_top,
                               "unit_bytes": unit_desc, "avg_launch_ms": ms_top / n_top}
        else:
            res["roofline"] = {"kernel": top, "bound": "latency", "achieved": None, "peak": peak,
                               "unit": "GB/s", "frac": None, "traffic": None}

    # the build's own dense flash-decoding kernel on the same cache
    if not args.no_dense:
        q0 = qs[0]
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K_steps)]
        for j in range(W_steps):
            zha.dense_decode(cfg, q0, K, V, lens, out, buf.workspace, buf.status)
        for j in range(K_steps):
            flush.fill_(float(j))
            ev[j][0].record(stream)
            zha.dense_decode(cfg, q0, K, V, lens, out, buf.workspace, buf.status)
            ev[j][1].record(stream)
        torch.cuda.synchronize()
        dense_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world) / K_steps
        n_now = int(lens[0])
        dense_bytes = G_groups * n_now * tok_bytes + qo_bytes
        res["dense"] = {"us_per_step": dense_ms * 1e3, "tokens_per_s": w.batch / (dense_ms / 1e3),
                        "gbs": dense_bytes / (dense_ms / 1e3) / 1e9, "frac_of_hbm": dense_bytes / (dense_ms / 1e3) / 1e9 / peak}
        res["speedup_vs_dense"] = dense_ms / ms_per_step

    # end to end through the public call with host buffers
    if not args.no_e2e:
        qh = qs[step_i:step_i + K_steps].cpu().pin_memory()
        kh = k_new[step_i:step_i + K_steps].cpu().pin_memory()
        vh = v_new[step_i:step_i + K_steps].cpu().pin_memory()
        oh = torch.empty((K_steps,) + tuple(out.shape), dtype=out.dtype).pin_memory()
        qd, kd, vd = torch.empty_like(qs[0]), torch.empty_like(k_new[0]), torch.empty_like(v_new[0])
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K_steps)]
        barrier(world)
        for j in range(K_steps):
            flush.fill_(float(j))
            ev[j][0].record(stream)
            if graph is not None:   # host -> the graph's input buffers, replay, result -> host
                graph.q.copy_(qh[j], non_blocking=True)
                graph.k_new.copy_(kh[j], non_blocking=True)
                graph.v_new.copy_(vh[j], non_blocking=True)
                graph.graph.replay()
                oh[j].copy_(graph.out, non_blocking=True)
            else:
                qd.copy_(qh[j], non_blocking=True)
                kd.copy_(kh[j], non_blocking=True)
                vd.copy_(vh[j], non_blocking=True)
                zha.decode(cfg, buf.tree, K, V, refs, lens, qd, kd, vd, p, buf.sel, out, buf.workspace,
                           buf.status)
                oh[j].copy_(out, non_blocking=True)
            ev[j][1].record(stream)
        torch.cuda.synchronize()
        buf.check_status("e2e steps")
        e2e_value, _ = job_throughput(float(w.batch * K_steps), sum(a.elapsed_time(b) for a, b in ev), world)
        res["e2e"] = {"value": e2e_value, "unit": "tokens/s",
                      "h2d_bytes_per_step": (qd.numel() + kd.numel() + vd.numel()) * qd.element_size(),
                      "d2h_bytes_per_step": out.numel() * out.element_size()}

    # routing quality of one more (untimed) step: needle recall of every head
    # from the GPU's selection; for one sampled group, the oracle's routing of
    # the same step (boundary flips) and each head's captured softmax mass
    zha.decode(cfg, buf.tree, K, V, refs, lens, qs[step_i], k_new[step_i], v_new[step_i], p, buf.sel, out,
               buf.workspace, buf.status)
    torch.cuda.synchronize()
    buf.check_status("quality step")
    with_oracle = rank == 0 and world == 1 and not args.no_cpu_baseline
    res["routing_quality"] = routing_quality(w, inp, buf, K, refs, lens, qs[step_i], p, with_oracle)
    if "sampled_group" in res["routing_quality"]:
        sg = res["routing_quality"]["sampled_group"]
        res["routing_flips"] = {"group": sg["group"], "heads": w.group, "flips": sg["flips"],
                                "max_dist_from_p": sg["flip_dist_max"], "dists": sg["flip_dists"]}
    step_i += 1

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        times, cores, sample = oracle_batch_steps(w, inp, qs, k_new, v_new, W_steps, steps=2)
        res["cpu_baseline"] = {"value": w.batch * len(times) / sum(times), "unit": "tokens/s", "cores": cores,
                               "kind": "oracle", "sample": sample}
    # the 1M deep tree built by appends (p = 0.9, 0.95, 0.99), the headline
    # configuration with aligned references on both routes, and a bounded
    # crossover summary against the dense kernel, on this GPU only
    if rank == 0 and world == 1 and not args.no_extras:
        import dataclasses

        from tree_indexed_sparse_02_b200.inputs import DEEP_1M
        w1m = dataclasses.replace(DEEP_1M, refs_mode=w.refs_mode)
        rec = incremental_record(w1m, steps=5, warmup=3)
        res["config_1m_incremental"] = {k: rec[k] for k in ("config", "append", "per_p", "dense",
                                                            "speedup_vs_dense_p095")}
        res["selective_256k"] = selective_summary()
        res["crossover"] = crossover_summary()
    if world > 1:
        torch.distributed.barrier()
    return res


def routing_quality(w, inp, buf, K, refs, lens, q_step, p_levels, with_oracle: bool):
    """What the GPU's routing of the last decode step retrieves.

    needle_recall: share of the planted needles (each head's own; the
    diffuse heads' ones spread over many top nodes reported apart) whose leaf
    chunk that head kept. With the oracle (with_oracle): for sequence 0, KV
    head 0, the oracle routes the same step on a tree built from the same
    cache; flips are nodes kept by one side only among the candidates both
    had (followed per head down to its first flip), each with the distance of
    the oracle's running mass before it from p; captured_mass is, per head,
    the share of its dense softmax mass (exact attention over every cached
    token) that its token set holds."""
    import numpy as np
    import torch

    G, c, L = w.group, w.chunk, w.levels
    cnt = buf.sel["count"].cpu().numpy()
    idx = buf.sel["leaf_idx"].cpu().numpy()
    hmask = buf.sel["head_mask"].cpu().numpy().astype(np.uint32)

    def kept_leaf(b, h, leaf):
        kvh, j = h // G, h % G
        row = idx[b, kvh, :cnt[b, kvh]]
        k = int(np.searchsorted(row, leaf))
        return k < row.size and row[k] == leaf and (int(hmask[b, kvh, k]) >> j) & 1 == 1

    hits = {"regular": [0, 0], "diffuse": [0, 0]}
    for b, placed in enumerate(inp.needle_pos):
        for k, (h, pos) in enumerate(placed):
            kind = "regular" if k < w.needles else "diffuse"
            hits[kind][1] += 1
            hits[kind][0] += kept_leaf(b, h, pos // c)
    res = {"needle_recall": hits["regular"][0] / max(hits["regular"][1], 1), "needles": hits["regular"][1]}
    if hits["diffuse"][1]:
        res["needle_recall_diffuse"] = hits["diffuse"][0] / hits["diffuse"][1]
        res["needles_diffuse"] = hits["diffuse"][1]
    if not with_oracle:
        return res
    orc = _oracle()
    N = int(lens[0])
    s = 1.0 / math.sqrt(w.head_dim)
    storage = "mxfp8" if w.summary == "mxfp8" else ("bf16" if w.dtype == "bf16" else "f32")
    K64 = K[0, 0, :N].to("cpu", torch.float64).numpy()
    tree = orc.build_tree(K64, refs[0].to("cpu", torch.float64).numpy(), N, c, L, s, storage=storage)
    qg = q_step[0, :G].to("cpu", torch.float64).numpy()
    r = orc.route(tree, qg, p_levels)
    flips = []
    states = {l: buf.level_state(l) for l in range(1, L + 1)}
    for h in range(G):
        bit = np.uint32(1 << h)
        for level in range(L, 0, -1):
            st = states[level]
            n = int(st["count"][0, 0])
            ci = st["cand_idx"][0, 0, :n].cpu().numpy().astype(np.int64)
            cm = st["cand_mask"][0, 0, :n].cpu().numpy().astype(np.uint32)
            km = st["kept_mask"][0, 0, :n].cpu().numpy().astype(np.uint32)
            n_l = orc.level_nodes(N, c, level)
            cand_g = np.zeros(n_l, dtype=bool)
            kept_g = np.zeros(n_l, dtype=bool)
            mem = (cm & bit) != 0
            cand_g[ci[mem]] = True
            kept_g[ci[mem & ((km & bit) != 0)]] = True
            common = cand_g & r.cand[level - 1][h]
            diff = np.nonzero(common & (kept_g != r.kept[level - 1][h]))[0]
            pl = float(p_levels[level - 1])
            flips += [abs(float(r.cumb[level - 1][h][j]) - pl) for j in diff]
            if diff.size:
                break
    logits = s * (K64 @ qg.T)                         # [N, G]
    wts = np.exp(logits - logits.max(axis=0))
    wts /= wts.sum(axis=0)
    n1 = N // c
    leaves, masks = idx[0, 0, :cnt[0, 0]], hmask[0, 0, :cnt[0, 0]]
    captured = []
    for h in range(G):
        kl = np.zeros(n1, dtype=bool)
        kl[leaves[(masks >> np.uint32(h)) & 1 == 1]] = True
        captured.append(float(wts[orc.token_set(N, c, kl), h].sum()))
    res["sampled_group"] = {"group": [0, 0], "tokens": N, "flips": len(flips),
                            "flip_dist_max": max(flips) if flips else None, "flip_dists": flips,
                            "captured_mass": captured, "captured_mass_min": min(captured),
                            "captured_mass_mean": sum(captured) / len(captured)}
    return res


# The translation unit that holds each profiled kernel (with every header).
KERNEL_SOURCE = {"score": "zha_route.cu", "select": "zha_route.cu", "join": "zha_route.cu",
                 "route": "zha_route.cu", "attn": "zha_attn.cu", "tree": "zha_tree.cu"}


def traffic_for(kernel: str, alg_bytes_per_launch: float):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of the kernel's translation unit; None otherwise."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        ent = d["kernels"][kernel]
        unit = KERNEL_SOURCE[kernel.split("[")[0].split("_")[0]]
        if ent.get("source_sha") != source_sha(unit):
            return None
        return ent["dram_bytes_per_alg_byte"] * alg_bytes_per_launch
    except Exception:
        return None


def source_sha(unit: str | None = None):
    """Hash of a kernel translation unit and every header (all units when
    None), comments and blank space removed (a comment edit does not
    invalidate counters taken on the same code)."""
    import hashlib
    import re
    hsh = hashlib.sha256()
    csrc = os.path.join(ROOT, "tree_indexed_sparse_02_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith(".cuh") or (name.endswith(".cu") and (unit is None or name == unit)):
            src = open(os.path.join(csrc, name)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            src = re.sub(r"//[^\n]*", "", src)
            hsh.update(re.sub(r"\s+", " ", src).encode())
    return hsh.hexdigest()[:16]


# ------------------------------------------------- extra modes (one GPU)


def _timed_decode(zha, cfg, buf, K, V, refs, lens, qs, k_new, v_new, p, out, flush, first, n, warmup,
                  w, with_counts=True):
    """Decode steps first .. first+warmup+n; returns (ms of the n timed steps, mean
    candidates scored, mean attended tokens) with an L2 flush before each timed step."""
    import torch
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        zha.decode(cfg, buf.tree, K, V, refs, lens, qs[first + i], k_new[first + i], v_new[first + i], p,
                   buf.sel, out, buf.workspace, buf.status)
    counts = [buf.level_state(l)["count"].view(-1) for l in range(1, w.levels + 1)]
    hist = torch.zeros((n, w.levels + 1, w.batch * w.n_kv_heads), dtype=torch.int32, device="cuda")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for j in range(n):
        i = first + warmup + j
        flush.fill_(float(j))
        ev[j][0].record(stream)
        zha.decode(cfg, buf.tree, K, V, refs, lens, qs[i], k_new[i], v_new[i], p, buf.sel, out,
                   buf.workspace, buf.status)
        ev[j][1].record(stream)
        if with_counts:
            for l in range(w.levels):
                hist[j, l].copy_(counts[l], non_blocking=True)
            hist[j, w.levels].copy_(buf.sel["count"].view(-1), non_blocking=True)
    torch.cuda.synchronize()
    buf.check_status("decode steps")
    h = hist.double().cpu()
    return (sum(a.elapsed_time(b) for a, b in ev), float(h[:, :w.levels].sum(dim=(1, 2)).mean()),
            float(h[:, w.levels].sum(dim=1).mean()) * w.chunk + w.batch * w.n_kv_heads * (w.chunk + 1))


def _timed_dense(zha, cfg, buf, q, K, V, lens, out, flush, n, warmup):
    import torch
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        zha.dense_decode(cfg, q, K, V, lens, out, buf.workspace, buf.status)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for j in range(n):
        flush.fill_(float(j))
        ev[j][0].record(stream)
        zha.dense_decode(cfg, q, K, V, lens, out, buf.workspace, buf.status)
        ev[j][1].record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev) / n


def fused_levels(c: int, L: int) -> int:
    """Levels the bf16 leaf kernel computes inside one 256-key work item
    (every level whose nodes span at most 256 keys)."""
    k, span = 1, c * c
    while k < L and span <= 256:
        k, span = k + 1, span * c
    return k


def tree_update_bytes(w, n_old: int, n_now: int) -> int:
    """Algorithmic DRAM bytes of bringing every group's tree from n_old to
    n_now tokens: the keys of the chunks that complete, every node record
    written (the changed leaves and each ancestor from the first changed node
    to the level's end; a record is the summary keys, biases and each plane's
    value at its own reference), and the children records read by the levels
    above the leaf kernel's fused subtree (fused parents read their children
    from L2, just written)."""
    c, L = w.chunk, w.levels
    es = 2 if w.dtype == "bf16" else 4
    rec = summary_node_bytes(w) + 4 * w.n_refs      # + each plane's value at its own reference
    kf = fused_levels(c, L) if w.dtype == "bf16" else 1

    def nodes(n, level):
        m = n // c
        for _ in range(2, level + 1):
            m = (m + c - 1) // c
        return m

    lo, hi = n_old // c, n_now // c
    if hi <= lo:
        return 0
    total = (hi - lo) * (c * w.head_dim * es + rec)
    for level in range(2, L + 1):
        lo_c, n_c = lo, nodes(n_now, level - 1)
        lo, hi = lo // c, nodes(n_now, level)
        total += (hi - lo) * rec
        if level > kf:
            total += (min(hi * c, n_c) - lo * c) * rec
    return total * w.batch * w.n_kv_heads


def append_graph(zha, cfg, tree, K, refs, n_tokens: int, block: int, status):
    """The appends that build a tree of n_tokens tokens per sequence from
    nothing in blocks of `block` tokens (each a device-side length update and
    a zha_tree_append), captured once as a CUDA graph so that a replay times
    the device work alone (after one ordinary pass, which also sets the
    kernels' attributes outside the capture)."""
    import torch
    lens = torch.zeros((cfg.batch,), dtype=torch.int32, device="cuda")

    def appends():
        for start in range(0, n_tokens, block):
            lens.fill_(min(start + block, n_tokens))
            zha.tree_append(cfg, tree, K, refs, lens, min(block, n_tokens - start), status)

    appends()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        appends()
    graph.lens = lens
    return graph


def build_append_timing(zha, cfg, w, K, refs, lens_now: int, flush, peak, reps: int = 3, block: int = 4096):
    """Device time (CUDA events on the launching stream, L2 flushed before
    each timed run) of building the whole tree of every group at once, and of
    building it by appends of `block` tokens (replayed from a CUDA graph);
    each with its algorithmic bytes and fraction of the measured copy
    bandwidth."""
    import torch
    stream = torch.cuda.current_stream()
    tree = torch.empty(zha.tree_bytes(cfg), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lens = torch.full((w.batch,), lens_now, dtype=torch.int32, device="cuda")

    def timed(fn):
        fn()   # warm-up
        ms = []
        for _ in range(reps):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        return statistics.median(ms)

    build_ms = timed(lambda: zha.tree_build(cfg, tree, K, refs, lens, status))
    graph = append_graph(zha, cfg, tree, K, refs, lens_now, block, status)
    app_ms = timed(graph.replay)
    del graph
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"tree build/append device status {int(status.item())}")
    tokens = w.batch * lens_now
    b_bytes = tree_update_bytes(w, 0, lens_now)
    a_bytes = sum(tree_update_bytes(w, s0, min(s0 + block, lens_now)) for s0 in range(0, lens_now, block))
    out = {}
    for name, ms, by, extra in (("build", build_ms, b_bytes, {}),
                                ("append", app_ms, a_bytes, {"block_tokens": block})):
        gbs = by / (ms / 1e3) / 1e9
        out[name] = {"ms": ms, "tokens_per_s": tokens / (ms / 1e3), "alg_bytes": by,
                     "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak},
                     **extra}
    del tree
    return out


def summary_node_bytes(w):
    """Bytes of one node record: mu (KV dtype, or E4M3 + one scale byte per 32) and fp32 offsets."""
    if w.summary == "mxfp8":
        return w.n_refs * w.head_dim + w.n_refs * (w.head_dim // 32) + w.n_refs * 4
    es = 2 if w.dtype == "bf16" else 4
    return w.n_refs * w.head_dim * es + w.n_refs * 4


def _bytes(w, cand, tokens):
    es = 2 if w.dtype == "bf16" else 4
    cand_bytes = summary_node_bytes(w)
    return cand * cand_bytes + tokens * 2 * w.head_dim * es + w.batch * w.n_kv_heads * 2 * w.group * w.head_dim * es


def sweep_point(N: int, tree: str, refs_mode: str, steps: int, warmup: int, p_schedule: str = "fixed",
                summary: str = "native", route: str = "levels", workload=None):
    """ZHA decode vs the dense kernel on one identical cache of N tokens (batch
    1, 32/4 heads, d 128): the deep, wide or speed-model tree with random or
    aligned references (or the given workload). Returns one record."""
    import dataclasses

    import torch

    from tree_indexed_sparse_02_b200 import zha
    from tree_indexed_sparse_02_b200.inputs import decode_stream, make_inputs, sweep_workload
    peak, _ = read_peaks()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    w = dataclasses.replace(workload if workload is not None else sweep_workload(N, tree), refs_mode=refs_mode,
                            p_schedule=p_schedule, summary=summary)
    n, W = steps, warmup
    cap = N + n + W + 8
    inp = make_inputs(w, device="cuda", capacity=cap)
    cfg = zha.config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.levels, w.n_refs,
                     w.dtype, cap, summary=w.summary, flags=zha.ZHA_FLAG_FUSED_ROUTE if route == "fused" else 0)
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, inp.K, inp.refs, inp.lens, buf.status)
    k_new, v_new, qs = decode_stream(w, n + W, device="cuda")
    out = torch.empty_like(qs[0])
    ms, cand, toks = _timed_decode(zha, cfg, buf, inp.K, inp.V, inp.refs, inp.lens, qs, k_new, v_new,
                                   zha.p_schedule(w.p, w.levels, w.p_schedule), out, flush, 0, n, W, w)
    dense_ms = _timed_dense(zha, cfg, buf, qs[0], inp.K, inp.V, inp.lens, out, flush, n, W)
    us = ms / n * 1e3
    touched = _bytes(w, cand, toks)
    rec = {"mode": "sweep", "tree": tree, "refs": refs_mode, "route": route,
           "route_run": "fused" if zha.route_fused(cfg) else "levels", "context": N, "batch": w.batch,
           "p": w.p, "summary": w.summary,
           "p_schedule": w.p_schedule, "zha_us_per_step": us, "dense_us_per_step": dense_ms * 1e3,
           "speedup_vs_dense": dense_ms * 1e3 / us,
           "keys_attended": toks / (w.batch * w.n_kv_heads * (N + W + n)),
           "touched_gbs": touched / (us / 1e6) / 1e9,
           "touched_frac_of_hbm": touched / (us / 1e6) / 1e9 / peak,
           "dense_frac_of_hbm": (w.batch * w.n_kv_heads * N * 2 * w.head_dim * 2) / dense_ms * 1e3 / 1e9 / peak}
    del inp, buf, k_new, v_new, qs, out, flush
    torch.cuda.empty_cache()
    return rec


def sweep_mode(args):
    """Context sweep: ZHA decode vs the dense kernel on identical caches, deep and
    wide trees, random and aligned references; one JSON line per point."""
    Ns = [int(x) for x in args.sweep_n.split(",")]
    for tree in args.sweep_trees.split(","):
        for refs_mode in ("random", "aligned"):
            for N in Ns:
                print(json.dumps(sweep_point(N, tree, refs_mode, args.steps, args.warmup, args.p_schedule,
                                             args.summary, args.route)), flush=True)


def selective_summary(steps: int = 10, warmup: int = 3):
    """The headline configuration (256K deep tree, B=4) with aligned
    references -- the selective regime trained references give -- on the
    per-level and on the fused route, each against the dense kernel on the
    same cache."""
    from tree_indexed_sparse_02_b200.inputs import DEEP_256K
    rows = []
    for route in ("levels", "fused"):
        r = sweep_point(DEEP_256K.context, "deep", "aligned", steps, warmup, route=route, workload=DEEP_256K)
        rows.append({k: r[k] for k in ("route", "route_run", "zha_us_per_step", "dense_us_per_step", "speedup_vs_dense",
                                       "keys_attended", "touched_frac_of_hbm")})
        rows[-1]["tokens_per_s"] = DEEP_256K.batch / (r["zha_us_per_step"] / 1e6)
    return {"workload": DEEP_256K.name, "refs": "aligned", "steps": steps, "warmup": warmup,
            "l2": "flushed before every timed step", "points": rows}


def crossover_summary(steps: int = 5, warmup: int = 3):
    """ZHA and dense us/step at 64K, 128K and 512K tokens for the deep and wide
    trees with both reference modes, the aligned (selective) one with both
    route modes (a bounded part of the context sweep)."""
    rows = []
    for tree in ("deep", "wide"):
        for refs_mode, route in (("random", "levels"), ("aligned", "levels"), ("aligned", "fused")):
            for N in (65536, 131072, 524288):
                r = sweep_point(N, tree, refs_mode, steps, warmup, route=route)
                rows.append({k: r[k] for k in ("tree", "refs", "route", "route_run", "context", "zha_us_per_step",
                                               "dense_us_per_step", "speedup_vs_dense", "keys_attended",
                                               "touched_frac_of_hbm")})
    return {"steps": steps, "warmup": warmup, "batch": 1, "l2": "flushed before every timed step", "points": rows}


def incremental_mode(args, w):
    """The 1M deep-tree workload built by zha_tree_append in 4,096-token blocks
    (append throughput), then decode steps at p = 0.9, 0.95 and 0.99."""
    print(json.dumps(incremental_record(w, args.steps, args.warmup)), flush=True)


def incremental_record(w, steps: int, warmup: int):
    """The record of incremental_mode (one dict)."""
    import dataclasses

    import torch

    from tree_indexed_sparse_02_b200 import zha
    from tree_indexed_sparse_02_b200.inputs import decode_stream, make_inputs
    peak, peak_kind = read_peaks()
    ps = (0.9, 0.95, 0.99)
    n, W = steps, warmup
    N = w.context
    cap = N + len(ps) * (n + W) + 8
    inp = make_inputs(w, device="cuda", capacity=cap)
    cfg = zha.config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.levels, w.n_refs, w.dtype, cap,
                     summary=w.summary)
    buf = zha.Buffers(cfg)
    lens = torch.zeros_like(inp.lens)
    block = 4096
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    graph = append_graph(zha, cfg, buf.tree, inp.K, inp.refs, N, block, buf.status)
    for rep in range(2):   # an untimed replay first (each recomputes the same tree)
        flush.fill_(float(rep))
        torch.cuda.synchronize()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    buf.check_status("appends")
    append_ms = e0.elapsed_time(e1)
    lens.copy_(graph.lens)
    del graph
    k_new, v_new, qs = decode_stream(w, len(ps) * (n + W), device="cuda")
    out = torch.empty_like(qs[0])
    per_p = {}
    for k, p in enumerate(ps):
        ms, cand, toks = _timed_decode(zha, cfg, buf, inp.K, inp.V, inp.refs, lens, qs, k_new, v_new, p, out,
                                       flush, k * (n + W), n, W, w)
        us = ms / n * 1e3
        touched = _bytes(w, cand, toks)
        per_p[str(p)] = {"tokens_per_s": w.batch / (us / 1e6), "us_per_step": us,
                         "keys_attended": toks / (w.batch * w.n_kv_heads * int(lens[0])),
                         "touched_bytes_per_step": touched, "touched_gbs": touched / (us / 1e6) / 1e9,
                         "touched_frac_of_hbm": touched / (us / 1e6) / 1e9 / peak}
    dense_ms = _timed_dense(zha, cfg, buf, qs[0], inp.K, inp.V, lens, out, flush, n, W)
    main_p = per_p["0.95"]
    res = {"metric": METRIC, "value": main_p["tokens_per_s"], "unit": "tokens/s", "n_gpus": 1, "steps": n,
           "warmup": W, "ms_per_step": main_p["us_per_step"] / 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": w.dtype, "data": "synthetic", "config": config_of(w),
           "append": {"block_tokens": block, "tokens_per_s": N * w.batch / (append_ms / 1e3), "ms": append_ms,
                      "timing": "replay of a CUDA graph of the appends"},
           "per_p": per_p, "dense": {"us_per_step": dense_ms * 1e3},
           "speedup_vs_dense_p095": dense_ms * 1e3 / main_p["us_per_step"], "peak_kind": peak_kind}
    app_bytes = sum(tree_update_bytes(w, s0, min(s0 + block, N)) for s0 in range(0, N, block))
    res["append"]["alg_bytes"] = app_bytes
    res["append"]["roofline"] = {"bound": "hbm", "achieved": app_bytes / (append_ms / 1e3) / 1e9, "peak": peak,
                                 "unit": "GB/s", "frac": app_bytes / (append_ms / 1e3) / 1e9 / peak}
    del inp, buf, k_new, v_new, qs, out, flush, lens
    torch.cuda.empty_cache()
    return res


def block_mode(args, w):
    """Multi-query blocks: zha_decode_block with T query positions per sequence
    (every summary and KV read shared by the T * G query rows of a group),
    against T single-query zha_decode steps on the same cache; one JSON line per T."""
    import torch

    from tree_indexed_sparse_02_b200 import zha
    from tree_indexed_sparse_02_b200.inputs import decode_stream, make_inputs
    Ts = [int(x) for x in args.block.split(",")]
    n, W = args.steps, args.warmup
    N = w.context
    steps_tokens = (n + W) * max(Ts)
    cap = N + len(Ts) * 2 * steps_tokens + 8
    inp = make_inputs(w, device="cuda", capacity=cap)
    cfg = zha.config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.levels, w.n_refs, w.dtype, cap,
                     summary=w.summary, queries=max(Ts))
    buf = zha.Buffers(cfg)
    zha.tree_build(cfg, buf.tree, inp.K, inp.refs, inp.lens, buf.status)
    p = zha.p_schedule(w.p, w.levels, w.p_schedule)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    # queries and new tokens from the workload's decode stream (aligned mode: near the references)
    k_s, v_s, q_s = decode_stream(w, max(Ts), device="cuda")

    def timed(call, reps):
        for _ in range(W):
            call()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for j in range(reps):
            flush.fill_(float(j))
            ev[j][0].record(stream)
            call()
            ev[j][1].record(stream)
        torch.cuda.synchronize()
        buf.check_status("block steps")
        return sum(a.elapsed_time(b) for a, b in ev) / reps

    for T in Ts:
        q = q_s[:T].transpose(0, 1).contiguous()          # [B, T, Hq, d]
        kn = k_s[:T].transpose(0, 1).contiguous()
        vn = v_s[:T].transpose(0, 1).contiguous()
        out = torch.empty_like(q)
        call = lambda: zha.decode_block(cfg, T, buf.tree, inp.K, inp.V, inp.refs, inp.lens, q, kn, vn, p,  # noqa: E731
                                        buf.sel, out, buf.workspace, buf.status)
        blk_ms = timed(call, n)
        zha.profile_enable(True)
        call()
        torch.cuda.synchronize()
        zha.profile_enable(False)
        kern = {k: round(v[0] * 1e3, 1) for k, v in zha.profile_read().items()}
        q1, k1, v1 = q[:, 0].contiguous(), kn[:, 0].contiguous(), vn[:, 0].contiguous()
        o1 = torch.empty_like(q1)
        one_ms = timed(lambda: zha.decode(cfg, buf.tree, inp.K, inp.V, inp.refs, inp.lens, q1, k1, v1, p, buf.sel,
                                          o1, buf.workspace, buf.status), n)
        print(json.dumps({"mode": "block", "workload": w.name, "refs": w.refs_mode, "summary": w.summary,
                          "queries_per_call": T, "us_per_call": blk_ms * 1e3,
                          "tokens_per_s": w.batch * T / (blk_ms / 1e3),
                          "single_query_us_per_step": one_ms * 1e3,
                          "single_query_tokens_per_s": w.batch / (one_ms / 1e3),
                          "speedup_vs_single_query": (one_ms * T) / blk_ms, "kernels_us": kern,
                          "l2": "flushed (256 MiB write) before every timed call"}), flush=True)


def main():
    args = parse()
    w = workload(args)
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        reference_arm(args, w, world, rank)
        return
    if args.sweep:
        sweep_mode(args)
        return
    if args.incremental:
        incremental_mode(args, w)
        return
    if args.block:
        block_mode(args, w)
        return
    res = zha_arm(args, w, world, rank, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
