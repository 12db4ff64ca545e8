#!/usr/bin/env python
"""Benchmark of the ZHA decode hot path on one B200 per process.

One step = one decode step over a batch of walks: append one key and one value
to every tree (making nodes as chunks fill), walk every query down its tree
(top-p 0.9), and attend over exactly the chosen keys. The trees are built once
before timing (reported separately). Metric: queries (walks) per second.

Workload (N=1 headline): 16 sequences x 4 KV heads x 262,144 keys, 16 query heads
(GQA 4:1), d = 128, bf16 K/V, chunk 8, 6 levels, R = 8 reference queries, top-p
0.9, one query per head: 256 walks per step; clustered synthetic keys (blocks of
64 around N(0, I) centres, noise 0.3), queries mixing 1-8 centres. Also reported:
the 1,048,576-key workload (8 x 8 KV heads, 32 query heads, chunk 16, 5 levels,
top-p 0.9 and top-K 16) with the full-scan indexer and the chunk-mass profile of
dense attention on the same trees, and the prefill workload (4,096 queries x 16
query heads against one sequence's four 262,144-key trees, scored on the tensor
cores).

Under torchrun each rank runs its own copy of the workload (distinct seeds) on its
GPU: weak scaling, no data-path collective; time = max over ranks.

`--impl reference` times the CPU oracle instead (rank 0 only), on a bounded
sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ZHA decode queries/s (search+attend) at 262K and 1M keys; HBM GB/s vs peak"
LABEL_256K = "kv256k decode: 16 seq x 4 KV heads x 262,144 keys, 16 q-heads, d=128, bf16, C=8, depth 6, R=8"
UNIT = "queries/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="skip the 1M-key workload")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="time budget of the oracle baseline")
    ap.add_argument("--profile-steps", type=int, default=20)
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--batch", type=int, default=0, help="sequences per GPU (default: the workload's)")
    ap.add_argument("--prefill-only", action="store_true",
                    help="time only the prefill workload and print its line (for profiling)")
    ap.add_argument("--build-only", action="store_true",
                    help="build the 256K workload's trees (--batch sequences), time zha_rebuild, print its line")
    ap.add_argument("--parity-trees", type=int, default=4,
                    help="trees per workload whose walks the CPU leg checks against the oracle (0: none)")
    ap.add_argument("--prefill-queries", type=int, default=0,
                    help="queries per query head of the prefill workload (default: the workload's 4,096)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def committed_traffic(kernel: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if the kernel's source
    has not changed since it was taken."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "tree_indexed_sparse_append_b200", "csrc", "zha_search.cu" if kernel == "score"
                       else "zha_attend.cu")
    try:
        with open(path) as f:
            rec = json.load(f)[f"{kernel}:{workload}"]
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
        return rec["dram_bytes_per_launch"] if rec.get("source_sha") == sha else None
    except Exception:
        return None


class Clocks:
    """nvidia-smi sampler running while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.index), "-lms", "50"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc:
            time.sleep(0.2)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        mhz, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(mhz)}


# ---------------------------------------------------------------------------
def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest value over the ranks (the slowest rank's time); no-op at world 1."""
    if world <= 1:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(walks_per_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job queries/s: every rank ran `steps` steps of `walks_per_step` walks;
    the job took as long as its slowest rank."""
    return walks_per_step * steps * world / (max_ms / 1e3)


CPU_TREES = 4  # trees of the 256K workload the CPU oracle legs sample


def build_roofline(w, tree, flush, st, elt: int):
    """Device time of the build kernels alone (zha_rebuild over the existing node
    storage: no allocation), and their achieved bandwidth: per tree, the level-1
    build reads the keys of its full chunks (C * d * elt per node), every level
    writes its nodes (4 * NF bytes each) and every level above 1 reads its
    children (C nodes each)."""
    import torch

    for _ in range(2):
        tree.rebuild()
    ts = []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(5):
        flush.zero_()
        e0.record(st)
        tree.rebuild()
        e1.record(st)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    ms = sorted(ts)[len(ts) // 2]
    sizes = tree.level_sizes()
    NF = w.R * w.d + ((w.R + 3) & ~3)
    read = sizes[1] * w.chunk * w.d * elt + sum(sizes[l] * w.chunk * NF * 4 for l in range(2, len(sizes)))
    write = sum(sizes[l] * NF * 4 for l in range(1, len(sizes)))
    nbytes = w.trees * (read + write)
    peak, kind = peaks()
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"ms": ms, "keys_per_s": w.trees * sizes[0] / (ms / 1e3), "levels": len(sizes) - 1,
            "timing": "CUDA events around zha_rebuild (the build kernels over the existing node storage; "
                      "allocation excluded), median of 5, L2 flushed before each",
            "roofline": {"bound": "hbm", "kernel": "build_nodes", "achieved": gbs, "peak": peak, "unit": "GB/s",
                         "frac": gbs / peak, "peak_source": kind, "bytes_per_build": nbytes,
                         "launches": len(sizes) - 1, "traffic": None}}


def learn_step(w, tree, inp, st, steps: int = 3, lr: float = 0.05):
    """One step of learning the reference queries (the split-loss gradient, an
    in-place update of the references, and the rebuild of every level), timed on
    the device over `steps` steps after one untimed step."""
    import torch

    losses = []

    def one():
        loss, grad = tree.ref_grad(inp.Q)
        inp.refs.sub_(lr * grad)
        tree.rebuild()
        return loss

    losses.append(float(one().item()))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        loss = one()
    e1.record(st)
    torch.cuda.synchronize()
    losses.append(float(loss.item()))
    tree.sync_status()
    return {"ms_per_step": e0.elapsed_time(e1) / steps, "steps": steps, "lr": lr, "walks": w.walks,
            "step": "zha_ref_grad + refs -= lr * grad + zha_rebuild", "loss_first": losses[0],
            "loss_last": losses[-1]}


def oracle_walks_per_second(w, trees, seconds: float, cores: int):
    """Oracle (CPU) append + search + attend over the sampled trees' walks,
    repeated for about `seconds`; returns (queries/s, walks timed)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle as O

    jobs = []
    for key, (ot, K, V, qs) in trees.items():
        for q in qs:
            jobs.append((ot, K, V, q))

    def one(job):
        ot, K, V, q = job
        wk = O.search(ot, q, O.TOP_P, 0.9, 0, w.top_width)
        O.attend(K[: ot.n_keys], V[: ot.n_keys], q, wk.sel, w.chunk, ot.n_nodes[1], w.beta)
        return 1

    done = 0
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=cores) as ex:
        while time.perf_counter() - t0 < seconds:
            for key, (ot, K, V, qs) in trees.items():
                if ot.n_keys < K.shape[0]:
                    O.append(ot, K, 1)
            done += sum(ex.map(one, jobs))
    return done / (time.perf_counter() - t0), done


def oracle_sample(w, inp, n_trees: int, threads: int):
    """Host copies + oracle trees of the first n_trees trees of the workload."""
    import numpy as np

    import oracle as O

    group = w.n_q_heads // w.n_kv_heads
    out = {}
    for t in range(n_trees):
        b, h = divmod(t, w.n_kv_heads)
        K = inp.K[b, h].double().cpu().numpy()
        V = inp.V[b, h].double().cpu().numpy()
        ot = O.build_tree(K[: w.n_keys], inp.refs[h].double().cpu().numpy(), w.chunk, w.depth, w.beta,
                          threads=threads, capacity=K.shape[0])
        qs = [inp.Q[b, hq, i].double().cpu().numpy() for hq in range(h * group, (h + 1) * group)
              for i in range(w.queries_per_head)]
        out[(b, h)] = (ot, np.ascontiguousarray(K), np.ascontiguousarray(V), qs)
    return out


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_parity_sample(w, inp, tree, sample_trees, modes, threads: int, label: str):
    """The CPU leg's check of the measured configuration: the oracle built over
    the sampled trees at the keys the GPU trees hold now (appends included), every
    walk of those trees searched and attended on the GPU (the call the bench
    times) and by the oracle. Reports, per mode: walks compared, walks whose set
    equals the oracle's, walks that part at an oracle near-tie (each must be an
    admissible walk, see oracle.ties) and oracle near-ties met, the largest
    attention error against the oracle's attention over the GPU's selection, keys
    read and the share of the dense attention the chosen keys hold (kept mass)."""
    import numpy as np
    import torch

    import oracle as O
    from oracle import ties as OT
    import tree_indexed_sparse_append_b200 as Z

    n = tree.n_keys
    group = w.n_q_heads // w.n_kv_heads
    per_mode = {}
    gpu = {}
    for mname, p, k in modes:
        mode = Z.TOP_P if mname == "top_p" else Z.TOP_K
        sel, cnt, _ = tree.search(inp.Q, mode, p, k)
        out, lse = tree.attend(inp.Q, sel, cnt, out_dtype=torch.float32)
        tree.sync_status()
        gpu[mname] = (sel.cpu().numpy(), cnt.cpu().numpy(), out.double().cpu().numpy().reshape(w.walks, w.d),
                      lse.double().cpu().numpy())
        per_mode[mname] = {"walks": 0, "identical": 0, "near_tie_partings": 0, "oracle_near_ties": 0,
                           "max_attention_err": 0.0, "keys_read": [], "kept_mass": []}
    t0 = time.perf_counter()
    for b, h in sample_trees:
        K = inp.K[b, h, :n].double().cpu().numpy()
        V = inp.V[b, h, :n].double().cpu().numpy()
        ot = O.build_tree(K, inp.refs[h].double().cpu().numpy(), w.chunk, w.depth, w.beta, threads=threads)
        for mname, p, k in modes:
            mode = O.TOP_P if mname == "top_p" else O.TOP_K
            sel, cnt, out, lse = gpu[mname]
            r = per_mode[mname]
            for hq in range(h * group, (h + 1) * group):
                for i in range(w.queries_per_head):
                    wi = (b * w.n_q_heads + hq) * w.queries_per_head + i
                    q = inp.Q[b, hq, i].double().cpu().numpy()
                    ow = O.search(ot, q, mode, p, k, w.top_width)
                    g = sel[wi, : cnt[wi]]
                    r["walks"] += 1
                    near = min(ow.tie_gap, ow.tie_sum) < OT_TOL
                    r["oracle_near_ties"] += int(near)
                    if np.array_equal(g, ow.sel):
                        r["identical"] += 1
                    elif near and tuple(int(x) for x in g) in OT.admissible_selections(ot, q, mode, p, k,
                                                                                       w.top_width, OT_TOL):
                        r["near_tie_partings"] += 1
                    o_out, o_lse = O.attend(K, V, q, g, w.chunk, ot.n_nodes[1], w.beta)
                    err = max(float(np.max(np.abs(out[wi] - o_out) / np.maximum(1.0, np.abs(o_out)))),
                              abs(lse[wi] - o_lse) / max(1.0, abs(o_lse)))
                    r["max_attention_err"] = max(r["max_attention_err"], err)
                    r["keys_read"].append(w.chunk * len(g) + (n - w.chunk * ot.n_nodes[1]))
                    r["kept_mass"].append(O.kept_mass(K, q, w.beta, g, w.chunk, ot.n_nodes[1]))
        del K, V, ot
    res = {}
    for mname, r in per_mode.items():
        kr, km = np.array(r["keys_read"]), np.array(r["kept_mass"])
        res[mname] = {"walks": r["walks"], "identical": r["identical"],
                      "near_tie_partings": r["near_tie_partings"],
                      "invalid": r["walks"] - r["identical"] - r["near_tie_partings"],
                      "near_tie_share": r["near_tie_partings"] / max(1, r["walks"]),
                      "oracle_near_ties": r["oracle_near_ties"],
                      "max_attention_err": r["max_attention_err"],
                      "keys_read_mean": float(kr.mean()), "keys_read_median": float(np.median(kr)),
                      "kept_mass_mean": float(km.mean()), "kept_mass_median": float(np.median(km)),
                      "kept_mass_min": float(km.min())}
    return {"workload": label, "keys": n, "trees": [list(x) for x in sample_trees], "tie_tol": OT_TOL,
            "seconds": time.perf_counter() - t0, "modes": res}


OT_TOL = 1e-5  # relative near-tie tolerance (the method's selection target)


# ---------------------------------------------------------------------------
def run_decode(w, args, rank, world, dev, with_baseline: bool, label: str, modes, with_dense: bool = False):
    import torch

    import synthetic as S
    import tree_indexed_sparse_append_b200 as Z

    steps, warmup = args.steps, args.warmup
    need = len(modes) * (warmup + steps + args.profile_steps) + args.e2e_steps + 8
    w = S.scaled(w, seed=w.seed + 7919 * rank, appends=max(w.appends, need))
    inp = S.draw(w, device="cuda")
    st = torch.cuda.current_stream()
    torch.cuda.synchronize()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tree = Z.Tree(inp.K, inp.V, inp.refs, w.n_keys, w.chunk, w.depth, w.beta, w.top_width)
    torch.cuda.synchronize()
    B, H, cap, d = inp.K.shape
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)  # 256 MB > L2
    build = build_roofline(w, tree, flush, st, inp.K.element_size())

    new_k = inp.K[:, :, w.n_keys:].permute(2, 0, 1, 3).contiguous()
    new_v = inp.V[:, :, w.n_keys:].permute(2, 0, 1, 3).contiguous()
    Wk = w.walks
    max_sel = cap // w.chunk
    sel = torch.empty(Wk, max_sel, dtype=torch.int32, device=dev)
    cnt = torch.empty(Wk, dtype=torch.int32, device=dev)
    out = torch.empty_like(inp.Q, dtype=inp.K.dtype)
    lse = torch.empty(Wk, dtype=torch.float32, device=dev)
    tree.reserve(Wk, max_sel)
    pos = [0]

    def step(mode, p, k):
        tree.append(new_k[pos[0]], new_v[pos[0]])
        pos[0] += 1
        tree.search(inp.Q, mode, p, k, max_sel=max_sel, out=(sel, cnt, None))
        tree.attend(inp.Q, sel, cnt, out=out, lse=lse)

    results = {}
    for mi, (mname, p, k) in enumerate(modes):
        mode = Z.TOP_P if mname == "top_p" else Z.TOP_K
        for _ in range(warmup):
            step(mode, p, k)
        tree.sync_status()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        launches0 = Z.kernel_launches()
        with Clocks(int(os.environ.get("LOCAL_RANK", 0))) as clk:
            for i in range(steps):
                flush.zero_()
                evs[i][0].record(st)
                step(mode, p, k)
                evs[i][1].record(st)
            torch.cuda.synchronize()
        launches = Z.kernel_launches() - launches0
        tree.sync_status()
        total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, dev)
        if world > 1:
            torch.distributed.barrier()
        qps = job_throughput(Wk, steps, world, total_ms)

        # profiled pass: per-kernel device time and the frontier sizes behind it
        tree.profile(True)
        kt = {}
        score_bytes = attend_bytes = walk_keys = walk_nodes = 0
        levels = w.depth
        NF = w.R * w.d + ((w.R + 3) & ~3)
        for i in range(args.profile_steps):
            flush.zero_()
            step(mode, p, k)
            info = tree.last_search_info()
            levels = info["start_level"]
            score_bytes += sum(info["union_nodes"][1:levels + 1]) * NF * 4 + levels * Wk * d * 4
            # attend: the union, per tree, of the keys its walks read (K and V rows)
            c = cnt.cpu().numpy()
            sl = sel.cpu().numpy()
            G = Wk // (B * H)
            tail = tree.n_keys - w.chunk * tree.level(1)[1]
            keys = 0
            import numpy as np
            for t in range(B * H):
                chunks = np.unique(np.concatenate([sl[t * G + g, : c[t * G + g]] for g in range(G)]))
                keys += chunks.size * w.chunk + tail
            elt = 2 if w.kv_dtype == "bf16" else 4
            attend_bytes += keys * 2 * d * elt + Wk * d * (elt + 4)
            walk_keys += int(c.sum()) * w.chunk + Wk * tail
            walk_nodes += sum(info["walk_nodes"][1:levels + 1])
        for name, (n, ms) in tree.profile_read().items():
            kt[name] = {"launches": n, "ms": ms}
        tree.profile(False)
        # the selector against its fixed cost: the same searches at top-K 1, where
        # every frontier below the start level holds C nodes (search only)
        tree.profile(True)
        n_floor = 5
        for _ in range(n_floor):
            flush.zero_()
            tree.search(inp.Q, Z.TOP_K, 0.0, 1, max_sel=max_sel, out=(sel, cnt, None))
        floor_ms = tree.profile_read()["select"][1] / n_floor
        tree.profile(False)
        peak, peak_kind = peaks()
        sc = kt["score"]
        score_gbs = score_bytes / (sc["ms"] / 1e3) / 1e9 if sc["ms"] else None
        ap = kt["attend_partial"]
        attend_gbs = attend_bytes / (ap["ms"] / 1e3) / 1e9 if ap["ms"] else None
        per_launch = score_bytes / max(1, sc["launches"])
        roof = {"bound": "hbm", "kernel": "score_level", "achieved": score_gbs, "peak": peak, "unit": "GB/s",
                "frac": score_gbs / peak if score_gbs else None, "peak_source": peak_kind,
                "bytes_per_launch": per_launch, "launch_ms": sc["ms"] / max(1, sc["launches"]),
                "traffic": committed_traffic("score", label)}
        attend_roof = {"bound": "hbm", "kernel": "attend_partial", "achieved": attend_gbs, "peak": peak,
                       "unit": "GB/s", "frac": attend_gbs / peak if attend_gbs else None,
                       "bytes_per_launch": attend_bytes / max(1, ap["launches"]),
                       "launch_ms": ap["ms"] / max(1, ap["launches"]), "traffic": committed_traffic("attend", label)}
        step_ms = sum(v["ms"] for v in kt.values()) / max(1, args.profile_steps)
        keys_per_walk = walk_keys / max(1, args.profile_steps * Wk)
        sel_ms = kt["select"]["ms"] / max(1, args.profile_steps)
        nodes_step = walk_nodes / max(1, args.profile_steps)
        select = {"bound": "latency", "ms_per_step": sel_ms, "levels": levels,
                  "floor_ms_per_step": floor_ms, "frontier_ms_per_step": sel_ms - floor_ms,
                  "walk_nodes_per_step": nodes_step, "score_bytes_per_step": 4 * nodes_step,
                  "what": "floor: the same trees and queries at top-K 1 (frontiers below the start level C "
                          "nodes wide), the selector's fixed cost over the levels; frontier_ms: the rest, "
                          "which grows with the widest frontier of each level; score bytes: 4 B per "
                          "frontier node of every walk, read from L2-resident score rows"}
        results[mname] = {"qps": qps, "ms_per_step": total_ms / steps, "launches": launches / steps,
                          "keys_per_walk": keys_per_walk, "selected_keys_per_s": qps * keys_per_walk,
                          "context_keys_per_s": qps * tree.n_keys,
                          "clocks": clk.summary(), "roofline": roof, "attend_roofline": attend_roof,
                          "select": select,
                          "kernel_ms_per_step": {kk: v["ms"] / max(1, args.profile_steps) for kk, v in kt.items()},
                          "kernel_sum_ms_per_step": step_ms, "levels_walked": levels}

    # the full-scan indexer on the same trees (the comparison the 1M workload asks for)
    dense = None
    if with_dense:
        dense = {}
        max_sel_d = tree.n_keys
        dsel = torch.empty(Wk, max_sel_d, dtype=torch.int32, device=dev)
        dcnt = torch.empty(Wk, dtype=torch.int32, device=dev)
        for mname, p, k in modes:
            mode = Z.TOP_P if mname == "top_p" else Z.TOP_K
            for _ in range(3):
                tree.dense_scan(inp.Q, mode, p, k, max_sel=max_sel_d, out=(dsel, dcnt))
            ts = []
            for _ in range(10):
                flush.zero_()
                e0.record(st)
                tree.dense_scan(inp.Q, mode, p, k, max_sel=max_sel_d, out=(dsel, dcnt))
                e1.record(st)
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1))
            tree.sync_status()
            ms = sorted(ts)[len(ts) // 2]
            tree.profile(True)
            flush.zero_()
            tree.dense_scan(inp.Q, mode, p, k, max_sel=max_sel_d, out=(dsel, dcnt))
            dk = {kk: round(v[1], 4) for kk, v in tree.profile_read().items() if v[0]}
            tree.profile(False)
            kbytes = B * H * tree.n_keys * d * inp.K.element_size()
            r = results[mname]
            search_ms = sum(r["kernel_ms_per_step"][k2] for k2 in ("search_init", "score", "select", "score_tc"))
            # the full-scan scorer against its own roofline: every key read once per
            # tree, every walk's score written once (4 B)
            peak, peak_kind = peaks()
            sbytes = kbytes + Wk * tree.n_keys * 4
            score_ms = dk.get("score")
            roof_ms = sbytes / (peak * 1e9) * 1e3
            dense[mname] = {"ms": ms, "key_read_gbs": kbytes / (ms / 1e3) / 1e9, "kernel_ms": dk,
                            "keys_selected_mean": float(dcnt.float().mean().item()),
                            "tree_search_ms": search_ms, "dense_over_tree_search": ms / search_ms,
                            "score_roofline": {"bound": "hbm", "kernel": "dense_score", "achieved":
                                               sbytes / (score_ms / 1e3) / 1e9 if score_ms else None,
                                               "peak": peak, "unit": "GB/s", "frac": sbytes / (score_ms / 1e3) / 1e9 /
                                               peak if score_ms else None, "peak_source": peak_kind,
                                               "bytes_per_launch": sbytes},
                            "score_at_roofline_ms": roof_ms,
                            "score_at_roofline_over_tree_search": roof_ms / search_ms,
                            "what": "score_at_roofline_ms: the full scan's key reads and score writes at the "
                                    "measured HBM peak, its selection not counted"}
        del dsel, dcnt
        # chunk-mass profile of the same dense attention: per walk, the fewest
        # 16-key chunks holding 90% of it (the statistic the pages quote for real
        # models at about 64K tokens; these keys are synthetic)
        group = 16
        n_chunks = (tree.n_keys + group - 1) // group
        csel = torch.empty(Wk, n_chunks, dtype=torch.int32, device=dev)
        ccnt = torch.empty(Wk, dtype=torch.int32, device=dev)
        for _ in range(3):
            tree.chunk_mass(inp.Q, group, 0.9, max_sel=n_chunks, out=(csel, ccnt))
        ts = []
        for _ in range(10):
            flush.zero_()
            e0.record(st)
            tree.chunk_mass(inp.Q, group, 0.9, max_sel=n_chunks, out=(csel, ccnt))
            e1.record(st)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        tree.sync_status()
        share = ccnt.float() / n_chunks
        dense["chunk_mass"] = {"group": group, "p": 0.9, "n_chunks": n_chunks, "ms": sorted(ts)[len(ts) // 2],
                               "share_median": float(share.median().item()),
                               "share_p10": float(share.quantile(0.1).item()),
                               "share_p90": float(share.quantile(0.9).item())}
        del csel, ccnt

    # end to end through the public API with host buffers
    mname, p, k = modes[0]
    mode = Z.TOP_P if mname == "top_p" else Z.TOP_K
    Qh = inp.Q.cpu().pin_memory()
    kh = new_k.cpu().pin_memory()
    vh = new_v.cpu().pin_memory()
    Qd = torch.empty_like(inp.Q)
    kd = torch.empty_like(new_k[0])
    vd = torch.empty_like(new_v[0])
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_h = torch.empty(Wk, dtype=torch.float32).pin_memory()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.perf_counter()
    ea.record(st)
    for i in range(args.e2e_steps):
        Qd.copy_(Qh, non_blocking=True)
        kd.copy_(kh[pos[0]], non_blocking=True)
        vd.copy_(vh[pos[0]], non_blocking=True)
        tree.append(kd, vd)
        pos[0] += 1
        tree.search(Qd, mode, p, k, max_sel=max_sel, out=(sel, cnt, None))
        tree.attend(Qd, sel, cnt, out=out, lse=lse)
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)
    eb.record(st)
    torch.cuda.synchronize()
    wall_ms = max_over_ranks((time.perf_counter() - wall0) * 1e3, world, dev)
    e2e_ms = max_over_ranks(ea.elapsed_time(eb), world, dev)
    elt = inp.K.element_size()
    e2e = {"value": job_throughput(Wk, args.e2e_steps, world, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": Qd.numel() * Qd.element_size() + 2 * kd.numel() * elt,
           "d2h_bytes_per_step": out.numel() * out.element_size() + lse.numel() * 4,
           "timing": "CUDA events on the launching stream",
           "wall_value": job_throughput(Wk, args.e2e_steps, world, wall_ms),
           "wall_timing": "host clock around the same loop, through the final synchronize"}

    baseline = parity = None
    if rank == 0:
        cores = os.cpu_count() or 1
        if with_baseline:
            n_trees = CPU_TREES
            tb = time.perf_counter()
            sample = oracle_sample(w, inp, n_trees, cores)
            build_s = time.perf_counter() - tb
            walks = sum(len(v[3]) for v in sample.values())
            used = min(cores, walks)
            v, done = oracle_walks_per_second(w, sample, args.cpu_seconds, used)
            v1, done1 = oracle_walks_per_second(w, sample, max(1.0, args.cpu_seconds / 4), 1)
            baseline = {"value": v, "unit": UNIT, "cores": used, "cpu_model": cpu_model(), "kind": "oracle",
                        "single_thread": {"value": v1, "walks": done1},
                        "sample": f"{n_trees} of {w.trees} trees ({walks} walks), append + search + attend per "
                                  f"step, {done} walks in {args.cpu_seconds:.0f} s, oracle trees built beforehand",
                        "oracle_build_s": build_s,
                        "oracle_build_keys_per_s": n_trees * w.n_keys / build_s}
            del sample
        if args.parity_trees:
            sample_trees = [(i * w.batch // args.parity_trees, (i * 3) % w.n_kv_heads)
                            for i in range(args.parity_trees)]
            parity = cpu_parity_sample(w, inp, tree, sample_trees, modes, cores, label)
    learn = learn_step(w, tree, inp, st) if with_baseline else None
    n_after = tree.n_keys
    tree.close()
    del inp, new_k, new_v, flush
    torch.cuda.empty_cache()
    return {"w": w, "results": results, "e2e": e2e, "build": build, "baseline": baseline,
            "n_keys_after": n_after, "dense": dense, "parity": parity, "learn": learn}


def run_prefill(args, dev):
    """Search + attend of the prefill workload (4,096 queries per query head against
    one sequence's 262,144-key trees), timed on the device; no append."""
    import torch

    import synthetic as S
    import tree_indexed_sparse_append_b200 as Z

    w = S.WORKLOADS["prefill256k"]
    if getattr(args, "prefill_queries", 0):
        w = S.scaled(w, queries_per_head=args.prefill_queries)
    inp = S.draw(w, device="cuda")
    st = torch.cuda.current_stream()
    tree = Z.Tree(inp.K, inp.V, inp.refs, w.n_keys, w.chunk, w.depth, w.beta, w.top_width)
    Wk = w.walks
    max_sel = tree.level(1)[1]
    sel = torch.empty(Wk, max_sel, dtype=torch.int32, device=dev)
    cnt = torch.empty(Wk, dtype=torch.int32, device=dev)
    out = torch.empty_like(inp.Q, dtype=inp.K.dtype)
    lse = torch.empty(Wk, dtype=torch.float32, device=dev)
    tree.reserve(Wk, max_sel)

    def step():
        tree.search(inp.Q, Z.TOP_P, 0.9, 0, max_sel=max_sel, out=(sel, cnt, None))
        tree.attend(inp.Q, sel, cnt, out=out, lse=lse)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    ts = []
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        step()
        e1.record(st)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    ms = sorted(ts)[len(ts) // 2]
    tree.profile(True)
    step()
    info = tree.last_search_info()
    kt = {k: round(v[1], 4) for k, v in tree.profile_read().items() if v[0]}
    tree.profile(False)
    tree.sync_status()
    walk_nodes = sum(info["walk_nodes"][1:info["start_level"] + 1])
    flops = 2.0 * w.R * w.d * walk_nodes
    # levels scored on the tensor cores (trees of >= 1,024 bf16 walks, d = 128), each
    # fp32 key taken as three bf16 parts: levels of <= 8,192 nodes as the dense
    # contraction (every walk x node x reference), larger levels sparsely (counted
    # as the frontier pairs they must score)
    G = Wk // (w.batch * w.n_kv_heads)
    rp = 1
    while rp < w.R:
        rp *= 2
    sizes = tree.level_sizes()
    tc_ops = 0.0
    if G >= 1024 and w.d == 128 and inp.Q.dtype == torch.bfloat16:
        for l, n in enumerate(sizes[1:], start=1):
            if l > info["start_level"] or n == 0:
                continue
            if n <= 8192:
                tc_ops += 2.0 * Wk * n * rp * w.d * 3
            elif w.R > 2:
                tc_ops += 2.0 * info["walk_nodes"][l] * rp * w.d * 3
    tc_ms = kt.get("score_tc")
    bf16_peak = None
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16_peak = float(json.load(f)["bf16_tflops"])
    except Exception:
        pass
    tensor = None
    if tc_ms and tc_ops:
        ach = tc_ops / (tc_ms / 1e3) / 1e12
        tensor = {"bound": "tensor", "kernel": "score_tc", "achieved": ach, "peak": bf16_peak, "unit": "TFLOP/s",
                  "frac": ach / bf16_peak if bf16_peak else None, "peak_source": "measured (burst)",
                  "ops_per_step": tc_ops, "ms_per_step": tc_ms}
    # tensor-core attention (trees of >= 1,024 bf16 walks): per (walk, 128-key tile)
    # pair the max pass and the accumulate pass each take S = QK^T (2 * 128 * 128
    # flops per walk row), and P V is taken on the hi and lo parts of P (2 x the same)
    cpt = 128 // w.chunk
    pairs = 0
    for r0 in range(0, Wk, 4096):
        sl, cn = sel[r0:r0 + 4096], cnt[r0:r0 + 4096]
        tl = torch.div(sl, cpt, rounding_mode="floor")
        valid = torch.arange(sl.shape[1], device=sl.device)[None, :] < cn[:, None]
        first = valid[:, :1] & (cn[:, None] > 0)
        new = (tl[:, 1:] != tl[:, :-1]) & valid[:, 1:]
        pairs += int(first.sum().item()) + int(new.sum().item())
    tail = tree.n_keys - w.chunk * tree.level(1)[1]
    if tail > 0:
        pairs += Wk  # every walk reads the tile holding the tail
    att_ms = kt.get("attend_partial", 0.0)
    att_flops = pairs * 4 * 2.0 * 128 * 128
    keys = int(cnt.long().sum().item()) * w.chunk + Wk * tail
    attention = {"path": "tensor cores (tree-major over 128-key tiles)" if kt.get("attend_combine") else "CUDA cores",
                 "walk_tile_pairs": pairs, "keys_attended": keys,
                 "ms": {k2: kt.get(k2) for k2 in ("attend_plan", "attend_partial", "attend_combine")},
                 "tensor": {"bound": "tensor", "kernel": "atc_max + atc_accum", "achieved":
                            att_flops / (att_ms / 1e3) / 1e12 if att_ms else None, "peak": bf16_peak,
                            "unit": "TFLOP/s", "frac": (att_flops / (att_ms / 1e3) / 1e12 / bf16_peak)
                            if att_ms and bf16_peak else None, "ops_per_step": att_flops,
                            "what": "MMA work issued: 4 x 2 x 128 x 128 per (walk, tile) pair"},
                 "algorithmic_tflops": keys * 4.0 * w.d / (att_ms / 1e3) / 1e12 if att_ms else None}
    res = {"workload": f"prefill: {w.queries_per_head:,} queries x 16 q-heads against the 4 KV-head trees of one "
                       "262,144-key sequence, d=128, bf16, C=8, depth 6, R=8, top-p 0.9",
           "walks": Wk, "ms": ms, "value": Wk / (ms / 1e3), "unit": UNIT, "kernel_ms": kt,
           "score_tflops": (flops / ((kt.get("score", 0) + kt.get("score_tc", 0)) / 1e3) / 1e12
                            if kt.get("score") or kt.get("score_tc") else None),
           "scored_walk_nodes": walk_nodes, "union_nodes": sum(info["union_nodes"][1:info["start_level"] + 1]),
           "tensor_roofline": tensor, "attention": attention}
    tree.close()
    del inp, sel, cnt, out, lse
    torch.cuda.empty_cache()
    return res


def append_rate(r, w):
    """Keys appended per second inside the timed step: the append kernels' device
    time per step (from the profiled pass) for one key per tree."""
    ms = r["kernel_ms_per_step"].get("append", 0.0) + r["kernel_ms_per_step"].get("build", 0.0)
    return {"keys_per_step": w.trees, "ms_per_step": ms, "keys_per_s": w.trees / (ms / 1e3) if ms else None,
            "what": "append kernel + the node builds of chunks that fill, per decode step"}


def config_of(w, label):
    return {"workload": label, "sequences": w.batch, "kv_heads": w.n_kv_heads, "q_heads": w.n_q_heads,
            "keys": w.n_keys, "d": w.d, "kv_dtype": w.kv_dtype, "chunk": w.chunk, "depth": w.depth, "R": w.R,
            "top_p": 0.9, "walks_per_step": w.walks, "step": "append 1 key/tree + search + attend",
            "l2": "flushed between timed steps (256 MB write)", "global_batch": w.walks}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.impl == "reference":
        return reference_arm(args, rank, world)
    import torch

    import synthetic as S

    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.prefill_only:
        if rank == 0:
            print(json.dumps(run_prefill(args, dev)), flush=True)
        return
    if args.build_only:
        if rank == 0:
            import tree_indexed_sparse_append_b200 as Z

            w = S.WORKLOADS["kv256k"]
            if args.batch:
                w = S.scaled(w, batch=args.batch)
            w = S.scaled(w, appends=0)
            inp = S.draw(w, device="cuda")
            tree = Z.Tree(inp.K, inp.V, inp.refs, w.n_keys, w.chunk, w.depth, w.beta, w.top_width)
            torch.cuda.synchronize()
            flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
            line = build_roofline(w, tree, flush, torch.cuda.current_stream(), inp.K.element_size())
            line["workload"] = f"kv256k build: {w.batch} seq x {w.n_kv_heads} KV heads x {w.n_keys:,} keys"
            print(json.dumps(line), flush=True)
            tree.close()
        return
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=dev)
    w = S.WORKLOADS["kv256k"]
    if args.batch:
        w = S.scaled(w, batch=args.batch)
    label = LABEL_256K.replace("16 seq", f"{w.batch} seq")
    head = run_decode(w, args, rank, world, dev, True, "kv256k", (("top_p", 0.9, 0),))
    extra = None
    if not args.no_extra:
        w4 = S.WORKLOADS["kv1m"]
        x = run_decode(w4, args, rank, world, dev, False, "kv1m", w4.modes, with_dense=True)
        extra = {"workload": "kv1m decode: 8 seq x 8 KV heads x 1,048,576 keys, 32 q-heads, d=128, bf16, C=16, "
                             "depth 5, R=8",
                 "build": x["build"], "parity_sample": x["parity"],
                 "modes": {m: {"value": r["qps"], "ms_per_step": r["ms_per_step"], "roofline": r["roofline"],
                               "keys_per_walk": r["keys_per_walk"], "selected_keys_per_s": r["selected_keys_per_s"],
                               "context_keys_per_s": r["context_keys_per_s"],
                               "attend_roofline": r["attend_roofline"], "select": r["select"],
                               "kernel_ms_per_step": r["kernel_ms_per_step"], "clocks": r["clocks"]}
                           for m, r in x["results"].items()},
                 "e2e": x["e2e"], "dense_scan": x["dense"]}
    prefill = None
    if not args.no_extra and rank == 0:
        prefill = run_prefill(args, dev)
    r = head["results"]["top_p"]
    line = {
        "metric": METRIC, "value": r["qps"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config_of(head["w"], label),
        "roofline": r["roofline"], "attend_roofline": r["attend_roofline"], "select": r["select"],
        "cpu_baseline": head["baseline"], "e2e": head["e2e"], "gpu_launches": round(r["launches"] * args.steps),
        "clocks": r["clocks"], "kernel_ms_per_step": r["kernel_ms_per_step"],
        "keys_per_walk": r["keys_per_walk"], "selected_keys_per_s": r["selected_keys_per_s"],
        "context_keys_per_s": r["context_keys_per_s"],
        "build": head["build"], "parity_sample": head["parity"], "learn": head["learn"],
        "append": append_rate(r, head["w"]),
        "kv1m": extra,
        "prefill": prefill,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def reference_arm(args, rank, world):
    """The CPU oracle on this host's cores, as the cpu_baseline leg runs it: the
    first CPU_TREES trees of the 256K workload (drawn on the CPU), every step one
    pass over their walks (append one key per tree, then search + attend of each
    walk), walks spread over all cores."""
    if rank != 0:
        return
    from concurrent.futures import ThreadPoolExecutor

    import oracle as O
    import synthetic as S

    w = S.WORKLOADS["kv256k"]
    cores = os.cpu_count() or 1
    group = w.n_q_heads // w.n_kv_heads
    trees = []
    for t in range(CPU_TREES):
        b, h = divmod(t, w.n_kv_heads)
        k, v, c = S.draw_tree(w, b, h, "cpu")
        K = k.double().numpy()
        V = v.double().numpy()
        refs = S.draw_refs(w, "cpu")[h].double().numpy()
        ot = O.build_tree(K[: w.n_keys], refs, w.chunk, w.depth, w.beta, threads=cores, capacity=K.shape[0])
        qs = [S.draw_queries(w, c, b, hq, "cpu")[0][0].double().numpy() for hq in range(h * group, (h + 1) * group)]
        trees.append((ot, K, V, qs))
    jobs = [(ot, K, V, q) for ot, K, V, qs in trees for q in qs]
    used = min(cores, len(jobs))

    def one(job):
        ot, K, V, q = job
        wk = O.search(ot, q, O.TOP_P, 0.9, 0, w.top_width)
        O.attend(K[: ot.n_keys], V[: ot.n_keys], q, wk.sel, w.chunk, ot.n_nodes[1], w.beta)

    with ThreadPoolExecutor(max_workers=used) as ex:
        def one_step():
            for ot, K, V, qs in trees:
                if ot.n_keys < K.shape[0]:
                    O.append(ot, K, 1)
            list(ex.map(one, jobs))

        for _ in range(args.warmup):
            one_step()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            one_step()
        dt = time.perf_counter() - t0
    value = args.steps * len(jobs) / dt
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_of(S.WORKLOADS["kv256k"], LABEL_256K),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "cpu_model": cpu_model(), "kind": "oracle",
                             "sample": f"{CPU_TREES} trees of the workload (262,144 keys, {len(jobs)} walks); a step "
                                       f"appends 1 key per tree and searches + attends every walk, over {used} "
                                       "threads"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
