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
    e0.record(st)
    tree = Z.Tree(inp.K, inp.V, inp.refs, w.n_keys, w.chunk, w.depth, w.beta, w.top_width)
    e1.record(st)
    torch.cuda.synchronize()
    build_ms = e0.elapsed_time(e1)

    B, H, cap, d = inp.K.shape
    new_k = inp.K[:, :, w.n_keys:].permute(2, 0, 1, 3).contiguous()
    new_v = inp.V[:, :, w.n_keys:].permute(2, 0, 1, 3).contiguous()
    Wk = w.walks
    max_sel = cap // w.chunk
    sel = torch.empty(Wk, max_sel, dtype=torch.int32, device=dev)
    cnt = torch.empty(Wk, dtype=torch.int32, device=dev)
    out = torch.empty_like(inp.Q, dtype=inp.K.dtype)
    lse = torch.empty(Wk, dtype=torch.float32, device=dev)
    tree.reserve(Wk, max_sel)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)  # 256 MB > L2
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
        score_bytes = attend_bytes = 0
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
        for name, (n, ms) in tree.profile_read().items():
            kt[name] = {"launches": n, "ms": ms}
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
        results[mname] = {"qps": qps, "ms_per_step": total_ms / steps, "launches": launches / steps,
                          "clocks": clk.summary(), "roofline": roof, "attend_roofline": attend_roof,
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
            dense[mname] = {"ms": ms, "key_read_gbs": kbytes / (ms / 1e3) / 1e9, "kernel_ms": dk,
                            "keys_selected_mean": float(dcnt.float().mean().item()),
                            "tree_search_ms": search_ms, "dense_over_tree_search": ms / search_ms}
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
    e2e_ms = max_over_ranks(ea.elapsed_time(eb), world, dev)
    elt = inp.K.element_size()
    e2e = {"value": job_throughput(Wk, args.e2e_steps, world, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": Qd.numel() * Qd.element_size() + 2 * kd.numel() * elt,
           "d2h_bytes_per_step": out.numel() * out.element_size() + lse.numel() * 4}

    baseline = None
    if with_baseline and rank == 0:
        cores = os.cpu_count() or 1
        n_trees = 4
        sample = oracle_sample(w, inp, n_trees, cores)
        walks = sum(len(v[3]) for v in sample.values())
        used = min(cores, walks)
        v, done = oracle_walks_per_second(w, sample, args.cpu_seconds, used)
        baseline = {"value": v, "unit": UNIT, "cores": used, "kind": "oracle",
                    "sample": f"{n_trees} of {w.trees} trees ({walks} walks), append + search + attend per step, "
                              f"{done} walks in {args.cpu_seconds:.0f} s, oracle trees built beforehand"}
        del sample
    n_after = tree.n_keys
    tree.close()
    del inp, new_k, new_v, flush
    torch.cuda.empty_cache()
    return {"w": w, "results": results, "e2e": e2e, "build_ms": build_ms, "baseline": baseline,
            "n_keys_after": n_after, "dense": dense}


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
    res = {"workload": f"prefill: {w.queries_per_head:,} queries x 16 q-heads against the 4 KV-head trees of one "
                       "262,144-key sequence, d=128, bf16, C=8, depth 6, R=8, top-p 0.9",
           "walks": Wk, "ms": ms, "value": Wk / (ms / 1e3), "unit": UNIT, "kernel_ms": kt,
           "score_tflops": (flops / ((kt.get("score", 0) + kt.get("score_tc", 0)) / 1e3) / 1e12
                            if kt.get("score") or kt.get("score_tc") else None),
           "scored_walk_nodes": walk_nodes, "union_nodes": sum(info["union_nodes"][1:info["start_level"] + 1]),
           "tensor_roofline": tensor}
    tree.close()
    del inp, sel, cnt, out, lse
    torch.cuda.empty_cache()
    return res


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
                 "build_ms": x["build_ms"],
                 "modes": {m: {"value": r["qps"], "ms_per_step": r["ms_per_step"], "roofline": r["roofline"],
                               "attend_roofline": r["attend_roofline"],
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
        "roofline": r["roofline"], "attend_roofline": r["attend_roofline"],
        "cpu_baseline": head["baseline"], "e2e": head["e2e"], "gpu_launches": round(r["launches"] * args.steps),
        "clocks": r["clocks"], "kernel_ms_per_step": r["kernel_ms_per_step"],
        "build": {"ms": head["build_ms"], "keys_per_s": head["w"].trees * head["w"].n_keys / (head["build_ms"] / 1e3)},
        "kv1m": extra,
        "prefill": prefill,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def reference_arm(args, rank, world):
    """The CPU oracle on this host's cores, one bounded sample per step."""
    if rank != 0:
        return
    import numpy as np
    import torch

    import oracle as O
    import synthetic as S

    w = S.WORKLOADS["kv256k"]
    cores = os.cpu_count() or 1
    w = S.scaled(w, batch=1)
    group = w.n_q_heads // w.n_kv_heads
    trees = []
    for h in range(2):
        k, v, c = S.draw_tree(w, 0, h, "cpu")
        K = k.double().numpy()
        V = v.double().numpy()
        refs = S.draw_refs(w, "cpu")[h].double().numpy()
        ot = O.build_tree(K[: w.n_keys], refs, w.chunk, w.depth, w.beta, threads=cores, capacity=K.shape[0])
        qs = [S.draw_queries(w, c, 0, hq, "cpu")[0][0].double().numpy() for hq in range(h * group, (h + 1) * group)]
        trees.append((ot, K, V, qs))
    jobs = [(ot, K, V, q) for ot, K, V, qs in trees for q in qs]

    def one_step(i):
        ot, K, V, q = jobs[i % len(jobs)]
        O.append(ot, K, 1)
        wk = O.search(ot, q, O.TOP_P, 0.9, 0, w.top_width)
        O.attend(K[: ot.n_keys], V[: ot.n_keys], q, wk.sel, w.chunk, ot.n_nodes[1], w.beta)

    for i in range(args.warmup):
        one_step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one_step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = args.steps / dt
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_of(S.WORKLOADS["kv256k"], LABEL_256K),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": "2 sampled trees of the workload (262,144 keys), one walk per step: "
                                       "append 1 key + search + attend, single thread"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
