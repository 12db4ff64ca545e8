"""Context-parallel tree walk: the CPU reference of one tree's walk with its keys
split across ranks.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT. Like the rest of ``oracle/``, only
``tests/``, the smoke check and ``bench.py``'s CPU legs may import it; it shares no
code with the CUDA library.

The keys of one tree are split across the ranks of a process group in runs of
whole top-level nodes (C^depth keys each); the last rank also takes the keys past
the last full top node. Each rank builds the levels of its own keys with the
oracle's build (page "How does a tree of summaries search a context? How ZHA
works", sections "How is the tree built?" and "What does a node summarize?").
Because the runs align with the top nodes, rank r's level-l nodes are the nodes
off_l(r) .. off_l(r) + n_l(r) - 1 of the tree over all keys, bit for bit.

The walk then takes the single-tree steps (section "Run a small tree yourself",
route; "How does top-p differ from top-K?") with the collective each one needs:
- the start level: the lowest level whose node count, summed over the ranks, is at
  most top_width (an all-reduce of the counts);
- the softmax over the whole frontier and the top-p / top-K choice: every rank
  scores its own frontier nodes and the (node id, score) lists are all-gathered
  in rank order, which is ascending node id, the single-tree frontier order; every
  rank makes the same choice and keeps the opened nodes it holds;
- the next frontier: each rank's children of its opened nodes, then the orphans
  of the level below, which only the last rank holds;
- the attention over the chosen keys (section "Common misunderstandings": plain
  attention over the original keys): each rank's partial maximum, sum of
  exponentials and weighted sum of values over its own chosen keys (and, on the
  last rank, the tail), combined by log-sum-exp through two all-reduces.
The result is the single-tree walk and attention over all keys.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import STORE_F32, TOP_K, TOP_P, build_tree


def key_ranges(N: int, C: int, depth: int, world: int):
    """[lo, hi) key range of every rank: whole top-level nodes shared out as
    evenly as possible in order; the last rank also takes the rest of the keys."""
    span = C ** depth
    tops = N // span
    base, extra = divmod(tops, world)
    out, lo = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        hi = lo + n * span if r < world - 1 else N
        out.append((lo, hi))
        lo = hi
    return out


def build_shard(K, refs, C: int, depth: int, beta: float, lo: int, hi: int):
    """This rank's levels (oracle build over keys lo..hi-1) and each level's first
    global node id."""
    t = build_tree(K[lo:hi], refs, C, depth, beta, store=STORE_F32)
    return t, [lo // C ** l for l in range(depth + 1)]


def _choose(ids: np.ndarray, score: np.ndarray, mode: int, p: float, k: int) -> np.ndarray:
    """Ids opened among a whole frontier: softmax, order by (mass desc, id asc),
    then the shortest prefix reaching p (top-p; all when p >= 1) or the first k."""
    w = np.exp(score - score.max())
    w = w / w.sum()
    order = np.lexsort((ids, -w))
    if mode == TOP_K:
        c = min(k, len(ids))
    elif p >= 1:
        c = len(ids)
    else:
        total, c = 0.0, 0
        while c < len(ids):
            total += w[order[c]]
            c += 1
            if total >= p:
                break
    return ids[order[:c]]


def walk(t, off, q, mode: int = TOP_P, p: float = 0.9, k: int = 1, top_width: int = 64, group=None):
    """This rank's share of the walk of q: the opened level-1 node ids (global,
    ascending) that it holds. The union over ranks is the single-tree walk."""
    depth, C, R = t.depth, t.C, t.R
    counts = torch.tensor([float(t.n_nodes[l]) for l in range(depth + 1)], dtype=torch.float64)
    dist.all_reduce(counts, group=group)
    n = [int(x) for x in counts.tolist()]
    s = next((l for l in range(1, depth + 1) if n[l] <= top_width), depth)
    world = dist.get_world_size(group)
    F = off[s] + np.arange(t.n_nodes[s], dtype=np.int64)  # global ids, ascending
    for l in range(s, 0, -1):
        keys, bias = t.level(l)
        local = F - off[l]
        score = (beta_dot(keys[local], q, t.beta) + bias[local]).max(axis=1) if len(F) else np.zeros(0)
        lists = [None] * world
        dist.all_gather_object(lists, (F, score), group=group)
        all_ids = np.concatenate([x[0] for x in lists])
        all_score = np.concatenate([x[1] for x in lists])
        opened = _choose(all_ids, all_score, mode, p, k) if len(all_ids) else np.zeros(0, dtype=np.int64)
        mine = np.sort(opened[(opened >= off[l]) & (opened < off[l] + t.n_nodes[l])])
        if l == 1:
            return mine
        children = (mine[:, None] * C + np.arange(C)[None, :]).reshape(-1)
        # orphans of level l-1 (no parent yet) belong to the rank holding them
        orphans = np.arange(C * n[l], n[l - 1], dtype=np.int64)
        orphans = orphans[(orphans >= off[l - 1]) & (orphans < off[l - 1] + t.n_nodes[l - 1])]
        F = np.concatenate([children, orphans]).astype(np.int64)
    return np.zeros(0, dtype=np.int64)


def beta_dot(keys: np.ndarray, q: np.ndarray, beta: float) -> np.ndarray:
    """beta * <key_{j,r}, q> for keys [F][R][d]."""
    return beta * np.einsum("jrd,d->jr", keys, q)


def attend(K, V, q, mine, C: int, n1_global: int, lo: int, hi: int, beta: float, group=None):
    """Attention of q over the chosen keys, combined across ranks: this rank
    contributes the keys of its opened level-1 nodes and, when it holds them, the
    tail keys C*n1_global .. N-1. Returns (out, lse), the same on every rank."""
    idx = [np.arange(c * C, c * C + C) for c in mine]
    tail0 = C * n1_global
    if hi > tail0:
        idx.append(np.arange(max(lo, tail0), hi))
    idx = np.concatenate(idx) if idx else np.zeros(0, dtype=np.int64)
    d = K.shape[1]
    if len(idx):
        s = beta * (K[idx] @ q)
        m = s.max()
        e = np.exp(s - m)
        part = (m, e.sum(), e @ V[idx])
    else:
        part = (-np.inf, 0.0, np.zeros(d))
    M = torch.tensor([part[0]], dtype=torch.float64)
    dist.all_reduce(M, op=dist.ReduceOp.MAX, group=group)
    M = float(M.item())
    scale = 0.0 if part[0] == -np.inf else np.exp(part[0] - M)
    acc = torch.tensor(np.concatenate([[part[1] * scale], part[2] * scale]), dtype=torch.float64)
    dist.all_reduce(acc, group=group)
    acc = acc.numpy()
    return acc[1:] / acc[0], M + np.log(acc[0])
