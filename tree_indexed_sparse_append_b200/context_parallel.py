"""Context-parallel walk and attention over a torch.distributed process group.

Page "Subquadratic Attention with a Hierarchical Tree-Structured Indexer",
abstract: the method aims at contexts of hundreds of millions of tokens, more
than one GPU holds. Each process holds a shard of every tree: a run of whole
top-level nodes (C^depth keys each; the last process also holds the keys past
the last full top node), built with an ordinary ``Tree`` over its keys. The walk
takes one level at a time (zha_cp_export, an all-gather of the (global node id,
score) lists in process order, zha_cp_select) and makes exactly the choices a
single search over all keys makes; the attention over each shard's chosen keys is
merged by log-sum-exp (zha_lse_combine).

This module only moves data: the collectives are torch.distributed's (NCCL on
device tensors, or gloo through host copies); every step of the walk and the
attention runs in libzha's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import TOP_P, Tree, lse_combine


def key_range(n_keys: int, chunk: int, depth: int, rank: int, world: int):
    """[begin, end) of the keys that process `rank` of `world` holds: the whole top
    nodes (chunk^depth keys each) shared out in order, as evenly as possible; the
    last process also takes the keys past the last full top node."""
    span = chunk ** depth
    tops = n_keys // span
    base, extra = divmod(tops, world)
    begin = span * (rank * base + min(rank, extra))
    n = base + (1 if rank < extra else 0)
    end = n_keys if rank == world - 1 else begin + n * span
    return begin, end


def level_counts(n_keys: int, chunk: int, depth: int) -> list:
    """Keys and nodes per level (0..depth) of the tree over all n_keys keys."""
    out = [n_keys]
    for _ in range(depth):
        out.append(out[-1] // chunk)
    return out


def _gather(x: torch.Tensor, group) -> torch.Tensor:
    """[world] + x.shape: every process's x, in process order."""
    world = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        out = torch.empty((world,) + tuple(x.shape), dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(out, x.contiguous(), group=group)
        return out
    parts = [torch.empty(x.shape, dtype=x.dtype) for _ in range(world)]
    dist.all_gather(parts, x.detach().cpu().contiguous(), group=group)
    return torch.stack(parts).to(x.device)


def _max(v: int, group) -> int:
    dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.int64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return int(t.item())


def search(tree: Tree, Q: torch.Tensor, key_begin: int, global_counts, mode: int = TOP_P, p: float = 0.9,
           k: int = 1, max_sel: int | None = None, group=None):
    """The walk of every query of Q ([B][H_q][n_q][d]) over the whole tree, this
    process holding the shard that starts at key `key_begin`. Returns (sel
    [walks][max_sel] int32, sel_count [walks] int32): this shard's chosen chunks
    (local level-1 ids). Every process of the group must call it together."""
    B, Hq, nq, d = Q.shape
    W = B * Hq * nq
    n1 = tree.level(1)[1] if tree.depth >= 1 else 0
    stride = _max(max(1, n1), group)  # no shard's frontier is longer than its level 1
    if max_sel is None:
        max_sel = max(1, n1)
    ids = torch.empty(W, stride, dtype=torch.int32, device=Q.device)
    scores = torch.empty(W, stride, dtype=torch.float32, device=Q.device)
    counts = torch.empty(W, dtype=torch.int32, device=Q.device)
    sel = torch.empty(W, max_sel, dtype=torch.int32, device=Q.device)
    cnt = torch.empty(W, dtype=torch.int32, device=Q.device)
    level = tree.cp_begin(Q, key_begin, global_counts)
    while level > 0:
        tree.cp_export(ids, scores, counts)
        g_counts = _gather(counts, group)  # [world][W]
        m = max(1, int(g_counts.max().item()))  # the longest list of any process this level
        g_ids = _gather(ids[:, :m], group)
        g_scores = _gather(scores[:, :m], group)
        level = tree.cp_select(g_ids, g_scores, g_counts, mode, p, k, sel, cnt)
    return sel, cnt


def attend(tree: Tree, Q: torch.Tensor, sel: torch.Tensor, sel_count: torch.Tensor, out_dtype=torch.float32,
           group=None):
    """Attention of every query over the keys all processes chose (each shard's
    chunks, and the tail on the last process): each process attends over its own
    chosen keys, and the results are merged by log-sum-exp. Returns (out
    [walks][d] of out_dtype, lse [walks] fp32), the same on every process."""
    B, Hq, nq, d = Q.shape
    out, lse = tree.attend(Q, sel, sel_count, out_dtype=torch.float32)
    outs = _gather(out.reshape(B * Hq * nq, d), group)
    lses = _gather(lse, group)
    return lse_combine(outs, lses, out_dtype)
