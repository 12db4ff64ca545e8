"""Host logic of the context-parallel driver (tree_indexed_sparse_append_b200.
context_parallel), on the CPU: the key ranges each process holds, the level counts
of the whole tree, and the collectives' gloo path (host copies) on 2 ranks.

Key ranges (page "Subquadratic Attention with a Hierarchical Tree-Structured
Indexer", abstract: the tree is over the whole context, which may be longer than
one GPU holds): every process holds whole top nodes, C^depth keys each, shared
out in order as evenly as possible; the last process also holds the keys past the
last full top node. The expected ranges below are worked out by hand.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from tree_indexed_sparse_append_b200 import context_parallel as CP  # noqa: E402


@pytest.mark.parametrize("case, expected", [
    # 4,796 keys, C = 4, depth 5: top nodes of 1,024 keys, 4 of them, 700 keys after;
    # 3 processes get 2, 1 and 1 top nodes, the last one the 700 keys too
    ((4796, 4, 5, 3), [(0, 2048), (2048, 3072), (3072, 4796)]),
    # 1,003 keys, C = 8, depth 3: one top node of 512 keys, 491 after
    ((1003, 8, 3, 2), [(0, 512), (512, 1003)]),
    # no full top node: the last process holds every key
    ((100, 8, 3, 2), [(0, 0), (0, 100)]),
    # 5 top nodes of 512 keys over 3 processes: 2, 2, 1 (and no keys after)
    ((2560, 8, 3, 3), [(0, 1024), (1024, 2048), (2048, 2560)]),
])
def test_key_ranges_worked_cases(case, expected):
    N, C, depth, world = case
    assert [CP.key_range(N, C, depth, r, world) for r in range(world)] == expected


@pytest.mark.parametrize("N", [0, 1, 63, 64, 65, 4095, 4096, 4097, 70001])
@pytest.mark.parametrize("C, depth", [(4, 3), (8, 2), (16, 2)])
@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_key_ranges_partition_the_keys(N, C, depth, world):
    span = C ** depth
    ranges = [CP.key_range(N, C, depth, r, world) for r in range(world)]
    # contiguous, in order, covering [0, N)
    assert ranges[0][0] == 0 and ranges[-1][1] == N
    for (a0, a1), (b0, _) in zip(ranges, ranges[1:]):
        assert a1 == b0 and a0 <= a1
    # every process but the last holds whole top nodes, and their counts differ by at most one
    tops = [(hi - lo) // span for lo, hi in ranges[:-1]]
    for lo, hi in ranges[:-1]:
        assert lo % span == 0 and (hi - lo) % span == 0
    last_lo, last_hi = ranges[-1]
    assert last_lo % span == 0
    last_tops = (last_hi - last_lo) // span
    counts = tops + [last_tops]
    assert max(counts) - min(counts) <= 1
    assert sum(counts) == N // span
    # the keys past the last full top node are on the last process
    assert last_hi - last_lo - last_tops * span == N % span


def test_level_counts():
    assert CP.level_counts(4796, 4, 5) == [4796, 1199, 299, 74, 18, 4]
    assert CP.level_counts(100, 8, 3) == [100, 12, 1, 0]
    assert CP.level_counts(0, 8, 2) == [0, 0, 0]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gather_rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from tree_indexed_sparse_append_b200 import context_parallel as cp

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        x = torch.arange(6, dtype=torch.int32).reshape(2, 3) + 100 * rank
        g = cp._gather(x, None)
        m = cp._max(7 * rank + 1, None)
        q.put((rank, g.tolist(), m))
    finally:
        dist.destroy_process_group()


def test_gather_and_max_over_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_rank, args=(r, world, port, q), daemon=True) for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r, (g, m)) for r, g, m in (q.get(timeout=120) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    expected = [[[r * 100 + 3 * i + j for j in range(3)] for i in range(2)] for r in range(world)]
    for r in range(world):
        g, m = got[r]
        assert g == expected  # every process gets every process's tensor, in process order
        assert m == 7 * (world - 1) + 1
