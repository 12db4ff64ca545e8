"""The context-parallel walk's CPU reference (oracle/context_parallel.py) on gloo
ranks: a tree's keys split across 2 or 3 ranks, walked and attended with
collectives, give the single-tree oracle's walk and attention."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, case, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle as O
    from oracle import context_parallel as CP

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        N, C, depth, top_width, seed = case
        d, R, beta = 8, 3, 0.6
        rng = np.random.default_rng(seed)
        centres = rng.standard_normal((N // 16 + 1, d)) * 1.5
        K = (centres.repeat(16, axis=0)[:N] + 0.3 * rng.standard_normal((N, d))).astype(np.float32).astype(np.float64)
        V = rng.standard_normal((N, d))
        refs = rng.standard_normal((R, d))
        lo, hi = CP.key_ranges(N, C, depth, world)[rank]
        t, off = CP.build_shard(K, refs, C, depth, beta, lo, hi)
        full = O.build_tree(K, refs, C, depth, beta, store=O.STORE_F32)
        levels_ok = all(
            np.array_equal(t.level(l)[0], full.level(l)[0][off[l]: off[l] + t.n_nodes[l]])
            and np.array_equal(t.level(l)[1], full.level(l)[1][off[l]: off[l] + t.n_nodes[l]])
            for l in range(1, depth + 1))
        results = []
        for qi in range(5):
            q = centres[rng.integers(len(centres))] * rng.uniform(0.5, 2.0) + 0.1 * rng.standard_normal(d)
            for mode, p, k in ((O.TOP_P, 0.9, 0), (O.TOP_P, 0.5, 0), (O.TOP_P, 1.0, 0), (O.TOP_K, 0, 3)):
                mine = CP.walk(t, off, q, mode, p, k, top_width)
                parts = [None] * world
                dist.all_gather_object(parts, mine)
                union = np.sort(np.concatenate(parts))
                ref = O.search(full, q, mode, p, k, top_width)
                same = bool(np.array_equal(union, ref.sel))
                near = min(ref.tie_gap, ref.tie_sum) < 1e-9
                out_g, lse_g = CP.attend(K, V, q, mine, C, full.n_nodes[1], lo, hi, beta)
                out_o, lse_o = O.attend(K, V, q, union, C, full.n_nodes[1], beta)
                err = float(np.abs(out_g - out_o).max() / max(1.0, np.abs(out_o).max()))
                results.append((same or near, err, abs(lse_g - lse_o)))
        out.put((rank, levels_ok, results))
    finally:
        dist.destroy_process_group()


# (keys, C, depth, top_width, seed): rank runs of whole top nodes, the last rank
# with the orphans and the tail; a small top_width starts the walk at the top
CASES = [(1003, 8, 3, 64, 1), (4796, 4, 5, 64, 2), (3000, 4, 4, 4, 3)]


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("case", CASES)
def test_context_parallel_walk_equals_the_single_tree(case, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, levels_ok, results in res:
        assert levels_ok, f"rank {rank}: shard levels differ from the full tree's"
        for i, (ok, err, dlse) in enumerate(results):
            assert ok, f"rank {rank} walk {i}: selection differs away from a tie"
            assert err < 1e-12 and dlse < 1e-12, (rank, i, err, dlse)


def test_key_ranges_align_with_top_nodes():
    sys.path.insert(0, ROOT)
    from oracle import context_parallel as CP

    assert CP.key_ranges(4796, 4, 5, 3) == [(0, 2048), (2048, 3072), (3072, 4796)]
    assert CP.key_ranges(1003, 8, 3, 2) == [(0, 512), (512, 1003)]
    assert CP.key_ranges(100, 8, 3, 2) == [(0, 0), (0, 100)]  # no full top node: all on the last rank
