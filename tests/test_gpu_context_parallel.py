"""The context-parallel walk on the GPU: a tree's keys split across 2 or 3
processes (runs of whole top nodes, the last process with the orphans and the
tail), each building its shard on the GPU, walking level by level with the
(global id, score) lists all-gathered between the steps, and merging the
attention by log-sum-exp (tree_indexed_sparse_append_b200.context_parallel over
zha_cp_begin / zha_cp_export / zha_cp_select / zha_lse_combine).

The processes share the one GPU of the test machine and exchange through gloo on
host copies; no kernel waits on another process. Checked per walk:
  * the union of the shards' chosen chunks equals the single-tree GPU search over
    all keys, exactly (same node values bit for bit, same scores, same selector);
  * it equals the oracle's walk, or parts at an oracle near-tie as an admissible
    walk;
  * the merged attention equals the oracle's attention over the union (1e-5 for
    fp32 caches, 3e-3 for bf16) and the single-tree GPU attention.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


MODES = ((0, 0.9, 0), (0, 0.5, 0), (0, 1.0, 0), (1, 0.0, 3))


def _inputs(N, d, R, Hq, nq, seed):
    """The same keys, values, references and queries in every process (CPU generator)."""
    import torch

    g = torch.Generator().manual_seed(seed)
    blocks = N // 64 + 1
    centres = torch.randn(blocks, d, generator=g)
    K = centres.repeat_interleave(64, 0)[:N] + 0.3 * torch.randn(N, d, generator=g)
    V = torch.randn(N, d, generator=g)
    refs = torch.randn(1, R, d, generator=g)
    Q = torch.zeros(1, Hq, nq, d)
    for hq in range(Hq):
        for i in range(nq):
            m = int(torch.randint(1, 4, (1,), generator=g))
            pick = torch.randint(0, blocks, (m,), generator=g)
            Q[0, hq, i] = centres[pick].sum(0)
    return K, V, refs, Q


def _rank(rank, world, port, case, out_q):
    """One process: its results, or the error that stopped it, go to out_q."""
    try:
        _rank_body(rank, world, port, case, out_q)
    except BaseException:
        import traceback

        out_q.put((rank, "error", traceback.format_exc()))
        raise


def _rank_body(rank, world, port, case, out_q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    import torch.distributed as dist

    import oracle as O
    import tree_indexed_sparse_append_b200 as Z
    from helpers import TIE_TOL, tree_walk_valid
    from tree_indexed_sparse_append_b200 import context_parallel as CP

    import datetime

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        N, C, depth, top_width, d, R, bf16, seed = case
        Hq, nq = 2, 5
        dtype = torch.bfloat16 if bf16 else torch.float32
        beta = 1 / np.sqrt(d)
        K, V, refs, Q = _inputs(N, d, R, Hq, nq, seed)
        K, V, Q = K.to(dtype), V.to(dtype), Q.to(dtype)
        lo, hi = CP.key_range(N, C, depth, rank, world)
        cap = max(1, hi - lo)
        Ks = torch.zeros(1, 1, cap, d, dtype=dtype)
        Vs = torch.zeros(1, 1, cap, d, dtype=dtype)
        Ks[0, 0, : hi - lo] = K[lo:hi]
        Vs[0, 0, : hi - lo] = V[lo:hi]
        Ks, Vs, Qd, refs_d = Ks.cuda(), Vs.cuda(), Q.cuda(), refs.cuda()
        shard = Z.Tree(Ks, Vs, refs_d, hi - lo, C, depth, beta, top_width)
        full = Z.Tree(K[None, None].cuda().contiguous(), V[None, None].cuda().contiguous(), refs_d, N, C, depth, beta,
                      top_width)
        counts = CP.level_counts(N, C, depth)
        Kh = K.double().numpy()
        Vh = V.double().numpy()
        ot = O.build_tree(Kh, refs[0].double().numpy(), C, depth, beta, store=O.STORE_F32)
        Qh = Q.double().numpy().reshape(-1, d)
        tol = 3e-3 if bf16 else 1e-5
        results = []
        for mode, p, k in MODES:
            sel, cnt = CP.search(shard, Qd, lo, counts, mode, p, k)
            out, lse = CP.attend(shard, Qd, sel, cnt)
            shard.sync_status()
            sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
            mine = [sel[w, : cnt[w]].astype(np.int64) + lo // C for w in range(sel.shape[0])]
            parts = [None] * world
            dist.all_gather_object(parts, mine)
            fsel, fcnt, _ = full.search(Qd, mode, p, k)
            fout, flse = full.attend(Qd, fsel, fcnt, out_dtype=torch.float32)
            full.sync_status()
            fsel, fcnt = fsel.cpu().numpy(), fcnt.cpu().numpy()
            out = out.double().cpu().numpy()
            lse = lse.double().cpu().numpy()
            fout = fout.double().cpu().numpy().reshape(-1, d)
            flse = flse.double().cpu().numpy()
            for w in range(sel.shape[0]):
                union = np.sort(np.concatenate([pp[w] for pp in parts]))
                same_gpu = bool(np.array_equal(union, fsel[w, : fcnt[w]]))
                ow = O.search(ot, Qh[w], mode, p, k, top_width)
                same_oracle = bool(np.array_equal(union, ow.sel))
                valid = same_oracle or (min(ow.tie_gap, ow.tie_sum) < TIE_TOL and tree_walk_valid(
                    ot, Qh[w], mode, p, k, top_width)(w, tuple(int(x) for x in union)))
                o_out, o_lse = O.attend(Kh, Vh, Qh[w], union, C, ot.n_nodes[1], beta)
                err_o = max(float(np.max(np.abs(out[w] - o_out) / np.maximum(1, np.abs(o_out)))),
                            abs(lse[w] - o_lse) / max(1, abs(o_lse)))
                err_g = max(float(np.max(np.abs(out[w] - fout[w]) / np.maximum(1, np.abs(fout[w])))),
                            abs(lse[w] - flse[w]) / max(1, abs(flse[w])))
                results.append((mode, p, k, w, same_gpu, same_oracle, valid, err_o, err_g, tol))
        shard.close()
        full.close()
        out_q.put((rank, "ok", results))
    finally:
        dist.destroy_process_group()


# (keys, C, depth, top_width, d, R, bf16 cache, seed)
CASES = [
    (4096 + 37, 4, 4, 16, 64, 4, False, 1),   # 16 top nodes of 256 keys, orphans, a tail of 37
    (3000, 8, 3, 64, 128, 8, True, 2),        # 5 top nodes of 512 keys; bf16, d = 128, R = 8
    (100, 8, 3, 64, 64, 2, False, 3),         # no full top node: the last process holds every key
]


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("case", CASES)
def test_context_parallel_walk_on_the_gpu(case, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, case, q), daemon=True) for r in range(world)]
    for p in procs:
        p.start()
    res = []
    for _ in procs:
        rank, status, payload = q.get(timeout=300)
        assert status == "ok", f"rank {rank} failed:\n{payload}"
        res.append((rank, payload))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    parted = 0
    for rank, results in res:
        for mode, p, k, w, same_gpu, same_oracle, valid, err_o, err_g, tol in results:
            what = f"rank {rank} mode {mode} p {p} k {k} walk {w}"
            assert same_gpu, f"{what}: the shards' union differs from the single-tree GPU search"
            assert valid, f"{what}: not an admissible walk"
            parted += int(not same_oracle)
            assert err_o <= tol, f"{what}: merged attention off the oracle by {err_o:.3g}"
            assert err_g <= tol, f"{what}: merged attention off the single-tree GPU attention by {err_g:.3g}"
    n = sum(len(r) for _, r in res)
    assert parted <= max(1, n // 100), f"{parted} of {n} walks part from the oracle at near-ties"
