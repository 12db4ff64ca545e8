"""Tensor-core scoring (trees walked by at least 1,024 bf16 queries): parity with
the oracle, and agreement with the CUDA-core scorer on the same query values.

The workload: one sequence, 2 KV heads and 4 query heads (2:1), 550 queries per
query head, so 1,100 walks per tree (not a multiple of the 128-walk tile);
clustered keys (blocks of 64 around random centres) with C = 8 and depth 4; R = 6
reference queries (padded to 8 columns per node); d = 128, bf16 keys, values and
queries. Two tree sizes:
  * 16,427 keys: level sizes 2,053 / 256 / 32 / 4, tail of 3 keys; every level the
    walk visits is scored densely (all walks x all nodes);
  * 70,003 keys: level sizes 8,750 / 1,093 / 136 / 17, tail of 3 keys; level 1
    (more than 8,192 nodes) is scored sparsely (per tile of 16 nodes, only the
    walks whose frontier holds one of them), the others densely.
"""
import numpy as np
import pytest
import torch

import oracle as O
from helpers import (assert_attention_close, assert_partings_bounded, compare_selection, host64, near_tie,
                     tree_walk_valid)

pytestmark = pytest.mark.gpu

C, DEPTH, D, R, H, HQ, NQ = 8, 4, 128, 6, 2, 4, 550
BETA = 1 / np.sqrt(D)


def zha():
    import tree_indexed_sparse_append_b200 as Z

    return Z


def inputs(N, seed=7):
    g = torch.Generator(device="cuda").manual_seed(seed)
    blocks = (N + 63) // 64
    centres = torch.randn(H, blocks, D, generator=g, device="cuda")
    K = (centres.repeat_interleave(64, dim=1)[:, :N] + 0.3 * torch.randn(H, N, D, generator=g, device="cuda"))
    V = torch.randn(H, N, D, generator=g, device="cuda")
    refs = torch.randn(H, R, D, generator=g, device="cuda")
    # queries: the sum of 1 to 3 centres of their tree
    Q = torch.zeros(HQ, NQ, D, device="cuda")
    group = HQ // H
    for hq in range(HQ):
        m = torch.randint(1, 4, (NQ,), generator=g, device="cuda")
        for j in range(3):
            pick = torch.randint(0, blocks, (NQ,), generator=g, device="cuda")
            Q[hq] += centres[hq // group, pick] * (m > j).unsqueeze(1)
    return (K.to(torch.bfloat16)[None], V.to(torch.bfloat16)[None], refs, Q.to(torch.bfloat16)[None])


def sample_walks():
    # walks at the edges of the 128-walk tiles and spread over each tree
    G = (HQ // H) * NQ
    picks = set()
    for t in range(H):
        for r in list(range(0, G, 37)) + [0, 127, 128, 255, 256, 1023, 1024, G - 1]:
            if r < G:
                picks.add(t * G + r)
    return sorted(picks)


@pytest.mark.parametrize("N", [16427, 70003])
@pytest.mark.parametrize("mode,p,k", [(O.TOP_P, 0.9, 0), (O.TOP_K, 0, 8)])
def test_tensor_core_search_matches_oracle(mode, p, k, N):
    Z = zha()
    K, V, refs, Q = inputs(N)
    tree = Z.Tree(K, V, refs, N, C, DEPTH, BETA)
    max_sel = N // C
    sel, cnt, st = tree.search(Q, mode, p, k, max_sel=max_sel, with_stats=True)
    out, lse = tree.attend(Q, sel, cnt, out_dtype=torch.float32)
    tree.sync_status()
    sel_h, cnt_h = sel.cpu().numpy(), cnt.cpu().numpy()
    stats = Z.parse_stats(st)
    out = host64(out).reshape(-1, D)
    lse = lse.cpu().numpy()
    Qh = host64(Q).reshape(-1, D)
    G = (HQ // H) * NQ
    otrees = [O.build_tree(host64(K[0, h, :N]), host64(refs[h]), C, DEPTH, BETA, store=O.STORE_F32) for h in range(H)]
    checked = parted = 0
    Kh = [host64(K[0, h, :N]) for h in range(H)]
    Vh = [host64(V[0, h, :N]) for h in range(H)]
    for wi in sample_walks():
        h = wi // G
        ow = O.search(otrees[h], Qh[wi], mode, p, k, 64)
        if compare_selection(sel_h, cnt_h, {wi: ow}, tree_walk_valid(otrees[h], Qh[wi], mode, p, k, 64)):
            parted += 1
        else:
            assert stats[wi]["work"] == ow.work and stats[wi]["keys_read"] == ow.keys_read
        # the oracle's attention over the GPU's selection
        o_out, o_lse = O.attend(Kh[h], Vh[h], Qh[wi], sel_h[wi, : cnt_h[wi]], C, otrees[h].n_nodes[1], BETA)
        assert_attention_close(out[wi], lse[wi], o_out, o_lse, 3e-3, f"walk {wi}")
        checked += 1
    assert_partings_bounded(parted, checked, "tensor-core scoring")

    # every level went through a tensor-core path (dense, or sparse above 8,192 nodes)
    tree.profile(True)
    tree.search(Q, mode, p, k, max_sel=max_sel)
    kinds = tree.profile_read()
    tree.profile(False)
    assert kinds["score"][0] == 0 and kinds["score_tc"][0] > 0, kinds

    # the same query values as fp32 take the CUDA-core scorer
    sel2, cnt2, _ = tree.search(Q.float(), mode, p, k, max_sel=max_sel)
    tree.sync_status()
    sel2, cnt2 = sel2.cpu().numpy(), cnt2.cpu().numpy()
    differ = [w for w in range(sel_h.shape[0])
              if cnt_h[w] != cnt2[w] or not np.array_equal(sel_h[w, :cnt_h[w]], sel2[w, :cnt2[w]])]
    for wi in differ:
        ow = O.search(otrees[wi // G], Qh[wi], mode, p, k, 64)
        assert near_tie(ow), f"walk {wi}: tensor-core and CUDA-core selections differ away from a tie"
        valid = tree_walk_valid(otrees[wi // G], Qh[wi], mode, p, k, 64)
        for s, c in ((sel_h, cnt_h), (sel2, cnt2)):
            assert valid(wi, tuple(int(x) for x in s[wi, : c[wi]])), f"walk {wi}: not an admissible walk"
    assert_partings_bounded(len(differ), sel_h.shape[0], "tensor-core vs CUDA-core scoring")
    print(f"tensor-core scoring: {checked} sampled walks checked, {parted} part from the oracle; "
          f"{len(differ)} of {sel_h.shape[0]} walks part from the CUDA-core path, all at oracle near-ties")
    tree.close()


def test_bounded_wait_runs_out_and_is_reported():
    """The tensor-core scorer's waits are bounded. With the test hook on, each
    CTA's first wait (before any copy or MMA) is on a barrier that nothing
    arrives at; it gives up after 2 ms, the search reports ZHA_ERR_TIMEOUT through
    zha_sync_status, and once the hook is off the same tree searches correctly
    again (the context is still usable)."""
    Z = zha()
    N = 16427
    K, V, refs, Q = inputs(N, seed=11)
    tree = Z.Tree(K, V, refs, N, C, DEPTH, BETA)
    max_sel = N // C
    sel_a, cnt_a, _ = tree.search(Q, Z.TOP_P, 0.9, 0, max_sel=max_sel)
    tree.sync_status()
    sel_a, cnt_a = sel_a.cpu().numpy(), cnt_a.cpu().numpy()

    tree.test_wait_limit(2_000_000, stall=True)
    tree.profile(True)
    tree.search(Q, Z.TOP_P, 0.9, 0, max_sel=max_sel)
    kinds = tree.profile_read()
    tree.profile(False)
    assert kinds["score_tc"][0] > 0  # the dense tensor-core scorer ran
    with pytest.raises(Z.ZhaError) as e:
        tree.sync_status()
    assert e.value.code == Z.ERR_TIMEOUT
    tree.sync_status()  # the status word was cleared

    tree.test_wait_limit(0, stall=False)
    sel_b, cnt_b, _ = tree.search(Q, Z.TOP_P, 0.9, 0, max_sel=max_sel)
    tree.sync_status()
    sel_b, cnt_b = sel_b.cpu().numpy(), cnt_b.cpu().numpy()
    assert np.array_equal(cnt_a, cnt_b)
    for w in range(len(cnt_a)):
        assert np.array_equal(sel_a[w, : cnt_a[w]], sel_b[w, : cnt_b[w]])
    tree.close()


@pytest.mark.parametrize("N", [16427, 70003])
def test_tensor_core_attention_matches_cuda_cores_and_oracle(N):
    """Trees of 1,100 bf16 walks take the tensor-core attention (tree-major, per
    128-key tile against the walks that chose one of its chunks); the same
    selection with the queries as fp32 takes the CUDA-core attention. Both agree
    with each other and with the oracle, on trees with a 3-key tail (N not a
    multiple of 128 or of C), for top-p and top-K selections."""
    Z = zha()
    K, V, refs, Q = inputs(N, seed=13)
    tree = Z.Tree(K, V, refs, N, C, DEPTH, BETA)
    max_sel = N // C
    Qh = host64(Q).reshape(-1, D)
    G = (HQ // H) * NQ
    otrees = [O.build_tree(host64(K[0, h, :N]), host64(refs[h]), C, DEPTH, BETA, store=O.STORE_F32) for h in range(H)]
    Kh = [host64(K[0, h, :N]) for h in range(H)]
    Vh = [host64(V[0, h, :N]) for h in range(H)]
    for mode, p, k in [(O.TOP_P, 0.9, 0), (O.TOP_K, 0, 8), (O.TOP_P, 0.3, 0)]:
        sel, cnt, _ = tree.search(Q, mode, p, k, max_sel=max_sel)
        tree.profile(True)
        out_tc, lse_tc = tree.attend(Q, sel, cnt, out_dtype=torch.float32)
        kinds = tree.profile_read()
        tree.profile(False)
        assert kinds["attend_combine"][0] > 0 and kinds["attend_partial"][0] > 0, kinds  # the tensor-core path ran
        out_bf, _ = tree.attend(Q, sel, cnt)  # bf16 output, same path
        out_cc, lse_cc = tree.attend(Q.float(), sel, cnt, out_dtype=torch.float32)  # CUDA cores
        tree.sync_status()
        out_tc, out_cc = host64(out_tc).reshape(-1, D), host64(out_cc).reshape(-1, D)
        lse_tc, lse_cc = lse_tc.cpu().numpy(), lse_cc.cpu().numpy()
        err = np.abs(out_tc - out_cc) / np.maximum(1.0, np.abs(out_cc))
        assert err.max() <= 1e-4, f"tensor-core vs CUDA-core attention: {err.max():.3g}"
        assert np.abs(lse_tc - lse_cc).max() <= 1e-4 * max(1.0, np.abs(lse_cc).max())
        assert np.abs(host64(out_bf).reshape(-1, D) - out_tc).max() <= 2 ** -8 * max(1.0, np.abs(out_tc).max())
        sel_h, cnt_h = sel.cpu().numpy(), cnt.cpu().numpy()
        for wi in sample_walks():
            h = wi // G
            o_out, o_lse = O.attend(Kh[h], Vh[h], Qh[wi], sel_h[wi, : cnt_h[wi]], C, otrees[h].n_nodes[1], BETA)
            assert_attention_close(out_tc[wi], lse_tc[wi], o_out, o_lse, 3e-3, f"walk {wi}")
    tree.close()
