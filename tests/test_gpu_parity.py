"""GPU parity: the CUDA library (through its C ABI) against the oracle, on the same
seeded inputs, at sizes the oracle finishes in seconds (several tiles, ragged
tails, orphans, GQA groups, several queries per head).

What is compared, per workload and mode:
  * every node key and bias of every level of every tree (1e-5 relative);
  * every walk's selected chunk set (identical except at oracle near-ties, which
    are counted and printed; such a walk must be an admissible walk under the
    oracle's masses, and at most 1% of the walks, at least one, may part) and its
    counters (frontier and opened per level, keys read, comparisons);
  * the attention over the oracle's own selection (GPU attend fed the oracle's
    chunk lists), and the end-to-end search + attend against the oracle's
    attention over the GPU's selection (the same as the oracle's own, except for
    a walk that parts at a near-tie);
  * p = 1 against dense attention.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from helpers import (assert_attention_close, assert_bf16_output_close, assert_nodes_close,
                     assert_partings_bounded, attn_tol, compare_selection, gpu_level, host64, one_level_valid,
                     oracle_tree, tree_walk_valid)

pytestmark = pytest.mark.gpu

SMALL = {
    "demo4k": S.WORKLOADS["demo4k"],
    "demo4k_iid": S.control(S.WORKLOADS["demo4k"]),
    "kv64k": S.WORKLOADS["kv64k"],
    "kv256k_small": S.scaled(S.WORKLOADS["kv256k"], name="kv256k_small", batch=2, n_keys=32768 + 5 * 8 + 3,
                             depth=5, appends=512),
    "kv1m_small": S.scaled(S.WORKLOADS["kv1m"], name="kv1m_small", batch=1, n_keys=65536, depth=4),
}

MODE = {"top_p": O.TOP_P, "top_k": O.TOP_K}


def zha():
    import tree_indexed_sparse_append_b200 as Z

    return Z


def walk_index(w, b, hq, i):
    return (b * w.n_q_heads + hq) * w.queries_per_head + i


class Case:
    def __init__(self, name, w):
        self.name, self.w = name, w
        self.inp = S.draw(w, device="cuda")
        self.tree = zha().Tree(self.inp.K, self.inp.V, self.inp.refs, w.n_keys, w.chunk, w.depth, w.beta,
                               w.top_width)
        torch.cuda.synchronize()
        self.otrees = {(b, h): oracle_tree(self.inp, b, h, threads=8)
                       for b in range(w.batch) for h in range(w.n_kv_heads)}
        self.Kh = {k: host64(self.inp.K[k[0], k[1], : w.n_keys]) for k in self.otrees}
        self.Vh = {k: host64(self.inp.V[k[0], k[1], : w.n_keys]) for k in self.otrees}
        self.Qh = host64(self.inp.Q)

    def walks(self):
        w = self.w
        group = w.n_q_heads // w.n_kv_heads
        for b in range(w.batch):
            for hq in range(w.n_q_heads):
                for i in range(w.queries_per_head):
                    yield walk_index(w, b, hq, i), (b, hq // group), self.Qh[b, hq, i]

    def oracle_search(self, mode, p, k):
        return {wi: O.search(self.otrees[key], q, MODE[mode], p, k, self.w.top_width)
                for wi, key, q in self.walks()}

    def valid(self, mode, p, k):
        """compare_selection's check that a parting walk is admissible."""
        where = {wi: (key, q) for wi, key, q in self.walks()}

        def check(wi, g):
            key, q = where[wi]
            return tree_walk_valid(self.otrees[key], q, MODE[mode], p, k, self.w.top_width)(wi, g)
        return check


@pytest.fixture(scope="module", params=list(SMALL))
def case(request):
    c = Case(request.param, SMALL[request.param])
    yield c
    c.tree.close()
    del c
    torch.cuda.empty_cache()


def test_build_matches_oracle(case):
    w = case.w
    for (b, h), ot in case.otrees.items():
        t = b * w.n_kv_heads + h
        for l in range(1, w.depth + 1):
            g, n = gpu_level(case.tree, l, t)
            assert n == ot.n_nodes[l]
            keys, bias = ot.level(l)
            assert_nodes_close(g, keys, bias, w.R, w.d, what=f"{case.name} tree {t} level {l}")


@pytest.mark.parametrize("mode_i", [0, 1])
def test_search_matches_oracle(case, mode_i):
    w = case.w
    if mode_i >= len(w.modes):
        pytest.skip("workload has one mode")
    mode, p, k = w.modes[mode_i]
    Z = zha()
    sel, cnt, st = case.tree.search(case.inp.Q, MODE[mode], p, k, with_stats=True)
    case.tree.sync_status()
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    stats = Z.parse_stats(st)
    ow = case.oracle_search(mode, p, k)
    differ = compare_selection(sel, cnt, ow, case.valid(mode, p, k))
    print(f"{case.name} {mode}: {len(differ)} of {len(ow)} walks part at oracle near-ties")
    assert_partings_bounded(len(differ), len(ow), f"{case.name} {mode}")
    for wi, o in ow.items():
        if wi in differ:
            continue
        s = stats[wi]
        assert s["start_level"] == o.start_level
        assert s["frontier"][: w.depth + 1][1:] == o.frontier[1:]
        assert s["opened"][: w.depth + 1][1:] == o.opened[1:]
        assert s["keys_read"] == o.keys_read and s["work"] == o.work


def test_attend_on_oracle_selection(case):
    w = case.w
    mode, p, k = w.modes[0]
    ow = case.oracle_search(mode, p, k)
    n1 = case.otrees[(0, 0)].n_nodes[1]
    W = w.walks
    max_sel = max(1, max(len(o.sel) for o in ow.values()))
    sel = np.zeros((W, max_sel), dtype=np.int32)
    cnt = np.zeros(W, dtype=np.int32)
    for wi, o in ow.items():
        sel[wi, : len(o.sel)] = o.sel
        cnt[wi] = len(o.sel)
    sel_d, cnt_d = torch.from_numpy(sel).cuda(), torch.from_numpy(cnt).cuda()
    out, lse = case.tree.attend(case.inp.Q, sel_d, cnt_d, out_dtype=torch.float32)
    out_c, _ = case.tree.attend(case.inp.Q, sel_d, cnt_d)  # in the cache dtype
    case.tree.sync_status()
    out = host64(out).reshape(W, w.d)
    out_c = host64(out_c).reshape(W, w.d)
    lse = lse.cpu().numpy()
    for wi, key, q in case.walks():
        o_out, o_lse = O.attend(case.Kh[key], case.Vh[key], q, ow[wi].sel, w.chunk, n1, w.beta)
        assert_attention_close(out[wi], lse[wi], o_out, o_lse, attn_tol(w), f"{case.name} walk {wi}")
        if w.kv_dtype == "bf16":
            assert_bf16_output_close(out_c[wi], o_out, f"{case.name} walk {wi}")


def test_search_then_attend_end_to_end(case):
    w = case.w
    mode, p, k = w.modes[0]
    sel, cnt, _ = case.tree.search(case.inp.Q, MODE[mode], p, k)
    out, lse = case.tree.attend(case.inp.Q, sel, cnt, out_dtype=torch.float32)
    case.tree.sync_status()
    ow = case.oracle_search(mode, p, k)
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    differ = compare_selection(sel, cnt, ow, case.valid(mode, p, k))
    assert_partings_bounded(len(differ), len(ow), f"{case.name} {mode}")
    out = host64(out).reshape(w.walks, w.d)
    lse = lse.cpu().numpy()
    n1 = case.otrees[(0, 0)].n_nodes[1]
    for wi, key, q in case.walks():
        # the oracle's attention over the GPU's own selection (the oracle's, unless
        # the walk parted at a near-tie)
        o_out, o_lse = O.attend(case.Kh[key], case.Vh[key], q, sel[wi, : cnt[wi]], w.chunk, n1, w.beta)
        assert_attention_close(out[wi], lse[wi], o_out, o_lse, attn_tol(w), f"{case.name} walk {wi}")


def test_p_one_is_dense_attention(case):
    w = case.w
    sel, cnt, _ = case.tree.search(case.inp.Q, O.TOP_P, 1.0, 0)
    out, lse = case.tree.attend(case.inp.Q, sel, cnt, out_dtype=torch.float32)
    case.tree.sync_status()
    n1 = case.otrees[(0, 0)].n_nodes[1]
    cnt = cnt.cpu().numpy()
    assert (cnt == n1).all()
    assert (sel.cpu().numpy()[:, :n1] == np.arange(n1)[None, :]).all()
    out = host64(out).reshape(w.walks, w.d)
    lse = lse.cpu().numpy()
    for j, (wi, key, q) in enumerate(case.walks()):
        if j % 7:
            continue
        Kd, Vd = case.Kh[key], case.Vh[key]
        s = w.beta * Kd @ q
        m = s.max()
        e = np.exp(s - m)
        ref = e @ Vd / e.sum()
        assert_attention_close(out[wi], lse[wi], ref, m + np.log(e.sum()), attn_tol(w), f"{case.name} walk {wi}")


# ---------------------------------------------------------------------------
# edge cases, each against the oracle


def _tiny(N, cap=None, C=8, depth=3, d=64, R=4, B=1, H=1, Hq=1, nq=4, dtype=torch.float32, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    cap = cap or max(N, 1)
    K = torch.randn(B, H, cap, d, generator=g, device="cuda").to(dtype)
    V = torch.randn(B, H, cap, d, generator=g, device="cuda").to(dtype)
    refs = torch.randn(H, R, d, generator=g, device="cuda")
    Q = (2 * torch.randn(B, Hq, nq, d, generator=g, device="cuda")).to(dtype)
    return K, V, refs, Q


def _check_against_oracle(K, V, refs, Q, N, C, depth, beta, top_width=64, modes=((O.TOP_P, 0.9, 0),)):
    Z = zha()
    tree = Z.Tree(K, V, refs, N, C, depth, beta, top_width)
    B, H, _, d = K.shape
    Hq, nq = Q.shape[1], Q.shape[2]
    group = Hq // H
    R = refs.shape[1]
    Qh = host64(Q)
    levels = tree.depth  # depth 0: the levels the keys fill, on both sides
    for b in range(B):
        for h in range(H):
            ot = O.build_tree(host64(K[b, h, :N]), host64(refs[h]), C, depth, beta, store=O.STORE_F32)
            assert ot.depth == levels
            for l in range(1, levels + 1):
                g, n = gpu_level(tree, l, b * H + h)
                assert n == ot.n_nodes[l]
                if n:
                    keys, bias = ot.level(l)
                    assert_nodes_close(g, keys, bias, R, d)
    parted = walks = 0
    for mode, p, k in modes:
        sel, cnt, st = tree.search(Q, mode, p, k, max_sel=max(1, N // C), with_stats=True)
        out, lse = tree.attend(Q, sel, cnt, out_dtype=torch.float32)
        out_c, _ = tree.attend(Q, sel, cnt)
        tree.sync_status()
        sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
        stats = Z.parse_stats(st)
        out = host64(out).reshape(-1, d)
        out_c = host64(out_c).reshape(-1, d)
        lse = lse.cpu().numpy()
        for b in range(B):
            for hq in range(Hq):
                h = hq // group
                ot = O.build_tree(host64(K[b, h, :N]), host64(refs[h]), C, depth, beta, store=O.STORE_F32)
                Kd, Vd = host64(K[b, h, :N]), host64(V[b, h, :N])
                for i in range(nq):
                    wi = (b * Hq + hq) * nq + i
                    ow = O.search(ot, Qh[b, hq, i], mode, p, k, top_width)
                    parted += len(compare_selection(sel, cnt, {wi: ow},
                                                    tree_walk_valid(ot, Qh[b, hq, i], mode, p, k, top_width)))
                    walks += 1
                    g = sel[wi, : cnt[wi]]
                    if np.array_equal(g, ow.sel):
                        assert stats[wi]["keys_read"] == ow.keys_read and stats[wi]["work"] == ow.work
                    if N == 0:
                        assert lse[wi] == -np.inf and not out[wi].any()
                        continue
                    # the oracle's attention over the GPU's selection
                    o_out, o_lse = O.attend(Kd, Vd, Qh[b, hq, i], g, C, ot.n_nodes[1], beta)
                    tol = 1e-5 if K.dtype == torch.float32 else 3e-3
                    assert_attention_close(out[wi], lse[wi], o_out, o_lse, tol)
                    if K.dtype == torch.bfloat16:
                        assert_bf16_output_close(out_c[wi], o_out)
    assert_partings_bounded(parted, walks)
    tree.close()


ALL_MODES = ((O.TOP_P, 0.9, 0), (O.TOP_P, 1.0, 0), (O.TOP_P, 0.3, 0), (O.TOP_K, 0, 1), (O.TOP_K, 0, 3),
             (O.TOP_K, 0, 1000))


def test_tail_and_orphans():
    # 1003 keys, C = 8: level sizes 125 / 15 / 1, five level-1 orphans, three tail keys
    K, V, refs, Q = _tiny(1003, nq=6)
    _check_against_oracle(K, V, refs, Q, 1003, 8, 3, 0.125, modes=ALL_MODES)


def test_tree_smaller_than_a_chunk():
    K, V, refs, Q = _tiny(5)
    _check_against_oracle(K, V, refs, Q, 5, 8, 3, 0.125, modes=ALL_MODES)


def test_empty_tree():
    K, V, refs, Q = _tiny(0, cap=16)
    _check_against_oracle(K, V, refs, Q, 0, 8, 2, 0.125)


def test_walk_from_the_root():
    K, V, refs, Q = _tiny(4096, C=4, depth=6, nq=8)
    _check_against_oracle(K, V, refs, Q, 4096, 4, 6, 0.125, top_width=1, modes=ALL_MODES)


def test_gqa_bf16_d128_and_d256():
    for d in (128, 256):
        K, V, refs, Q = _tiny(3000, C=16, depth=3, d=d, R=8, B=2, H=2, Hq=4, nq=3, dtype=torch.bfloat16, seed=d)
        _check_against_oracle(K, V, refs, Q, 3000, 16, 3, 1 / np.sqrt(d), modes=ALL_MODES[:4])


def test_odd_reference_count_and_chunk():
    K, V, refs, Q = _tiny(2000, C=5, depth=4, d=64, R=3, nq=5)
    _check_against_oracle(K, V, refs, Q, 2000, 5, 4, 0.2, modes=ALL_MODES)


def test_large_frontiers():
    # 200,000 keys, C = 8: 25,000 level-1 nodes under 3,125 level-2 nodes; with the
    # walk starting at level 2, the level-1 frontier reaches 25,000 nodes (more
    # than a 512-thread selector stages in shared memory) at p = 1, and between
    # 8,192 and 16,384 nodes for the smaller p
    K, V, refs, Q = _tiny(200000, C=8, depth=2, d=64, R=2, nq=3, seed=5)
    _check_against_oracle(K, V, refs, Q, 200000, 8, 2, 0.125, top_width=4096,
                          modes=((O.TOP_P, 1.0, 0), (O.TOP_P, 0.9, 0), (O.TOP_P, 0.5, 0), (O.TOP_K, 0, 2500),
                                 (O.TOP_K, 0, 1500)))


@pytest.mark.parametrize("N", [8192, 16384])
def test_many_walks_warp_selector(N):
    # 8,192 walks (a prefill-sized call) on trees of C = 4, depth 6: 8,192 keys give
    # levels of 2,048, 512, 128, 32, 8 and 2 nodes, 16,384 keys levels of 4,096,
    # 1,024, 256, 64, 16 and 4, so the walk starts at 32 or 64 nodes and the levels
    # of 128, 256 and 512 nodes are selected by the one-warp-per-walk selector with
    # 4, 8 and 16 keys per lane; every walk is checked against the oracle
    K, V, refs, Q = _tiny(N, C=4, depth=6, d=64, R=4, nq=8192, seed=11)
    _check_against_oracle(K, V, refs, Q, N, 4, 6, 0.125, top_width=64,
                          modes=((O.TOP_P, 0.9, 0), (O.TOP_K, 0, 3)))


def test_max_sel_overflow_is_reported():
    Z = zha()
    K, V, refs, Q = _tiny(1024, C=8, depth=2)
    tree = Z.Tree(K, V, refs, 1024, 8, 2, 0.125)
    sel, cnt, _ = tree.search(Q, O.TOP_P, 1.0, 0, max_sel=3)
    with pytest.raises(Z.ZhaError) as e:
        tree.sync_status()
    assert e.value.code == Z.ERR_CAPACITY
    assert (cnt.cpu().numpy() == 3).all()
    assert (sel.cpu().numpy() == np.arange(3)[None, :]).all()
    tree.sync_status()  # cleared
    tree.close()


def test_append_equals_build():
    Z = zha()
    B, H, d, R, C, depth = 2, 2, 128, 8, 8, 4
    N0, M = 1000, 1100
    K, V, refs, Q = _tiny(N0 + M, C=C, depth=depth, d=d, R=R, B=B, H=H, Hq=4, nq=2, dtype=torch.bfloat16)
    grown_K = K.clone()
    grown_V = V.clone()
    grown_K[:, :, N0:] = 0
    grown_V[:, :, N0:] = 0
    grown = Z.Tree(grown_K, grown_V, refs, N0, C, depth, 1 / np.sqrt(d))
    for i in range(N0, N0 + M):
        grown.append(K[:, :, i].contiguous(), V[:, :, i].contiguous())
    assert grown.n_keys == N0 + M
    assert torch.equal(grown_K, K) and torch.equal(grown_V, V)
    direct = Z.Tree(K, V, refs, N0 + M, C, depth, 1 / np.sqrt(d))
    assert grown.level_sizes() == direct.level_sizes() == [2100, 262, 32, 4, 0]
    for l in range(1, depth + 1):
        a, n = grown.level(l)
        b, m = direct.level(l)
        assert torch.equal(a[:, :n], b[:, :m])  # same kernel, same inputs: bit-identical
    ot = O.build_tree(host64(K[1, 1, :N0]), host64(refs[1]), C, depth, 1 / np.sqrt(d), capacity=N0 + M)
    O.append(ot, host64(K[1, 1]), M)
    for l in range(1, depth + 1):
        g, n = gpu_level(grown, l, 3)
        if n:
            assert_nodes_close(g, *ot.level(l), R, d)
    grown.close()
    direct.close()


def test_growing_depth():
    """depth 0: the trees keep every level that holds a node, and the append that
    completes a full group of C top nodes starts a new level. The grown trees
    equal a growing build over the final keys bit for bit, and the oracle."""
    Z = zha()
    B, H, d, R, C = 2, 2, 128, 8, 4
    N0, M = 250, 30
    K, V, refs, Q = _tiny(N0 + M, C=C, d=d, R=R, B=B, H=H, Hq=4, nq=3, dtype=torch.bfloat16, seed=5)
    beta = 1 / np.sqrt(d)
    grown_K, grown_V = K.clone(), V.clone()
    grown_K[:, :, N0:] = 0
    grown_V[:, :, N0:] = 0
    grown = Z.Tree(grown_K, grown_V, refs, N0, C, 0, beta)
    # 250 keys: 62, 15, 3 nodes; the 256th key (4^4) completes a group at every level
    assert grown.depth == 3 and grown.level_sizes() == [250, 62, 15, 3]
    for i in range(N0, N0 + M):
        grown.append(K[:, :, i].contiguous(), V[:, :, i].contiguous())
        assert grown.depth == (4 if i + 1 >= 256 else 3), i
    direct = Z.Tree(K, V, refs, N0 + M, C, 0, beta)
    assert direct.depth == 4
    assert grown.level_sizes() == direct.level_sizes() == [280, 70, 17, 4, 1]
    for l in range(1, 5):
        a, n = grown.level(l)
        b, m = direct.level(l)
        assert torch.equal(a[:, :n], b[:, :m])  # same kernel, same inputs: bit-identical
    ot = O.build_tree(host64(K[1, 0, :N0]), host64(refs[0]), C, 0, beta, capacity=N0 + M)
    O.append(ot, host64(K[1, 0]), M)
    assert ot.depth == 4
    for l in range(1, 5):
        g, n = gpu_level(grown, l, 2)
        assert n == ot.n_nodes[l]
        assert_nodes_close(g, *ot.level(l), R, d)
    grown.close()
    direct.close()
    # search and attention on a growing tree against the oracle
    _check_against_oracle(K, V, refs, Q, N0 + M, C, 0, beta, top_width=2,
                          modes=((O.TOP_P, 0.9, 0), (O.TOP_K, 0, 3)))


def test_append_past_capacity_is_refused():
    Z = zha()
    K, V, refs, Q = _tiny(64, C=8, depth=2)
    tree = Z.Tree(K, V, refs, 64, 8, 2, 0.125)
    with pytest.raises(Z.ZhaError) as e:
        tree.append(K[:, :, 0].contiguous(), V[:, :, 0].contiguous())
    assert e.value.code == Z.ERR_CAPACITY
    tree.close()


# ---------------------------------------------------------------------------
# the full-scan indexer


class _Sel:
    def __init__(self, sel, gap, sd):
        self.sel, self.tie_gap, self.tie_sum = sel, gap, sd


def _softmax(s):
    e = np.exp(s - s.max())
    return e / e.sum()


@pytest.mark.parametrize("N,d,dtype,Hq,nq", [(4096, 64, torch.float32, 1, 8), (3001, 128, torch.bfloat16, 4, 2),
                                             (200000, 64, torch.float32, 2, 2), (65536, 128, torch.bfloat16, 4, 8)])
def test_dense_scan_matches_oracle(N, d, dtype, Hq, nq):
    Z = zha()
    K, V, refs, Q = _tiny(N, C=8, depth=3, d=d, R=4, B=2, H=1, Hq=Hq, nq=nq, dtype=dtype, seed=N % 97)
    beta = 1 / np.sqrt(d)
    tree = Z.Tree(K, V, refs, N, 8, 3, beta)
    Qh = host64(Q)
    parted = walks = 0
    for mode, p, k in ((O.TOP_P, 0.9, 0), (O.TOP_P, 0.5, 0), (O.TOP_P, 1.0, 0), (O.TOP_K, 0, 16), (O.TOP_K, 0, 1)):
        sel, cnt = tree.dense_scan(Q, mode, p, k)
        tree.sync_status()
        sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
        for b in range(2):
            Kd = host64(K[b, 0, :N])
            for hq in range(Hq):
                for i in range(nq):
                    wi = (b * Hq + hq) * nq + i
                    s, gap, sd = O.dense_scan(Kd, Qh[b, hq, i], beta, mode, p, k)
                    parted += len(compare_selection(sel, cnt, {wi: _Sel(s, gap, sd)},
                                                    one_level_valid(_softmax(beta * Kd @ Qh[b, hq, i]), mode, p, k)))
                    walks += 1
    assert_partings_bounded(parted, walks)
    tree.close()


@pytest.mark.parametrize("N,d,dtype,Hq,nq,group", [(4096, 64, torch.float32, 1, 8, 16),
                                                   (3001, 128, torch.bfloat16, 4, 2, 16),
                                                   (1000, 64, torch.float32, 1, 4, 1),
                                                   (70001, 128, torch.bfloat16, 4, 1, 16)])
def test_chunk_mass_matches_oracle(N, d, dtype, Hq, nq, group):
    """The chunk-mass profile: per walk the fewest chunks of `group` keys holding p
    of the dense attention, against the oracle (selections may part only at an
    oracle near-tie); with chunks of one key it is the full-scan indexer."""
    Z = zha()
    K, V, refs, Q = _tiny(N, C=8, depth=3, d=d, R=4, B=2, H=1, Hq=Hq, nq=nq, dtype=dtype, seed=N % 89)
    beta = 1 / np.sqrt(d)
    tree = Z.Tree(K, V, refs, N, 8, 3, beta)
    Qh = host64(Q)
    parted = walks = 0
    for p in (0.9, 0.5, 1.0):
        sel, cnt, n_chunks = tree.chunk_mass(Q, group, p)
        tree.sync_status()
        assert n_chunks == (N + group - 1) // group
        sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
        for b in range(2):
            Kd = host64(K[b, 0, :N])
            for hq in range(Hq):
                for i in range(nq):
                    wi = (b * Hq + hq) * nq + i
                    s, nc, gap, sd = O.chunk_mass(Kd, Qh[b, hq, i], beta, group, p)
                    assert nc == n_chunks
                    e = _softmax(beta * Kd @ Qh[b, hq, i])
                    m = np.add.reduceat(e, np.arange(0, N, group))
                    parted += len(compare_selection(sel, cnt, {wi: _Sel(s, gap, sd)},
                                                    one_level_valid(m, O.TOP_P, p, 0)))
                    walks += 1
    assert_partings_bounded(parted, walks)
    if group == 1:
        s1, c1 = tree.dense_scan(Q, O.TOP_P, 0.9, 0)
        s2, c2, _ = tree.chunk_mass(Q, 1, 0.9)
        tree.sync_status()
        assert torch.equal(c1, c2)
        for w in range(c1.numel()):
            assert torch.equal(s1[w, : c1[w]], s2[w, : c2[w]])
    tree.close()


@pytest.mark.parametrize("dtype,d,C,depth", [(torch.float32, 64, 4, 4), (torch.bfloat16, 128, 8, 3)])
def test_ref_grad_matches_oracle(dtype, d, C, depth):
    """The split loss and its gradient with respect to the references against the
    CPU reference (explicit backward in double precision), to what fp32 gives."""
    from oracle import ref_learning as RL

    Z = zha()
    B, H, R, Hq, nq = 1, 2, 3, 4, 2
    N = C ** depth * 2 + 37  # a tail past the last full node
    K, V, refs, Q = _tiny(N, C=C, d=d, R=R, B=B, H=H, Hq=Hq, nq=nq, dtype=dtype, seed=9)
    beta = 0.3
    tree = Z.Tree(K, V, refs, N, C, depth, beta)
    loss, grad = tree.ref_grad(Q)
    tree.sync_status()
    loss, grad = float(loss.item()), grad.double().cpu().numpy()
    group = Hq // H
    Qh = host64(Q)
    losses, grads = [], []
    for h in range(H):
        q = Qh[0, h * group: (h + 1) * group].reshape(-1, d)
        lo, go = RL.split_loss_and_grad(host64(K[0, h, :N]), host64(refs[h]), q, C, depth, beta)
        losses.append(lo)
        grads.append(go / H)  # the GPU averages over all walks of all trees
    loss_err = abs(loss - np.mean(losses)) / max(1.0, abs(np.mean(losses)))
    grad_err = max(np.abs(grad[h] - grads[h]).max() / max(1e-6, np.abs(grads[h]).max()) for h in range(H))
    print(f"ref_grad {dtype}: loss error {loss_err:.3g}, gradient error {grad_err:.3g} of its largest element")
    # fp32 arithmetic over sums of a few thousand terms: observed on B200 1.4e-7 on
    # the loss and 9e-7 (fp32 caches) / 1.5e-6 (bf16) of the largest gradient element
    assert loss_err <= 2e-6, (loss, losses)
    assert grad_err <= 2e-5, grad_err
    tree.close()


def test_rebuild_after_refs_update_equals_build():
    """zha_rebuild after the refs were changed in place equals a fresh build with
    the new refs, bit for bit, and the oracle built with them."""
    Z = zha()
    N, C, depth, d, R = 3000, 8, 3, 128, 8
    K, V, refs, Q = _tiny(N, C=C, depth=depth, d=d, R=R, B=2, H=2, Hq=4, nq=2, dtype=torch.bfloat16, seed=21)
    beta = 1 / np.sqrt(d)
    tree = Z.Tree(K, V, refs, N, C, depth, beta)
    g = torch.Generator(device="cuda").manual_seed(22)
    refs.mul_(0.5).add_(torch.randn(refs.shape, generator=g, device="cuda"))  # in place: the tree keeps the pointer
    launches = Z.kernel_launches()
    tree.rebuild()
    assert Z.kernel_launches() - launches == depth  # one build launch per level, nothing else
    fresh = Z.Tree(K, V, refs.clone(), N, C, depth, beta)
    for l in range(1, depth + 1):
        a, n = tree.level(l)
        b, m = fresh.level(l)
        assert n == m and torch.equal(a[:, :n], b[:, :m])
    ot = O.build_tree(host64(K[1, 1, :N]), host64(refs[1]), C, depth, beta, store=O.STORE_F32)
    for l in range(1, depth + 1):
        gl, n = gpu_level(tree, l, 3)
        assert_nodes_close(gl, *ot.level(l), R, d)
    tree.close()
    fresh.close()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_reference_learning_loop_follows_the_cpu_reference(dtype):
    """Gradient descent on the references on the GPU (zha_ref_grad, an in-place
    update, zha_rebuild) follows the CPU reference's descent (autograd in double
    precision) step by step, and lowers the loss."""
    from oracle import ref_learning as RL

    Z = zha()
    B, H, R, Hq, nq, d, C, depth = 1, 2, 3, 4, 4, 64, 4, 3
    N = C ** depth * 2 + 37
    K, V, refs, Q = _tiny(N, C=C, d=d, R=R, B=B, H=H, Hq=Hq, nq=nq, dtype=dtype, seed=31)
    beta, lr, steps = 0.3, 0.5, 6
    refs0 = refs.clone()
    tree = Z.Tree(K, V, refs, N, C, depth, beta)
    gpu = []
    for _ in range(steps):
        loss, grad = tree.ref_grad(Q)
        gpu.append(float(loss.item()))
        refs.sub_(lr * grad)
        tree.rebuild()
    loss, _ = tree.ref_grad(Q)
    gpu.append(float(loss.item()))
    tree.sync_status()
    tree.close()
    # the GPU loss is the mean over the walks of both trees (equal walks per tree),
    # so its gradient for head h is 1/H of that head's own: the same trajectory as
    # per-head descent with step lr / H
    group = Hq // H
    Qh = host64(Q)
    per_head = []
    for h in range(H):
        q = torch.from_numpy(Qh[0, h * group: (h + 1) * group].reshape(-1, d))
        _, losses = RL.learn_refs(torch.from_numpy(host64(K[0, h, :N])), torch.from_numpy(host64(refs0[h])), q, C,
                                  depth, beta, steps, lr / H)
        per_head.append(losses)
    ref = np.mean(np.array(per_head), axis=0)
    err = np.abs(np.array(gpu) - ref) / np.maximum(1.0, np.abs(ref))
    print("losses (GPU, CPU reference):", list(zip(np.round(gpu, 6), np.round(ref, 6))))
    assert err.max() <= 1e-4, (gpu, ref.tolist())
    assert gpu[-1] < gpu[0]
