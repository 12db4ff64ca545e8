"""Pins of the oracle against what the mathematics and the pages fix.

Page "How does a tree of summaries search a context? How ZHA works":
  * section "What does a node summarize?": a node's estimate is exact at each
    reference query and never exceeds the true log-sum-exp of its region (a
    tangent of a convex function), and merging child nodes equals summarizing the
    original keys directly;
  * section "How does top-p differ from top-K?": top-p opens the smallest group
    holding p of the mass, top-K exactly K;
  * section "How is the tree built?": the original keys are kept and the final
    attention runs on exactly the chosen ones; a node is made when a chunk fills.

The checks below do not call the oracle to get their expected values: they use
closed forms (softmax-weighted means, log-sum-exp, the gradient of log-sum-exp),
textbook dense attention, scipy's logsumexp/softmax, exhaustive subset search on
small frontiers, and counting formulas.
"""
import itertools
from fractions import Fraction

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle as O


def _tree(seed, N, d, R, C, depth, beta, store=O.STORE_F64, zero_ref=False, scale=1.0):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((N, d)) * scale
    refs = rng.standard_normal((R, d))
    if zero_ref:
        refs[0] = 0.0
    return K, refs, O.build_tree(K, refs, C, depth, beta, store=store)


def _leaves(K, C, level, j):
    span = C**level
    return K[j * span:(j + 1) * span]


def _direct(leaves, q, beta):
    """Summary of a region straight from its keys: the softmax-weighted mean key
    and the log-sum-exp corrected by the key's own score."""
    a = beta * leaves @ q
    key = softmax(a) @ leaves
    return key, logsumexp(a) - beta * key @ q


CASES = [
    dict(seed=1, N=256, d=16, R=4, C=4, depth=4, beta=0.25),
    dict(seed=2, N=512, d=32, R=3, C=8, depth=3, beta=1 / np.sqrt(32)),
    dict(seed=3, N=243, d=8, R=5, C=3, depth=5, beta=0.7),
]


@pytest.mark.parametrize("case", CASES)
def test_estimate_exact_at_reference(case):
    K, refs, t = _tree(**case)
    C, beta = case["C"], case["beta"]
    for l in range(1, t.depth + 1):
        keys, bias = t.level(l)
        for j in range(t.n_nodes[l]):
            leaves = _leaves(K, C, l, j)
            for r in range(t.R):
                est = beta * keys[j, r] @ refs[r] + bias[j, r]
                true = logsumexp(beta * leaves @ refs[r])
                assert abs(est - true) <= 1e-12 * max(1.0, abs(true))


@pytest.mark.parametrize("case", CASES)
def test_estimate_is_a_lower_bound(case):
    K, refs, t = _tree(**case)
    C, beta, d = case["C"], case["beta"], case["d"]
    rng = np.random.default_rng(99)
    qs = rng.standard_normal((10000 // t.depth, d)) * rng.uniform(0.1, 3.0, (10000 // t.depth, 1))
    for l in range(1, t.depth + 1):
        keys, bias = t.level(l)
        for j in range(t.n_nodes[l]):
            leaves = _leaves(K, C, l, j)
            est = np.max(beta * np.einsum("rd,qd->qr", keys[j], qs) + bias[j][None, :], axis=1)
            true = logsumexp(beta * qs @ leaves.T, axis=1)
            assert np.all(est <= true + 1e-12 * np.maximum(1.0, np.abs(true)))


@pytest.mark.parametrize("case", CASES)
def test_merged_nodes_equal_direct_summary(case):
    K, refs, t = _tree(**case)
    C, beta = case["C"], case["beta"]
    for l in range(1, t.depth + 1):
        keys, bias = t.level(l)
        for j in range(t.n_nodes[l]):
            leaves = _leaves(K, C, l, j)
            for r in range(t.R):
                key, b = _direct(leaves, refs[r], beta)
                np.testing.assert_allclose(keys[j, r], key, rtol=1e-12, atol=1e-12)
                assert abs(bias[j, r] - b) <= 1e-11 * max(1.0, abs(b))


def test_key_is_gradient_of_logsumexp():
    # key_r = (1/beta) d/dq logsumexp(beta K q) at q = q_r (central differences)
    case = CASES[0]
    K, refs, t = _tree(**case)
    beta, C = case["beta"], case["C"]
    keys, _ = t.level(2)
    leaves = _leaves(K, C, 2, 3)
    h = 1e-5
    for r in range(t.R):
        g = np.zeros(case["d"])
        for i in range(case["d"]):
            e = np.zeros(case["d"])
            e[i] = h
            g[i] = (logsumexp(beta * leaves @ (refs[r] + e)) - logsumexp(beta * leaves @ (refs[r] - e))) / (2 * h)
        np.testing.assert_allclose(keys[3, r], g / beta, rtol=1e-6, atol=1e-8)


def test_zero_reference_gives_mean_and_log_count():
    K, refs, t = _tree(seed=4, N=256, d=16, R=3, C=4, depth=4, beta=0.5, zero_ref=True)
    for l in range(1, 5):
        keys, bias = t.level(l)
        for j in range(t.n_nodes[l]):
            leaves = _leaves(K, 4, l, j)
            np.testing.assert_allclose(keys[j, 0], leaves.mean(axis=0), rtol=1e-12, atol=1e-13)
            assert abs(bias[j, 0] - np.log(len(leaves))) < 1e-12


def test_fp32_storage_stays_close_to_exact():
    K, refs, t64 = _tree(seed=5, N=4096, d=64, R=4, C=4, depth=6, beta=1 / 8)
    t32 = O.build_tree(K, refs, 4, 6, 1 / 8, store=O.STORE_F32)
    for l in range(1, 7):
        k64, b64 = t64.level(l)
        k32, b32 = t32.level(l)
        assert np.all(k32 == k32.astype(np.float32))  # values are fp32
        np.testing.assert_allclose(k32, k64, rtol=2e-6, atol=2e-6 * np.abs(k64).max())
        np.testing.assert_allclose(b32, b64, rtol=2e-6, atol=2e-6 * np.abs(b64).max())


def _dense_attention(K, V, q, beta):
    w = softmax(beta * K @ q)
    return w @ V, logsumexp(beta * K @ q)


@pytest.mark.parametrize("N", [1003, 4096, 517])
def test_p_one_reads_everything_and_equals_dense_attention(N):
    d, R, C, depth, beta = 16, 4, 8, 4, 0.3
    rng = np.random.default_rng(N)
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    refs = rng.standard_normal((R, d))
    t = O.build_tree(K, refs, C, depth, beta)
    q = rng.standard_normal(d) * 2
    w = O.search(t, q, O.TOP_P, 1.0, 0, top_width=64)
    n = t.n_nodes
    s = w.start_level
    assert s == min([l for l in range(1, depth + 1) if n[l] <= 64] or [depth])
    assert list(w.sel) == list(range(n[1]))
    for l in range(1, s + 1):
        assert w.frontier[l] == n[l]  # every node of every level at or below the start
    assert w.keys_read == N
    assert w.work == R * sum(n[1:s + 1]) + N
    out, lse = O.attend(K, V, q, w.sel, C, n[1], beta)
    ref_out, ref_lse = _dense_attention(K, V, q, beta)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-12)
    assert abs(lse - ref_lse) < 1e-12 * abs(ref_lse)


def test_top_k_counts_closed_form():
    # a full tree of 4096 keys, C = 4, six levels: the walk starts at the 64-node
    # level (3); each level opens K nodes, so the next frontier has K*C nodes:
    # work = R*(64 + 2*K*C) + K*C = 472 for K = 6, R = 4.
    K, refs, t = _tree(seed=6, N=4096, d=32, R=4, C=4, depth=6, beta=0.2, store=O.STORE_F32)
    rng = np.random.default_rng(0)
    for _ in range(5):
        w = O.search(t, rng.standard_normal(32), O.TOP_K, 0.0, 6, top_width=64)
        assert w.start_level == 3
        assert w.frontier[1:4] == [24, 24, 64]
        assert w.opened[1:4] == [6, 6, 6]
        assert w.keys_read == 24 and len(w.sel) == 6
        assert w.work == 472


def _exact(m):
    """Masses as exact integers over a common power-of-two denominator, so that
    subset sums and comparisons with p are exact."""
    return [int(Fraction(float(x)) * (1 << 1100)) for x in m], (1 << 1100)


def _brute_walk(t, q, mode, p, k, top_width):
    """Walk by exhaustive subset search at each level (frontiers up to 16), else
    by checking the optimality conditions of the chosen set. Sums are exact."""
    n, R, C, beta = t.n_nodes, t.R, t.C, t.beta
    s = next((l for l in range(1, t.depth + 1) if n[l] <= top_width), t.depth)
    F = list(range(n[s]))
    for l in range(s, 0, -1):
        keys, bias = t.level(l)
        sc = np.array([max(beta * keys[j, r] @ q + bias[j, r] for r in range(R)) for j in F])
        m = softmax(sc)
        mi, one = _exact(m)
        target = Fraction(p) * sum(mi) if p < 1 else None
        if mode == O.TOP_K:
            size = min(k, len(F))
            if len(F) <= 16:
                best = max(itertools.combinations(range(len(F)), size), key=lambda c: sum(mi[i] for i in c))
            else:
                best = tuple(np.argsort(-m, kind="stable")[:size])
        elif p >= 1:
            best = tuple(range(len(F)))
        elif len(F) <= 16:
            best = None
            for size in range(1, len(F) + 1):
                ok = [c for c in itertools.combinations(range(len(F)), size) if sum(mi[i] for i in c) >= target]
                if ok:
                    best = max(ok, key=lambda c: sum(mi[i] for i in c))
                    break
        else:
            order = np.argsort(-m, kind="stable")
            run, size = 0, 0
            while run < target:
                run += mi[order[size]]
                size += 1
            best = tuple(order[:size])
            # optimality: no smaller set reaches p (the size-1 largest masses fall short)
            assert sum(sorted(mi, reverse=True)[: size - 1]) < target
        chosen = sorted(F[i] for i in best)
        if l == 1:
            return chosen
        F = [c * C + i for c in chosen for i in range(C)] + list(range(C * n[l], n[l - 1]))
    return []


@pytest.mark.parametrize("seed", range(12))
@pytest.mark.parametrize("N,C,depth,tw", [(64, 4, 3, 4), (256, 4, 4, 4), (200, 3, 4, 8), (250, 2, 7, 2)])
def test_walk_matches_brute_force(seed, N, C, depth, tw):
    d, R = 8, 3
    rng = np.random.default_rng(1000 * seed + N)
    centres = rng.standard_normal((N // 16 + 1, d)) * 2
    K = centres.repeat(16, axis=0)[:N] + 0.3 * rng.standard_normal((N, d))
    refs = rng.standard_normal((R, d))
    t = O.build_tree(K, refs, C, depth, 0.6, store=O.STORE_F32)
    for qi in range(4):
        q = centres[rng.integers(len(centres))] * rng.uniform(0.5, 2.0) + 0.1 * rng.standard_normal(d)
        for mode, p, k in [(O.TOP_P, 0.9, 0), (O.TOP_P, 0.5, 0), (O.TOP_P, 1.0, 0), (O.TOP_K, 0, 2), (O.TOP_K, 0, 5)]:
            w = O.search(t, q, mode, p, k, top_width=tw)
            if min(w.tie_gap, w.tie_sum) < 1e-12:
                continue  # exact sums and the oracle's double sums may part at a tie
            assert list(w.sel) == _brute_walk(t, q, mode, p, k, tw), (qi, mode, p, k)
            tail = N - C * t.n_nodes[1]
            assert w.keys_read == C * len(w.sel) + tail


def test_orphans_and_tail_join_the_walk():
    # n = [1003, 125, 15, 1]: 5 level-1 orphans (ids 120..124), 3 tail keys
    d, R, C = 8, 2, 8
    rng = np.random.default_rng(7)
    K = rng.standard_normal((1003, d))
    t = O.build_tree(K, rng.standard_normal((R, d)), C, 3, 0.5)
    assert t.n_nodes == [1003, 125, 15, 1]
    w = O.search(t, rng.standard_normal(d), O.TOP_P, 1.0, 0, top_width=64)
    assert w.start_level == 2 and w.frontier[2] == 15 and w.frontier[1] == 125
    assert w.keys_read == 1003
    # with top-K 1, the level-1 frontier is the opened node's 8 children plus the 5 orphans
    w = O.search(t, rng.standard_normal(d), O.TOP_K, 0, 1, top_width=64)
    assert w.frontier[1] == 8 + 5 and w.keys_read == 8 + 3


def test_tree_smaller_than_a_chunk_reads_every_key():
    d = 8
    rng = np.random.default_rng(8)
    K = rng.standard_normal((5, d))
    V = rng.standard_normal((5, d))
    t = O.build_tree(K, rng.standard_normal((2, d)), 8, 3, 0.5)
    assert t.n_nodes == [5, 0, 0, 0]
    q = rng.standard_normal(d)
    w = O.search(t, q, O.TOP_P, 0.9, 0)
    assert len(w.sel) == 0 and w.keys_read == 5 and w.work == 5
    out, lse = O.attend(K, V, q, w.sel, 8, 0, 0.5)
    ref_out, ref_lse = _dense_attention(K, V, q, 0.5)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12)


def test_append_equals_build():
    d, R, C, depth = 16, 3, 4, 4
    rng = np.random.default_rng(9)
    K = rng.standard_normal((1300, d)).astype(np.float32).astype(np.float64)
    refs = rng.standard_normal((R, d))
    grown = O.build_tree(K[:1000], refs, C, depth, 0.3, capacity=1300)
    O.append(grown, K, 300)
    direct = O.build_tree(K, refs, C, depth, 0.3)
    assert grown.n_nodes == direct.n_nodes == [1300, 325, 81, 20, 5]
    for l in range(1, depth + 1):
        a, b = grown.level(l), direct.level(l)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# Depths worked by hand: 4096 = 4^6 keys fill 6 levels; 4095 stop one short
# (1023, 255, 63, 15, 3, then 0); 7 keys fill no chunk of 8 (one empty level);
# 100 keys with C = 8 give 12 and 1; 1003 give 125, 15, 1; 250 with C = 2 give
# 125, 62, 31, 15, 7, 3, 1.
@pytest.mark.parametrize("N,C,D", [(4096, 4, 6), (4095, 4, 5), (7, 8, 1), (100, 8, 2), (1003, 8, 3), (250, 2, 7)])
def test_growing_tree_keeps_every_filled_level(N, C, D):
    d, R = 8, 2
    rng = np.random.default_rng(N + C)
    K = rng.standard_normal((N, d))
    refs = rng.standard_normal((R, d))
    t = O.build_tree(K, refs, C, 0, 0.5)
    assert t.grow and t.depth == D
    # the top level holds a node (when any chunk is full) but never a full group
    # of C, which would have a parent one level up
    assert (t.n_nodes[D] >= 1) == (N >= C)
    assert t.n_nodes[D] < C
    # it is the fixed-depth tree of D levels, walks included
    fixed = O.build_tree(K, refs, C, D, 0.5)
    for l in range(1, D + 1):
        a, b = t.level(l), fixed.level(l)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    for qi in range(3):
        q = rng.standard_normal(d)
        w, v = O.search(t, q, O.TOP_P, 0.9, 0, top_width=4), O.search(fixed, q, O.TOP_P, 0.9, 0, top_width=4)
        assert list(w.sel) == list(v.sel) and w.start_level == v.start_level


def test_append_grows_the_depth_at_a_full_top_group():
    # C = 4: 60 keys give 15 and 3 nodes (depth 2); the 64th key completes the 16th
    # level-1 node, which completes the 4th level-2 node, whose group of 4 gets a
    # parent: depth 3
    d, R, C = 8, 3, 4
    rng = np.random.default_rng(11)
    K = rng.standard_normal((80, d)).astype(np.float32).astype(np.float64)
    refs = rng.standard_normal((R, d))
    grown = O.build_tree(K[:60], refs, C, 0, 0.4, capacity=80)
    assert grown.depth == 2 and grown.max_depth == 3
    O.append(grown, K, 3)
    assert grown.depth == 2 and grown.n_nodes == [63, 15, 3, 0]
    O.append(grown, K, 1)
    assert grown.depth == 3 and grown.n_nodes == [64, 16, 4, 1]
    direct = O.build_tree(K[:64], refs, C, 0, 0.4, capacity=80)
    assert direct.depth == 3 and direct.n_nodes == grown.n_nodes
    for l in range(1, 4):
        a, b = grown.level(l), direct.level(l)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    for qi in range(4):
        q = rng.standard_normal(d) * 2
        for mode, p, k in [(O.TOP_P, 0.9, 0), (O.TOP_K, 0, 3)]:
            w = O.search(grown, q, mode, p, k, top_width=2)
            assert w.start_level == 3
            if min(w.tie_gap, w.tie_sum) < 1e-12:
                continue
            assert list(w.sel) == _brute_walk(grown, q, mode, p, k, 2)


def test_chunk_mass_of_single_keys_is_the_dense_scan():
    # chunks of one key: the fewest keys reaching p, the full-scan indexer's top-p
    # (computed by the C oracle, independently)
    rng = np.random.default_rng(12)
    K = rng.standard_normal((500, 16))
    for i in range(6):
        q = rng.standard_normal(16) * (0.5 + i)
        for p in (0.5, 0.9, 0.99):
            sel, n_chunks, gap, tsum = O.chunk_mass(K, q, 0.7, group=1, p=p)
            ref, _, _ = O.dense_scan(K, q, 0.7, O.TOP_P, p, 0)
            assert n_chunks == 500 and list(sel) == list(ref), (i, p)


def test_chunk_mass_closed_forms():
    rng = np.random.default_rng(13)
    # q = 0: every key weighs 1/n, so a chunk weighs its key count / n.
    # 64 keys in 4 chunks of 16: 0.25 each, exact in binary: p = 0.75 takes 3, 0.9 takes 4
    K = rng.standard_normal((64, 8))
    q = np.zeros(8)
    sel, n_chunks, _, _ = O.chunk_mass(K, q, 1.0, 16, 0.75)
    assert n_chunks == 4 and list(sel) == [0, 1, 2]
    assert list(O.chunk_mass(K, q, 1.0, 16, 0.9)[0]) == [0, 1, 2, 3]
    assert list(O.chunk_mass(K, q, 1.0, 16, 0.5)[0]) == [0, 1]
    # 40 keys: chunks of 16, 16 and a partial 8 weigh 0.4, 0.4, 0.2; ties to the lower chunk
    K = rng.standard_normal((40, 8))
    sel, n_chunks, _, _ = O.chunk_mass(K, np.zeros(8), 1.0, 16, 0.3)
    assert n_chunks == 3 and list(sel) == [0]
    assert list(O.chunk_mass(K, np.zeros(8), 1.0, 16, 0.9)[0]) == [0, 1, 2]
    # one key far above the rest: its chunk alone holds almost all the mass
    K = rng.standard_normal((256, 8)) * 0.01
    K[37] = 10.0
    q = np.ones(8)
    sel, n_chunks, _, _ = O.chunk_mass(K, q, 1.0, 16, 0.9)
    assert n_chunks == 16 and list(sel) == [37 // 16]
    # p >= 1 takes every chunk
    assert list(O.chunk_mass(K, q, 1.0, 16, 1.0)[0]) == list(range(16))


@pytest.mark.parametrize("seed", range(8))
def test_chunk_mass_count_is_the_minimum(seed):
    # no smaller set of chunks reaches p (exhaustive over tiny inputs, exact sums)
    rng = np.random.default_rng(100 + seed)
    n, g = int(rng.integers(20, 80)), int(rng.integers(4, 9))
    K = rng.standard_normal((n, 6))
    q = rng.standard_normal(6) * rng.uniform(0.5, 3.0)
    for p in (0.5, 0.8, 0.9):
        sel, n_chunks, gap, tsum = O.chunk_mass(K, q, 1.0, g, p)
        if min(gap, tsum) < 1e-12:
            continue
        s = K @ q
        w = np.exp(s - s.max())
        m = [Fraction(float(x)) for x in np.add.reduceat(w, np.arange(0, n, g))]
        total = sum(m)
        assert sum(m[c] for c in sel) >= Fraction(p) * total
        smaller = [c for c in itertools.combinations(range(n_chunks), len(sel) - 1)
                   if sum(m[i] for i in c) >= Fraction(p) * total]
        assert not smaller, (seed, p, len(sel))


def test_attend_on_a_subset_is_softmax_attention():
    rng = np.random.default_rng(10)
    N, d, C = 333, 12, 4
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    q = rng.standard_normal(d)
    n1 = N // C
    sel = np.sort(rng.choice(n1, 17, replace=False))
    idx = np.concatenate([np.arange(j * C, j * C + C) for j in sel] + [np.arange(C * n1, N)])
    out, lse = O.attend(K, V, q, sel, C, n1, 0.4)
    ref_out, ref_lse = _dense_attention(K[idx], V[idx], q, 0.4)
    np.testing.assert_allclose(out, ref_out, rtol=1e-12, atol=1e-14)
    assert abs(lse - ref_lse) < 1e-12 * max(1, abs(ref_lse))
    kept = O.kept_mass(K, q, 0.4, sel, C, n1)
    assert abs(kept - softmax(0.4 * K @ q)[idx].sum()) < 1e-12


def test_dense_scan_selects_by_exact_softmax():
    rng = np.random.default_rng(11)
    K = rng.standard_normal((14, 6))
    q = rng.standard_normal(6) * 2
    m = softmax(0.5 * K @ q)
    sel, gap, _ = O.dense_scan(K, q, 0.5, O.TOP_K, 0, 4)
    assert set(sel) == set(np.argsort(-m)[:4].tolist())
    for p in (0.3, 0.6, 0.9, 0.99):
        sel, _, sd = O.dense_scan(K, q, 0.5, O.TOP_P, p, 0)
        for size in range(1, 15):
            ok = [c for c in itertools.combinations(range(14), size) if m[list(c)].sum() >= p]
            if ok:
                break
        assert len(sel) == size and m[sel].sum() == pytest.approx(max(m[list(c)].sum() for c in ok))
    sel, _, _ = O.dense_scan(K, q, 0.5, O.TOP_P, 1.0, 0)
    assert list(sel) == list(range(14))


def test_tie_measures_flag_exact_ties():
    rng = np.random.default_rng(12)
    K = rng.standard_normal((10, 4))
    K[7] = K[3]  # two keys with the same score
    q = rng.standard_normal(4)
    s = 0.5 * K @ q
    rank = int(np.where(np.argsort(-s, kind="stable") == 3)[0][0])
    k = min(rank, int(np.where(np.argsort(-s, kind="stable") == 7)[0][0])) + 1
    sel, gap, _ = O.dense_scan(K, q, 0.5, O.TOP_K, 0, k)
    assert gap == 0.0
    assert 3 in sel and 7 not in sel  # the tie goes to the lower index
