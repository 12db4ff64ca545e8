"""Pins of the near-tie enumerator (``oracle/ties.py``): the walks a query may take
when a level's choice is within a relative tolerance of a tie.

  * at tolerance 0 (and masses without exact ties) the only admissible walk is the
    one the exhaustive subset search of ``test_oracle_pins._brute_walk`` finds,
    which is the oracle's walk (page "How does top-p differ from top-K?": the
    smallest group reaching p, exactly K);
  * the band enumeration of one level returns exactly the subsets that pass the
    admissibility test, checked over every subset of frontiers of up to 12 nodes
    with planted near-equal masses and sums near p;
  * a choice made exactly on masses perturbed by a relative eps (what fp32
    arithmetic does to them) is admissible at tolerance 8 * eps / p: the property
    the GPU parity tests rely on;
  * two identical subtrees make an exact tie at level 2: with K = 1 the two
    walks differ only by which subtree they enter, and the level-1 chunks of the
    second are those of the first shifted by the subtrees' offset.
"""
import itertools

import numpy as np
import pytest

import oracle as O
from oracle import ties as T
from test_oracle_pins import _brute_walk

MODES = [(O.TOP_P, 0.9, 0), (O.TOP_P, 0.5, 0), (O.TOP_P, 1.0, 0), (O.TOP_K, 0, 2), (O.TOP_K, 0, 5)]


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("N,C,depth,tw", [(64, 4, 3, 4), (256, 4, 4, 4), (200, 3, 4, 8), (1003, 8, 3, 64)])
def test_zero_tolerance_is_the_brute_force_walk(seed, N, C, depth, tw):
    d, R = 8, 3
    rng = np.random.default_rng(7000 + 100 * seed + N)
    centres = rng.standard_normal((N // 16 + 1, d)) * 2
    K = centres.repeat(16, axis=0)[:N] + 0.3 * rng.standard_normal((N, d))
    refs = rng.standard_normal((R, d))
    t = O.build_tree(K, refs, C, depth, 0.6, store=O.STORE_F32)
    for qi in range(3):
        q = centres[rng.integers(len(centres))] * rng.uniform(0.5, 2.0) + 0.1 * rng.standard_normal(d)
        for mode, p, k in MODES:
            w = O.search(t, q, mode, p, k, top_width=tw)
            if min(w.tie_gap, w.tie_sum) < 1e-12:
                continue
            got = T.admissible_selections(t, q, mode, p, k, tw, tol=0.0)
            assert got == {tuple(w.sel)}, (qi, mode, p, k)
            if N <= 256:
                assert got == {tuple(_brute_walk(t, q, mode, p, k, tw))}


def _planted_masses(rng, F, gap=2e-5):
    """Masses with a pair at a random rank whose relative gap is below ``gap``."""
    m = rng.exponential(1.0, F)
    m /= m.sum()
    order = np.argsort(-m)
    r = int(rng.integers(0, F - 1))
    a, b = order[r], order[r + 1]
    m[b] = m[a] * (1 - rng.uniform(0, gap))
    m /= m.sum()
    return m


@pytest.mark.parametrize("seed", range(40))
def test_band_enumeration_is_every_admissible_subset(seed):
    rng = np.random.default_rng(seed)
    F = int(rng.integers(1, 13))
    m = _planted_masses(rng, F) if F > 1 else np.ones(1)
    # top-p with p placed at a prefix sum, just below or above it
    order = np.argsort(-m)
    cum = np.cumsum(m[order])
    p_at = float(cum[int(rng.integers(0, F))]) * (1 + rng.uniform(-2e-5, 2e-5))
    for mode, p, k in [(O.TOP_P, min(p_at, 0.999999), 0), (O.TOP_P, 0.5, 0), (O.TOP_P, 1.0, 0),
                       (O.TOP_K, 0, int(rng.integers(1, F + 1)))]:
        for tol in (0.0, 1e-5, 1e-3):
            got = {tuple(np.flatnonzero(A)) for A in T.level_choices(m, mode, p, k, tol)}
            want = set()
            for bits in itertools.product([False, True], repeat=F):
                A = np.array(bits, dtype=bool)
                if T.admissible(m, A, mode, p, k, tol):
                    want.add(tuple(np.flatnonzero(A)))
            assert got == want, (F, mode, p, k, tol)
            assert got, "some choice is always admissible"


@pytest.mark.parametrize("seed", range(200))
def test_choice_on_perturbed_masses_is_admissible(seed):
    """The pair of near-equal masses sits at the boundary of the choice (rank r and
    r + 1), and top-p's p within a relative eps of the prefix sum through rank r,
    so the perturbation can flip both the order and the stopping point."""
    rng = np.random.default_rng(100 + seed)
    F = int(rng.integers(3, 200))
    m = rng.exponential(1.0, F)
    m /= m.sum()
    order = np.argsort(-m)
    r = int(rng.integers(0, F - 2))
    m[order[r + 1]] = m[order[r]] * (1 - rng.uniform(0, 2e-6))
    m /= m.sum()
    order = np.lexsort((np.arange(F), -m))
    cum = np.cumsum(m[order])
    tol = 1e-5
    for mode, p, k in [(O.TOP_P, float(cum[r]) * (1 + rng.uniform(-1e-6, 1e-6)), 0), (O.TOP_K, 0, r + 1)]:
        if mode == O.TOP_P and not 0 < p < 1:
            continue
        eps = tol * (p if mode == O.TOP_P else 1.0) / 8
        mp = m * (1 + rng.uniform(-eps, eps, F))
        # the exact choice on the perturbed masses: sort, then prefix or K largest
        po = np.lexsort((np.arange(F), -mp))
        if mode == O.TOP_K:
            c = min(k, F)
        else:
            c = int(np.searchsorted(np.cumsum(mp[po]), p, side="left")) + 1
        A = np.zeros(F, dtype=bool)
        A[po[:c]] = True
        assert T.admissible(m, A, mode, p, k, tol)
        assert any(np.array_equal(A, B) for B in T.level_choices(m, mode, p, k, tol))


def test_exact_tie_at_level_two_gives_both_subtrees():
    rng = np.random.default_rng(5)
    C, d, R = 4, 8, 3
    N = C ** 3  # depth 3, one node at level 3, four at level 2
    K = rng.standard_normal((N, d))
    span = C * C
    K[2 * span: 3 * span] = K[0: span]  # level-2 nodes 0 and 2 summarize the same keys
    refs = rng.standard_normal((R, d))
    t = O.build_tree(K, refs, C, 3, 0.5, store=O.STORE_F32)
    assert np.array_equal(t.keys[2][0], t.keys[2][2]) and np.array_equal(t.bias[2][0], t.bias[2][2])
    # a query near the duplicated region, so that nodes 0 and 2 lead level 2
    q = K[0:span].mean(axis=0) * 3
    w = O.search(t, q, O.TOP_K, 0, 1, top_width=4)
    assert w.start_level == 2 and w.tie_gap == 0.0
    got = T.admissible_selections(t, q, O.TOP_K, 0, 1, top_width=4, tol=1e-5)
    shifted = tuple(int(x) + 2 * C for x in w.sel)  # the same child of level-2 node 2
    assert got == {tuple(w.sel), shifted}
    assert all(x < C for x in w.sel)  # the oracle's own walk enters node 0 (lower id)


def test_too_many_ties_is_refused():
    m = np.full(40, 1 / 40)  # forty equal masses: C(40, 20) choices
    with pytest.raises(T.TooManyTies):
        T.level_choices(m, O.TOP_K, 0, 20, 1e-5)
