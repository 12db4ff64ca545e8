"""The walks a query may take when a level's choice sits at a near-tie.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT. Like the rest of ``oracle/``, only
``tests/``, the smoke check and ``bench.py``'s CPU legs may import it; it shares no
code with the CUDA library.

The walk's choice at one level (page "How does a tree of summaries search a
context? How ZHA works", section "How does top-p differ from top-K?": top-p opens
the smallest group of nodes whose mass reaches p, top-K exactly K nodes; section
"Run a small tree yourself", route: the softmax over the whole frontier, sorted by
mass, then the prefix) is unique in exact arithmetic once ties are broken by node
id. A GPU computes the masses in fp32, so where two masses, or the running sum and
p, are closer than its rounding, it may take the other side. This module lists
every choice that is correct within a relative tolerance ``tol`` of the exact
masses, and follows each of them down the tree.

A set A of frontier nodes (masses m, exact softmax of the level's scores in
double) is admissible at tolerance tol when:
  (i)   it is mass-ordered up to tol: min over A of m >= (1 - tol) * max over the
        rest of m (no node left out beats a node taken by more than tol);
  top-K:  (ii) |A| = min(K, |F|);
  top-p, p < 1:
        (ii)  sum over A of m >= p * (1 - tol)   (it reaches p, within tol);
        (iii) sum over A of m - min over A of m < p * (1 + tol)   (dropping its
              smallest node leaves less than p, within tol: it is the smallest
              such group);
  top-p, p >= 1: A is the whole frontier (both sides open every node).
At tol = 0 with distinct masses the only admissible set is the oracle's own
choice (the shortest mass-ordered prefix reaching p, or the K largest).

The scores are the oracle's: max over r of beta * <key_r, q> + bias_r on the
stored (fp32-rounded) node keys and biases of an ``oracle.Tree``, in double.
"""
from __future__ import annotations

from itertools import combinations
from math import comb

import numpy as np

from . import TOP_K, TOP_P

MAX_PATHS = 4096  # walks followed at most (each near-tie level multiplies them)


class TooManyTies(RuntimeError):
    """The tolerance admits more alternative walks than ``MAX_PATHS``."""


def level_masses(t, l: int, F: np.ndarray, q: np.ndarray) -> np.ndarray:
    """Exact softmax over the frontier F (level-l node ids) of the node scores."""
    if len(F) == 0:
        return np.zeros(0)
    keys, bias = t.keys[l][F], t.bias[l][F]
    s = (t.beta * np.einsum("jrd,d->jr", keys, q) + bias).max(axis=1)
    e = np.exp(s - s.max())
    return e / e.sum()


def admissible(m: np.ndarray, A: np.ndarray, mode: int, p: float, k: int, tol: float) -> bool:
    """Whether the positions A (a boolean mask over the frontier) are an
    admissible choice for the masses m (the definition in the module docstring)."""
    F = len(m)
    n = int(A.sum())
    if F == 0:
        return n == 0
    if mode == TOP_P and p >= 1:
        return n == F
    if n == 0:
        return False
    lo = m[A].min()
    hi = m[~A].max() if n < F else -np.inf
    if lo < (1 - tol) * hi:
        return False
    if mode == TOP_K:
        return n == min(k, F)
    total = m[A].sum()
    return total >= p * (1 - tol) and total - lo < p * (1 + tol)


def level_choices(m: np.ndarray, mode: int, p: float, k: int, tol: float) -> list:
    """Every admissible choice at one level, as boolean masks over the frontier.

    Sizes: top-K takes min(K, |F|); top-p the sizes whose mass-ordered prefix
    could meet (ii) and (iii). For a size c, with the masses sorted descending
    (ties by position), a set can only be admissible if it holds every node whose
    mass exceeds ms[c] / (1 - tol) and none whose mass is below (1 - tol) *
    ms[c - 1]: otherwise (i) fails. The nodes in between (the band) are tried in
    every combination and each candidate is checked against the definition."""
    F = len(m)
    if F == 0:
        return [np.zeros(0, dtype=bool)]
    if mode == TOP_P and p >= 1:
        return [np.ones(F, dtype=bool)]
    order = np.lexsort((np.arange(F), -m))
    ms = m[order]
    if mode == TOP_K:
        sizes = [min(k, F)]
    else:
        cum = np.cumsum(ms)
        slack = 4 * tol
        sizes = [c for c in range(1, F + 1)
                 if cum[c - 1] >= p * (1 - tol) - slack and (cum[c - 2] if c >= 2 else 0.0) < p * (1 + tol) + slack]
    out = []
    for c in sizes:
        upper = ms[c] / (1 - tol) if c < F else -np.inf
        lower = (1 - tol) * ms[c - 1]
        must = [i for i in range(F) if ms[i] > upper and i < c]
        band = [i for i in range(F) if i not in must and ms[i] >= lower]
        need = c - len(must)
        if need < 0 or need > len(band):
            continue
        if comb(len(band), need) > MAX_PATHS:
            raise TooManyTies(f"{comb(len(band), need)} near-equal choices at one level")
        for pick in combinations(band, need):
            A = np.zeros(F, dtype=bool)
            A[order[must]] = True
            A[order[list(pick)]] = True
            if admissible(m, A, mode, p, k, tol):
                out.append(A)
    return out


def admissible_selections(t, q, mode: int = TOP_P, p: float = 0.9, k: int = 1, top_width: int = 64,
                          tol: float = 1e-5) -> set:
    """The level-1 chunk sets (sorted tuples of node ids) of every walk of q down
    the oracle tree t whose choice at each level is admissible at tolerance tol.
    The walk starts, expands and ends as the oracle's search does: at the lowest
    level with at most top_width nodes (else the deepest), children of the opened
    nodes then the orphans of the level below, the opened level-1 ids as result."""
    q = np.asarray(q, dtype=np.float64)
    n = t.n_nodes
    depth = t.depth
    s = next((l for l in range(1, depth + 1) if n[l] <= top_width), depth)
    results = set()
    stack = [(s, np.arange(n[s], dtype=np.int64))]
    paths = 0
    while stack:
        l, F = stack.pop()
        m = level_masses(t, l, F, q)
        for A in level_choices(m, mode, p, k, tol):
            opened = np.sort(F[A])
            if l == 1:
                results.add(tuple(int(x) for x in opened))
                continue
            children = (opened[:, None] * t.C + np.arange(t.C)[None, :]).reshape(-1)
            orphans = np.arange(t.C * n[l], n[l - 1], dtype=np.int64)
            stack.append((l - 1, np.concatenate([children, orphans]).astype(np.int64)))
            paths += 1
            if paths > MAX_PATHS:
                raise TooManyTies(f"more than {MAX_PATHS} admissible walks")
    return results
