"""ZHA oracle: ctypes binding of the plain C oracle in ``zha_oracle.c``.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT. Only ``tests/``, the smoke check in
``__graft_entry__.py`` and the ``cpu_baseline`` leg (and reference arm) of
``bench.py`` may import this package. It shares no code with the CUDA library in
``tree_indexed_sparse_append_b200`` and never imports it.

The arithmetic lives in ``zha_oracle.c`` (double precision); this file only
marshals numpy arrays and keeps the per-level arrays of one tree. The tree
shape follows page "How does a tree of summaries search a context? How ZHA
works", sections "How is the tree built?" and "Run a small tree yourself":
level l has floor(n_{l-1} / C) nodes, node j summarizing nodes C*j .. C*j+C-1
of level l-1, and a node is made when its chunk fills. A tree built with depth 0
grows its depth with the keys (page "Subquadratic Attention with a Hierarchical
Tree-Structured Indexer", abstract: the tree's depth grows with the context): it
keeps every level that holds a node, and the parent made when a group of C top
nodes fills starts a new level.

Two modules sit beside it: ``ref_learning.py`` (the loss that teaches the
reference queries and its gradient, in double precision) and
``context_parallel.py`` (the walk of one tree whose keys are split across the
ranks of a process group).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zha_oracle.c")
_HDR = os.path.join(_HERE, "zha_oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

TOP_P = 0
TOP_K = 1
MAX_LEVELS = 16
ROUND_KEYS = 1
ROUND_BIAS = 2
STORE_F32 = ROUND_KEYS | ROUND_BIAS  # node keys and biases stored as fp32
STORE_F64 = 0  # nothing rounded: exact double arithmetic, for the mathematical pins

_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_llp = ctypes.POINTER(ctypes.c_longlong)
_ip = ctypes.POINTER(ctypes.c_int)


def build_library(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (no fast-math) if it is missing or stale."""
    stale = (not os.path.exists(_LIB)) or any(
        os.path.getmtime(src) > os.path.getmtime(_LIB) for src in (_SRC, _HDR)
    )
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fno-fast-math", "-ffp-contract=off",
               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build_library()
            L = ctypes.CDLL(_LIB)
            L.orc_summarize.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                        _dp, ctypes.c_longlong, ctypes.c_longlong, _dp,
                                        ctypes.c_longlong, _dp, ctypes.c_int, _dp, _dp]
            L.orc_build_level1.argtypes = [ctypes.c_longlong, ctypes.c_int, _dp, ctypes.c_int, _dp,
                                           ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                           ctypes.c_longlong, ctypes.c_longlong, _dp, _dp,
                                           ctypes.c_int]
            L.orc_build_level_up.argtypes = [ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, ctypes.c_int,
                                             ctypes.c_double, ctypes.c_int, ctypes.c_longlong,
                                             ctypes.c_longlong, _dp, _dp, ctypes.c_int]
            L.orc_search.argtypes = [ctypes.c_int, _llp, ctypes.POINTER(_dp), ctypes.POINTER(_dp),
                                     ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                     ctypes.c_int, _dp, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                     _llp, ctypes.c_longlong, _llp, _llp, _llp, _ip, _llp, _llp,
                                     _dp, _dp]
            L.orc_attend.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_double, _dp, _dp, _dp,
                                     _llp, ctypes.c_longlong, ctypes.c_int, ctypes.c_longlong,
                                     _dp, _dp]
            L.orc_dense_scan.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_double, _dp, _dp,
                                         ctypes.c_int, ctypes.c_double, ctypes.c_int, _llp,
                                         ctypes.c_longlong, _llp, _dp, _dp]
            L.orc_kept_mass.argtypes = [ctypes.c_longlong, ctypes.c_int, ctypes.c_double, _dp, _dp,
                                        _llp, ctypes.c_longlong, ctypes.c_int, ctypes.c_longlong]
            L.orc_kept_mass.restype = ctypes.c_double
            _lib = L
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def _pl(a: np.ndarray):
    return a.ctypes.data_as(_llp)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with status {rc}")


def summarize(child_keys, child_bias, refs, beta: float, store: int = STORE_F64):
    """One node from explicit children.

    ``child_keys`` is [n][R][d] (or [n][d] for leaves, shared by every reference);
    ``child_bias`` is [n][R] or None (zero). Returns (keys [R][d], biases [R]).
    """
    refs = _f64(refs)
    R, d = refs.shape
    ck = _f64(child_keys)
    n = ck.shape[0]
    if ck.ndim == 2:
        s_child, s_ref = d, 0
    else:
        s_child, s_ref = R * d, d
    keys = np.zeros((R, d))
    bias = np.zeros(R)
    if child_bias is None:
        cb_ptr, cb_stride = None, 0
        cb = None
    else:
        cb = _f64(child_bias)
        cb_ptr, cb_stride = _p(cb), R
    _check(lib().orc_summarize(n, R, d, beta, _p(ck), s_child, s_ref, cb_ptr, cb_stride, _p(refs),
                               store, _p(keys), _p(bias)), "summarize")
    return keys, bias


@dataclass
class Tree:
    """The levels of one tree: ``keys[l]`` is [n_l][R][d], ``bias[l]`` is [n_l][R]
    (index 0 unused). Arrays are allocated for ``capacity`` keys so that the tree
    can grow by appends; ``n_nodes[l]`` is the live count."""

    C: int
    depth: int
    beta: float
    R: int
    d: int
    store: int
    refs: np.ndarray
    n_nodes: list = field(default_factory=list)
    keys: list = field(default_factory=list)
    bias: list = field(default_factory=list)
    grow: bool = False  # depth follows the key count
    max_depth: int = 0  # levels with storage (depth unless the tree grows)

    @property
    def n_keys(self) -> int:
        return self.n_nodes[0]

    def level(self, l: int):
        n = self.n_nodes[l]
        return self.keys[l][:n], self.bias[l][:n]


def _alloc_tree(capacity: int, refs, C: int, depth: int, beta: float, store: int) -> Tree:
    refs = _f64(refs)
    R, d = refs.shape
    t = Tree(C=C, depth=depth, beta=float(beta), R=R, d=d, store=store, refs=refs, max_depth=depth)
    t.n_nodes = [0] * (depth + 1)
    t.keys = [None] * (depth + 1)
    t.bias = [None] * (depth + 1)
    cap = capacity
    for l in range(1, depth + 1):
        cap //= C
        t.keys[l] = np.zeros((max(cap, 1), R, d))
        t.bias[l] = np.zeros((max(cap, 1), R))
    return t


def _build_nodes(t: Tree, K: np.ndarray, l: int, begin: int, end: int, threads: int):
    if end <= begin:
        return
    L = lib()
    if l == 1:
        _check(L.orc_build_level1(K.shape[0], t.d, _p(K), t.R, _p(t.refs), t.C, t.beta, t.store,
                                  begin, end, _p(t.keys[1]), _p(t.bias[1]), threads), "level-1 build")
    else:
        _check(L.orc_build_level_up(t.d, t.R, _p(t.keys[l - 1]), _p(t.bias[l - 1]), _p(t.refs), t.C,
                                    t.beta, t.store, begin, end, _p(t.keys[l]), _p(t.bias[l]),
                                    threads), f"level-{l} build")


def levels_filled(count: int, C: int, limit: int = MAX_LEVELS - 1) -> int:
    """The number of levels ``count`` keys fill with at least one node each (at
    least 1, at most ``limit``)."""
    levels, n = 0, count
    while levels < limit:
        n //= C
        if n < 1:
            break
        levels += 1
    return max(levels, 1)


def build_tree(K, refs, C: int, depth: int, beta: float, store: int = STORE_F32,
               threads: int = 0, capacity: int | None = None, max_levels: int = MAX_LEVELS - 1) -> Tree:
    """Build every level of the tree over the keys ``K`` [N][d] (exact doubles).
    depth >= 1: that many levels. depth == 0: the depth grows with the keys, every
    level holding a node is kept (at most ``max_levels``), with storage for every
    level the capacity can fill."""
    K = _f64(K)
    N = K.shape[0]
    cap = max(N, capacity or 0)
    grow = depth == 0
    levels = levels_filled(cap, C, max_levels) if grow else depth
    t = _alloc_tree(cap, refs, C, levels, beta, store)
    t.grow = grow
    t.n_nodes[0] = N
    n = N
    for l in range(1, levels + 1):
        n //= C
        t.n_nodes[l] = n
        _build_nodes(t, K, l, 0, n, threads)
    if grow:
        t.depth = max([1] + [l for l in range(1, levels + 1) if t.n_nodes[l] > 0])
    return t


def append(t: Tree, K_all, count: int, threads: int = 0) -> None:
    """Append ``count`` keys one at a time (the keys are ``K_all[n0 : n0+count]``,
    where n0 is the current key count). Each time a chunk fills, its level-1 node is
    made; each time a group of C nodes fills at level l < depth, its parent is made
    (for a growing tree, up to the deepest level with storage: the parent of a full
    top group starts a new level)."""
    K = _f64(K_all)
    for _ in range(count):
        n0 = t.n_nodes[0] + 1
        if n0 > K.shape[0]:
            raise ValueError("append past the keys provided")
        t.n_nodes[0] = n0
        below = n0
        for l in range(1, t.max_depth + 1):
            if below % t.C != 0:
                break
            j = below // t.C - 1
            if j + 1 > t.keys[l].shape[0]:
                raise ValueError("append past the tree's capacity")
            _build_nodes(t, K, l, j, j + 1, threads)
            t.n_nodes[l] = j + 1
            if l > t.depth:
                t.depth = l
            below = j + 1


@dataclass
class Walk:
    sel: np.ndarray  # opened level-1 node ids, ascending
    frontier: list  # frontier size per level (index 0 unused)
    opened: list
    start_level: int
    keys_read: int
    work: int
    tie_gap: float
    tie_sum: float


def search(t: Tree, q, mode: int = TOP_P, p: float = 0.9, k: int = 1, top_width: int = 64) -> Walk:
    """One walk of query ``q`` [d] down the tree."""
    L = lib()
    q = _f64(q)
    nn = np.array(t.n_nodes + [0] * (MAX_LEVELS - len(t.n_nodes)), dtype=np.int64)
    live = [None] + [np.ascontiguousarray(t.keys[l]) for l in range(1, t.depth + 1)]
    liveb = [None] + [np.ascontiguousarray(t.bias[l]) for l in range(1, t.depth + 1)]
    kp = (_dp * (t.depth + 1))(*([None] + [_p(a) for a in live[1:]]))
    bp = (_dp * (t.depth + 1))(*([None] + [_p(a) for a in liveb[1:]]))
    max_sel = max(t.n_nodes[1], 1)
    sel = np.zeros(max_sel, dtype=np.int64)
    n_sel = ctypes.c_longlong(0)
    fr = np.zeros(MAX_LEVELS, dtype=np.int64)
    op = np.zeros(MAX_LEVELS, dtype=np.int64)
    s = ctypes.c_int(0)
    kr = ctypes.c_longlong(0)
    wk = ctypes.c_longlong(0)
    tg = ctypes.c_double(0)
    ts = ctypes.c_double(0)
    _check(L.orc_search(t.depth, _pl(nn), kp, bp, t.R, t.d, t.C, t.beta, top_width, _p(q), mode,
                        float(p), int(k), _pl(sel), max_sel, ctypes.byref(n_sel), _pl(fr), _pl(op),
                        ctypes.byref(s), ctypes.byref(kr), ctypes.byref(wk), ctypes.byref(tg),
                        ctypes.byref(ts)), "search")
    return Walk(sel=sel[: n_sel.value].copy(), frontier=fr[: t.depth + 1].tolist(),
                opened=op[: t.depth + 1].tolist(), start_level=s.value, keys_read=kr.value,
                work=wk.value, tie_gap=tg.value, tie_sum=ts.value)


def attend(K, V, q, sel, C: int, n1: int, beta: float):
    """Attention of ``q`` over the keys of the chunks ``sel`` plus the tail
    [C*n1, N). Returns (out [d], lse)."""
    K = _f64(K)
    V = _f64(V)
    q = _f64(q)
    sel = np.ascontiguousarray(np.asarray(sel, dtype=np.int64))
    out = np.zeros(K.shape[1])
    lse = ctypes.c_double(0)
    _check(lib().orc_attend(K.shape[0], K.shape[1], beta, _p(K), _p(V), _p(q), _pl(sel), sel.size,
                            C, n1, _p(out), ctypes.byref(lse)), "attend")
    return out, lse.value


def dense_scan(K, q, beta: float, mode: int = TOP_P, p: float = 0.9, k: int = 1):
    """Full-scan indexer: returns (selected key ids ascending, tie_gap, tie_sum)."""
    K = _f64(K)
    q = _f64(q)
    sel = np.zeros(K.shape[0], dtype=np.int64)
    n = ctypes.c_longlong(0)
    tg = ctypes.c_double(0)
    ts = ctypes.c_double(0)
    _check(lib().orc_dense_scan(K.shape[0], K.shape[1], beta, _p(K), _p(q), mode, float(p), int(k),
                                _pl(sel), sel.size, ctypes.byref(n), ctypes.byref(tg),
                                ctypes.byref(ts)), "dense scan")
    return sel[: n.value].copy(), tg.value, ts.value


def chunk_mass(K, q, beta: float, group: int = 16, p: float = 0.9):
    """How concentrated the dense attention of ``q`` is over chunks of keys (page
    "How does a tree of summaries search a context? How ZHA works", section "How
    does top-p differ from top-K?": the share of 16-key chunks holding 90% of the
    attention). The softmax of beta*<q, k_j> over all keys, summed over
    consecutive chunks of ``group`` keys (the last may be partial); the fewest
    chunks whose masses reach ``p``, taken largest first, ties to the lower chunk
    (every chunk when p >= 1). Returns (chunk ids ascending, number of chunks,
    tie_gap, tie_sum): tie_gap is the relative mass gap between the last chunk
    taken and the first left out, tie_sum the distance of the running sum before
    or after the last chunk taken from p, relative to p."""
    K = _f64(K)
    q = _f64(q)
    n = K.shape[0]
    if n == 0:
        return np.zeros(0, dtype=np.int64), 0, np.inf, np.inf
    s = beta * (K @ q)
    w = np.exp(s - s.max())
    w /= w.sum()
    m = np.add.reduceat(w, np.arange(0, n, group))
    order = np.argsort(-m, kind="stable")
    cum = np.cumsum(m[order])
    take = len(m) if p >= 1 else min(len(m), int(np.searchsorted(cum, p, side="left")) + 1)
    last = m[order[take - 1]]
    gap = (last - m[order[take]]) / last if take < len(m) else np.inf
    tsum = min(abs(cum[take - 1] - p), abs(cum[take - 1] - last - p)) / p if p < 1 else np.inf
    return np.sort(order[:take]), len(m), gap, tsum


def kept_mass(K, q, beta: float, sel, C: int, n1: int) -> float:
    """Share of the dense attention of ``q`` held by the chosen chunks plus tail."""
    K = _f64(K)
    q = _f64(q)
    sel = np.ascontiguousarray(np.asarray(sel, dtype=np.int64))
    return float(lib().orc_kept_mass(K.shape[0], K.shape[1], beta, _p(K), _p(q), _pl(sel), sel.size,
                                     C, n1))
