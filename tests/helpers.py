"""Shared helpers of the parity tests: the oracle side of a workload, and the
element-wise comparisons with the tolerances the method's targets fix.

Tolerances (per element g = GPU, o = oracle):
  node keys and biases: |g - o| <= rtol * max|o over the row|, rtol = 1e-5 (a row
      = one reference key of a node, or a node's R biases): 1e-5 relative to the
      magnitude of the vector the element belongs to. An element near zero is a
      cancellation of weighted terms of the row's size, so fp32 gives it an
      absolute error of a few ulps of the row, not of itself;
  attention outputs (fp32) and lse: |g - o| <= atol * max(1, |o|), atol = 1e-5
      for an fp32 cache and 3e-3 for a bf16 cache;
  attention outputs stored as bf16: |g - o| <= half a bf16 ulp (the rounding of
      the stored value) + 1e-5 * max(1, max|o| over the output row) (the fp32
      arithmetic before rounding); rounding alone moves a value by up to 2^-9
      relative, so the 3e-3 target is checked on the fp32 output;
  selected chunk sets: identical, unless the oracle's walk met a near-tie: a
      relative gap below 1e-5 between the last opened and the first unopened
      mass, or a running top-p sum within 1e-5 * p of p. A walk that parts there
      must still be a correct walk: one of the walks whose choice at every level is
      admissible at that tolerance under the oracle's exact masses
      (``oracle.ties``), and its attention is then checked against the oracle's
      attention over the GPU's own selection. At most 1% of a test's walks (at
      least one) may part.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from oracle import ties as OT

NODE_RTOL = 1e-5
TIE_TOL = 1e-5
MAX_PARTING_SHARE = 0.01


def attn_tol(w) -> float:
    return 1e-5 if w.kv_dtype == "f32" else 3e-3


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def oracle_tree(inp, b: int, h: int, n_keys: int | None = None, threads: int = 0, capacity=None):
    w = inp.w
    n = w.n_keys if n_keys is None else n_keys
    K = host64(inp.K[b, h, :n])
    refs = host64(inp.refs[h])
    return O.build_tree(K, refs, w.chunk, w.depth, w.beta, store=O.STORE_F32, threads=threads,
                        capacity=capacity)


def gpu_level(tree, l: int, t: int):
    nodes, n = tree.level(l)
    return host64(nodes[t, :n]), n


def assert_nodes_close(g: np.ndarray, keys: np.ndarray, bias: np.ndarray, R: int, d: int,
                       rtol: float = NODE_RTOL, what: str = ""):
    n = keys.shape[0]
    assert g.shape[0] == n, (what, g.shape, keys.shape)
    gk = g[:, : R * d].reshape(n, R, d)
    gb = g[:, R * d: R * d + R]
    scale_k = np.abs(keys).max(axis=2, keepdims=True)
    bad_k = np.abs(gk - keys) > rtol * scale_k
    assert not bad_k.any(), f"{what}: {bad_k.sum()} node key elements off; worst |diff| " \
                            f"{np.abs(gk - keys).max():.3g}"
    scale_b = np.abs(bias).max(axis=1, keepdims=True)
    bad_b = np.abs(gb - bias) > rtol * scale_b
    assert not bad_b.any(), f"{what}: {bad_b.sum()} biases off; worst |diff| {np.abs(gb - bias).max():.3g}"


def near_tie(walk) -> bool:
    return min(walk.tie_gap, walk.tie_sum) < TIE_TOL


def compare_selection(sel: np.ndarray, cnt: np.ndarray, walks: dict, valid=None):
    """walks: {walk index: oracle Walk}. Returns the walk ids whose GPU selection
    differs from the oracle's. Each of them must be an oracle near-tie and, when
    ``valid`` is given, ``valid(walk index, GPU chunk ids as a tuple)`` must hold
    (the GPU walk is admissible under the oracle's masses)."""
    differ = []
    for w, ow in walks.items():
        g = sel[w, : cnt[w]]
        if not np.array_equal(g, ow.sel):
            assert near_tie(ow), (f"walk {w}: GPU and oracle selections differ away from a tie "
                                  f"(gap {ow.tie_gap:.3g}, sum {ow.tie_sum:.3g}; "
                                  f"{len(g)} vs {len(ow.sel)} chunks)")
            if valid is not None:
                assert valid(w, tuple(int(x) for x in g)), (
                    f"walk {w}: the GPU selection parts from the oracle at a near-tie but is not an "
                    f"admissible walk at tolerance {TIE_TOL} ({len(g)} vs {len(ow.sel)} chunks)")
            differ.append(w)
    return differ


def tree_walk_valid(otree, q, mode: int, p: float, k: int, top_width: int):
    """Check for compare_selection: the GPU chunk set is the result of a walk of q
    down the oracle tree whose choice at every level is admissible at TIE_TOL."""
    def check(_w, g):
        return g in OT.admissible_selections(otree, q, mode, p, k, top_width, TIE_TOL)
    return check


def one_level_valid(m: np.ndarray, mode: int, p: float, k: int):
    """Check for compare_selection on a one-level choice (the full-scan indexer,
    the chunk-mass profile) over candidates of exact masses m: the GPU's set must
    be an admissible choice of them."""
    def check(_w, g):
        A = np.zeros(len(m), dtype=bool)
        A[list(g)] = True
        return OT.admissible(m, A, mode, p, k, TIE_TOL)
    return check


def assert_partings_bounded(parted: int, walks: int, what: str = ""):
    allowed = max(1, int(MAX_PARTING_SHARE * walks))
    assert parted <= allowed, f"{what}: {parted} of {walks} walks part at near-ties (at most {allowed})"


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_bf16_output_close(out_g: np.ndarray, out_o: np.ndarray, what: str = ""):
    allow = 0.5 * bf16_ulp(np.maximum(np.abs(out_g), np.abs(out_o))) + 1e-5 * max(1.0, np.abs(out_o).max())
    bad = np.abs(out_g - out_o) > allow
    assert not bad.any(), f"{what}: {bad.sum()} bf16 outputs off by more than half an ulp"


def assert_attention_close(out_g: np.ndarray, lse_g: float, out_o: np.ndarray, lse_o: float, atol: float,
                           what: str = ""):
    err = np.abs(out_g - out_o) / np.maximum(1.0, np.abs(out_o))
    assert err.max() <= atol, f"{what}: attention output off by {err.max():.3g} (tol {atol})"
    assert abs(lse_g - lse_o) <= atol * max(1.0, abs(lse_o)), f"{what}: lse {lse_g} vs {lse_o}"
