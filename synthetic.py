"""Seeded synthetic workloads for the ZHA hot path.

This module only draws inputs (keys, values, reference queries, queries). It
holds none of the method's arithmetic and is the one piece that both the CUDA
path's tests/bench and the oracle consume. Everything is drawn with torch's
seeded generators, on the CPU or on a CUDA device; on a device, the tests copy
the drawn tensors to the host for the oracle, so both sides see the same bits.

Key recipe (clustered keys): contiguous blocks of 64 keys; each block has a
centre ~ N(0, I) and each key is its centre + N(0, 0.3^2 I). Values ~ N(0, I).
Reference queries ~ N(0, I), one set of R per KV head, shared by every sequence.
Queries mix m random distinct block centres of their tree (q = their sum), with
m uniform in 1..m_max; the demo-sized workload also has "one-place" queries,
4 x one centre + N(0, 0.1^2 I), and "eight-place" ones, the sum of 8 centres.
Appended keys continue the block structure with fresh blocks.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

BLOCK = 64
BASE_SEED = 1


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int  # sequences
    n_kv_heads: int
    n_q_heads: int
    n_keys: int  # keys per (sequence, KV head) when the tree is built
    d: int
    kv_dtype: str  # "f32" or "bf16"
    chunk: int
    depth: int
    R: int
    beta: float
    queries_per_head: int = 1
    m_max: int = 8  # queries mix 1..m_max centres
    query_kind: str = "mix"  # "mix" | "demo" (one-place + eight-place)
    modes: tuple = (("top_p", 0.9, 0),)
    appends: int = 0
    iid_keys: bool = False  # control: unstructured keys
    seed: int = 0
    noise: float = 0.3
    top_width: int = 64

    @property
    def capacity(self) -> int:
        return self.n_keys + self.appends

    @property
    def n_blocks(self) -> int:
        return (self.capacity + BLOCK - 1) // BLOCK

    @property
    def trees(self) -> int:
        return self.batch * self.n_kv_heads

    @property
    def walks(self) -> int:
        return self.batch * self.n_q_heads * self.queries_per_head

    @property
    def torch_dtype(self):
        return torch.float32 if self.kv_dtype == "f32" else torch.bfloat16

    def level_sizes(self, n_keys: int | None = None) -> list:
        n = self.n_keys if n_keys is None else n_keys
        out = [n]
        for _ in range(self.depth):
            n //= self.chunk
            out.append(n)
        return out


def _beta(d):
    return 1.0 / math.sqrt(d)


# The five workloads: a demo-sized fp32 tree, then 64K, 256K (with appends),
# prefill against the 256K tree, and 1M keys.
WORKLOADS = {
    "demo4k": Workload("demo4k", 1, 1, 1, 4096, 64, "f32", 4, 6, 4, _beta(64), queries_per_head=32,
                       query_kind="demo", modes=(("top_p", 0.9, 0), ("top_k", 0.0, 6)), seed=1000),
    "kv64k": Workload("kv64k", 1, 8, 32, 65536, 128, "bf16", 16, 4, 8, _beta(128), queries_per_head=32,
                      m_max=8, modes=(("top_p", 0.9, 0), ("top_k", 0.0, 8)), seed=1001),
    "kv256k": Workload("kv256k", 16, 4, 16, 262144, 128, "bf16", 8, 6, 8, _beta(128),
                       queries_per_head=1, m_max=8, modes=(("top_p", 0.9, 0),), appends=4096,
                       seed=1002),
    "prefill256k": Workload("prefill256k", 1, 4, 16, 262144, 128, "bf16", 8, 6, 8, _beta(128),
                            queries_per_head=4096, m_max=4, modes=(("top_p", 0.9, 0),), appends=4096,
                            seed=1002),
    "kv1m": Workload("kv1m", 8, 8, 32, 1048576, 128, "bf16", 16, 5, 8, _beta(128),
                     queries_per_head=1, m_max=8, modes=(("top_p", 0.9, 0), ("top_k", 0.0, 16)),
                     seed=1004),
}


def control(w: Workload) -> Workload:
    """The same workload with iid N(0, I) keys (no structure)."""
    return replace(w, name=w.name + "_iid", iid_keys=True)


def scaled(w: Workload, **kw) -> Workload:
    """A smaller copy of a workload (same recipe) for fast tests."""
    return replace(w, **kw)


def _gen(device, *key) -> torch.Generator:
    h = 0x9E3779B97F4A7C15
    for k in (BASE_SEED,) + key:
        h ^= (int(k) + 0x632BE59BD9B4E019 + ((h << 6) & (2**64 - 1)) + (h >> 2)) & (2**64 - 1)
    g = torch.Generator(device=device)
    g.manual_seed(h & (2**63 - 1))
    return g


@dataclass
class Inputs:
    w: Workload
    K: torch.Tensor  # [B][H_kv][capacity][d], kv dtype
    V: torch.Tensor  # [B][H_kv][capacity][d], kv dtype
    refs: torch.Tensor  # [H_kv][R][d] fp32
    Q: torch.Tensor  # [B][H_q][n_q][d], bf16 (fp32 for an fp32 workload)
    centres: torch.Tensor  # [B][H_kv][n_blocks][d] fp32 (recipe by-product)
    q_blocks: list = field(default_factory=list)


def draw_tree(w: Workload, b: int, h: int, device="cpu"):
    """Keys, values and block centres of one (sequence, KV head) tree."""
    g = _gen(device, w.seed, 1, b, h)
    cap = w.capacity
    centres = torch.randn(w.n_blocks, w.d, generator=g, device=device, dtype=torch.float32)
    noise = torch.randn(cap, w.d, generator=g, device=device, dtype=torch.float32)
    if w.iid_keys:
        k = noise
    else:
        k = centres.repeat_interleave(BLOCK, dim=0)[:cap] + w.noise * noise
    v = torch.randn(cap, w.d, generator=g, device=device, dtype=torch.float32)
    return k.to(w.torch_dtype), v.to(w.torch_dtype), centres


def draw_refs(w: Workload, device="cpu") -> torch.Tensor:
    g = _gen(device, w.seed, 2)
    return torch.randn(w.n_kv_heads, w.R, w.d, generator=g, device=device, dtype=torch.float32)


def draw_queries(w: Workload, centres: torch.Tensor, b: int, hq: int, device="cpu"):
    """Queries of one (sequence, query head) against its tree's block centres
    (only the blocks present when the tree was built)."""
    g = _gen(device, w.seed, 3, b, hq)
    n = w.queries_per_head
    nb = w.n_keys // BLOCK
    qdt = torch.float32 if w.kv_dtype == "f32" else torch.bfloat16
    if w.query_kind == "demo":
        half = n // 2
        one = torch.randint(0, nb, (half,), generator=g, device=device)
        q1 = 4.0 * centres[one] + 0.1 * torch.randn(half, w.d, generator=g, device=device)
        pick = torch.rand(n - half, nb, generator=g, device=device).argsort(dim=1)[:, :8]
        q8 = centres[pick].sum(dim=1)
        blocks = [[int(x)] for x in one.tolist()] + [r.tolist() for r in pick]
        return torch.cat([q1, q8]).to(qdt), blocks
    m = torch.randint(1, w.m_max + 1, (n,), generator=g, device=device)
    pick = torch.rand(n, nb, generator=g, device=device).argsort(dim=1)[:, : w.m_max]
    q = torch.zeros(n, w.d, device=device, dtype=torch.float32)
    for j in range(w.m_max):
        on = (m > j).to(torch.float32).unsqueeze(1)
        q = q + on * centres[pick[:, j]]
    blocks = [pick[i, : int(m[i])].tolist() for i in range(n)] if n <= 4096 else []
    return q.to(qdt), blocks


def draw(w: Workload, device="cpu", with_values: bool = True) -> Inputs:
    """All inputs of a workload, laid out for the library:
    K, V [B][H_kv][capacity][d]; refs [H_kv][R][d]; Q [B][H_q][n_q][d]."""
    B, H, cap, d = w.batch, w.n_kv_heads, w.capacity, w.d
    K = torch.empty(B, H, cap, d, dtype=w.torch_dtype, device=device)
    V = torch.empty(B, H, cap, d, dtype=w.torch_dtype, device=device) if with_values else None
    centres = torch.empty(B, H, w.n_blocks, d, dtype=torch.float32, device=device)
    for b in range(B):
        for h in range(H):
            k, v, c = draw_tree(w, b, h, device)
            K[b, h] = k
            if with_values:
                V[b, h] = v
            centres[b, h] = c
            del k, v
    refs = draw_refs(w, device)
    qdt = torch.float32 if w.kv_dtype == "f32" else torch.bfloat16
    Q = torch.empty(B, w.n_q_heads, w.queries_per_head, d, dtype=qdt, device=device)
    group = w.n_q_heads // w.n_kv_heads
    blocks = []
    for b in range(B):
        for hq in range(w.n_q_heads):
            q, bl = draw_queries(w, centres[b, hq // group], b, hq, device)
            Q[b, hq] = q
            blocks.append(bl)
    return Inputs(w=w, K=K, V=V, refs=refs, Q=Q, centres=centres, q_blocks=blocks)
