"""Python binding of libzha, the B200 (sm_100a) library for Zyphra Hierarchical
Attention: a tree of compressed key summaries over a KV cache, walked top-down by
each query, followed by attention over exactly the keys the walk chose.

This module only marshals arguments (torch tensors -> device pointers, the current
CUDA stream) into the C ABI declared in include/zha.h; every step runs in the
library's CUDA kernels. There is no CPU fallback: without libzha.so or a CUDA
device the calls raise.

Names follow the C ABI: build / append / search / attend.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzha.so")
MAX_DEPTH = 12

OK, ERR_INVALID, ERR_CAPACITY, ERR_OOM, ERR_CUDA, ERR_INTERNAL, ERR_TIMEOUT = 0, -1, -2, -3, -4, -5, -6
F32, BF16 = 0, 1
TOP_P, TOP_K = 0, 1

# Every symbol include/zha.h declares.
SYMBOLS = ("zha_build", "zha_append", "zha_search", "zha_attend", "zha_reserve", "zha_level",
           "zha_num_keys", "zha_depth", "zha_sync_status", "zha_destroy", "zha_last_error", "zha_version",
           "zha_profile", "zha_profile_read", "zha_kernel_launches", "zha_last_search_info",
           "zha_dense_scan", "zha_attend_noalloc", "zha_chunk_mass", "zha_ref_grad", "zha_rebuild",
           "zha_test_wait_limit", "zha_cp_begin", "zha_cp_export", "zha_cp_select", "zha_lse_combine")
KERNEL_KINDS = ("build", "append", "search_init", "score", "select", "attend_plan", "attend_partial",
                "attend_combine", "score_tc")


class ZhaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"zha error {code}: {msg}")
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("n_kv_heads", ctypes.c_int), ("d", ctypes.c_int),
                ("R", ctypes.c_int), ("chunk", ctypes.c_int), ("depth", ctypes.c_int),
                ("top_width", ctypes.c_int), ("capacity", ctypes.c_longlong),
                ("sharpness", ctypes.c_float), ("kv_dtype", ctypes.c_int)]


class Stats(ctypes.Structure):
    _fields_ = [("start_level", ctypes.c_int), ("frontier", ctypes.c_int * (MAX_DEPTH + 1)),
                ("opened", ctypes.c_int * (MAX_DEPTH + 1)), ("keys_read", ctypes.c_longlong),
                ("work", ctypes.c_longlong)]


STATS_BYTES = ctypes.sizeof(Stats)


class KernelTime(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_longlong), ("ms", ctypes.c_double)]


class SearchInfo(ctypes.Structure):
    _fields_ = [("start_level", ctypes.c_int), ("union_nodes", ctypes.c_longlong * (MAX_DEPTH + 1)),
                ("walk_nodes", ctypes.c_longlong * (MAX_DEPTH + 1))]

_lib = None


def lib():
    """The loaded libzha.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run __graft_entry__.build() (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, ll, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float
        L.zha_build.argtypes = [ctypes.POINTER(Config), vp, vp, vp, ll, vp, ctypes.POINTER(vp)]
        L.zha_append.argtypes = [vp, vp, vp, vp]
        L.zha_rebuild.argtypes = [vp, vp]
        L.zha_test_wait_limit.argtypes = [vp, ll, i]
        L.zha_cp_begin.argtypes = [vp, vp, i, i, i, ll, ctypes.POINTER(ll), i, ctypes.POINTER(i), vp]
        L.zha_cp_export.argtypes = [vp, vp, vp, vp, ll, ctypes.POINTER(i), vp]
        L.zha_cp_select.argtypes = [vp, i, vp, vp, vp, ll, i, f, i, vp, vp, i, ctypes.POINTER(i), vp]
        L.zha_lse_combine.argtypes = [i, ll, i, vp, vp, vp, i, vp, vp]
        L.zha_search.argtypes = [vp, vp, i, i, i, i, f, i, vp, vp, i, vp, vp]
        L.zha_attend.argtypes = [vp, vp, i, i, i, vp, vp, i, vp, i, vp, vp]
        L.zha_attend_noalloc.argtypes = [vp, vp, i, i, i, vp, vp, i, vp, i, vp, vp]
        L.zha_reserve.argtypes = [vp, ll, i]
        L.zha_dense_scan.argtypes = [vp, vp, i, i, i, i, f, i, vp, vp, i, vp]
        L.zha_chunk_mass.argtypes = [vp, vp, i, i, i, i, f, vp, vp, i, vp]
        L.zha_ref_grad.argtypes = [vp, vp, i, i, i, vp, vp, vp]
        L.zha_level.argtypes = [vp, i, ctypes.POINTER(vp), ctypes.POINTER(ll), ctypes.POINTER(ll),
                                ctypes.POINTER(i)]
        L.zha_num_keys.argtypes = [vp]
        L.zha_num_keys.restype = ll
        L.zha_depth.argtypes = [vp]
        L.zha_depth.restype = ctypes.c_int
        L.zha_sync_status.argtypes = [vp, vp]
        L.zha_destroy.argtypes = [vp]
        L.zha_destroy.restype = None
        L.zha_profile.argtypes = [vp, i]
        L.zha_profile_read.argtypes = [vp, ctypes.POINTER(KernelTime), vp]
        L.zha_kernel_launches.restype = ll
        L.zha_kernel_launches.argtypes = []
        L.zha_last_search_info.argtypes = [vp, ctypes.POINTER(SearchInfo), vp]
        L.zha_last_error.restype = ctypes.c_char_p
        L.zha_version.restype = ctypes.c_char_p
        for name in SYMBOLS:
            getattr(L, name)
        _lib = L
    return _lib


def _check(rc: int):
    if rc != OK:
        raise ZhaError(rc, lib().zha_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}: use float32 or bfloat16")


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class _DeviceArray:
    """A non-owning __cuda_array_interface__ view of library-owned device memory."""

    def __init__(self, ptr: int, shape, typestr: str, owner):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (ptr, False), "version": 3, "strides": None}
        self._owner = owner


class Tree:
    """The summary trees of a KV cache [B][H_kv][capacity][d] (one per sequence and
    KV head). K, V and refs stay referenced here: the library keeps their pointers."""

    def __init__(self, K: torch.Tensor, V: torch.Tensor, refs: torch.Tensor, n_keys: int, chunk: int,
                 depth: int, sharpness: float, top_width: int = 64, stream=None):
        if K.dim() != 4 or V.shape != K.shape:
            raise ValueError("K and V must both be [B][H_kv][capacity][d]")
        if refs.dim() != 3 or refs.dtype != torch.float32 or refs.shape[0] != K.shape[1] or refs.shape[2] != K.shape[3]:
            raise ValueError("refs must be fp32 [H_kv][R][d]")
        if V.dtype != K.dtype:
            raise ValueError("K and V must have the same dtype")
        B, H, cap, d = K.shape
        self.cfg = Config(batch=B, n_kv_heads=H, d=d, R=refs.shape[1], chunk=chunk, depth=depth,
                          top_width=top_width, capacity=cap, sharpness=sharpness,
                          kv_dtype=_dtype_code(K))
        self.K, self.V, self.refs = K, V, refs
        self._h = ctypes.c_void_p()
        _check(lib().zha_build(ctypes.byref(self.cfg), _dev(K, "K"), _dev(V, "V"), _dev(refs, "refs"),
                               int(n_keys), _stream(stream), ctypes.byref(self._h)))

    # -- properties -------------------------------------------------------
    @property
    def handle(self) -> int:
        return self._h.value

    @property
    def n_keys(self) -> int:
        return int(lib().zha_num_keys(self._h))

    @property
    def depth(self) -> int:
        """Levels the trees have now (the configured depth, or for depth=0 the
        deepest level holding a node)."""
        return int(lib().zha_depth(self._h))

    def level_sizes(self) -> list:
        out = [self.n_keys]
        for l in range(1, self.depth + 1):
            out.append(self.level(l)[1])
        return out

    def level(self, l: int):
        """(nodes view [B*H_kv][level_capacity][node_floats] fp32, live node count)."""
        ptr = ctypes.c_void_p()
        n = ctypes.c_longlong()
        cap = ctypes.c_longlong()
        nf = ctypes.c_int()
        _check(lib().zha_level(self._h, l, ctypes.byref(ptr), ctypes.byref(n), ctypes.byref(cap),
                               ctypes.byref(nf)))
        T = self.cfg.batch * self.cfg.n_kv_heads
        if not ptr.value:
            return torch.zeros(T, 0, nf.value, device=self.K.device), n.value
        view = torch.as_tensor(_DeviceArray(ptr.value, (T, cap.value, nf.value), "<f4", self),
                               device=self.K.device)
        return view, n.value

    # -- the hot path -----------------------------------------------------
    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> None:
        B, H, _, d = self.K.shape
        if k_new.shape != (B, H, d) or v_new.shape != (B, H, d) or k_new.dtype != self.K.dtype or v_new.dtype != self.K.dtype:
            raise ValueError("k_new and v_new must be [B][H_kv][d] of the cache dtype")
        _check(lib().zha_append(self._h, _dev(k_new, "k_new"), _dev(v_new, "v_new"), _stream(stream)))

    def rebuild(self, stream=None) -> None:
        """Summarize every level again in place from the cache and the current
        refs (after the refs were updated in place); allocates nothing."""
        _check(lib().zha_rebuild(self._h, _stream(stream)))

    def search(self, Q: torch.Tensor, mode: int = TOP_P, p: float = 0.9, k: int = 1, max_sel: int | None = None,
               with_stats: bool = False, out=None, stream=None):
        """Q: [B][H_q][n_q][d]. Returns (sel [walks][max_sel] int32, sel_count [walks] int32,
        stats uint8 [walks][sizeof zha_stats] or None)."""
        B, Hq, nq, d = Q.shape
        W = B * Hq * nq
        if max_sel is None:
            max_sel = max(1, self.level(1)[1])
        if out is None:
            sel = torch.empty(W, max_sel, dtype=torch.int32, device=Q.device)
            cnt = torch.empty(W, dtype=torch.int32, device=Q.device)
            st = torch.empty(W, STATS_BYTES, dtype=torch.uint8, device=Q.device) if with_stats else None
        else:
            sel, cnt, st = out
        _check(lib().zha_search(self._h, _dev(Q, "Q"), _dtype_code(Q), Hq, nq, mode, float(p), int(k),
                                _dev(sel, "sel"), _dev(cnt, "sel_count"), max_sel,
                                _dev(st, "stats") if st is not None else None, _stream(stream)))
        return sel, cnt, st

    def attend(self, Q: torch.Tensor, sel: torch.Tensor, sel_count: torch.Tensor, out=None, lse=None,
               out_dtype=None, stream=None):
        """Returns (out [B][H_q][n_q][d] of out_dtype (default: the cache dtype), lse [walks] fp32)."""
        B, Hq, nq, d = Q.shape
        W = B * Hq * nq
        if out is None:
            out = torch.empty(B, Hq, nq, d, dtype=out_dtype or self.K.dtype, device=Q.device)
        if lse is None:
            lse = torch.empty(W, dtype=torch.float32, device=Q.device)
        _check(lib().zha_attend(self._h, _dev(Q, "Q"), _dtype_code(Q), Hq, nq, _dev(sel, "sel"),
                                _dev(sel_count, "sel_count"), sel.shape[1], _dev(out, "out"), _dtype_code(out),
                                _dev(lse, "lse"), _stream(stream)))
        return out, lse

    def attend_noalloc(self, Q: torch.Tensor, sel: torch.Tensor, sel_count: torch.Tensor, out: torch.Tensor,
                       lse: torch.Tensor | None = None, stream=None):
        """attend() for callers whose device memory may not be allocated by the library:
        zha_attend_noalloc uses a fixed static device array as scratch. The caller
        provides out (and lse) already allocated; nothing is allocated here."""
        B, Hq, nq, d = Q.shape
        _check(lib().zha_attend_noalloc(self._h, _dev(Q, "Q"), _dtype_code(Q), Hq, nq, _dev(sel, "sel"),
                                        _dev(sel_count, "sel_count"), sel.shape[1], _dev(out, "out"),
                                        _dtype_code(out), _dev(lse, "lse") if lse is not None else None,
                                        _stream(stream)))
        return out, lse

    def dense_scan(self, Q: torch.Tensor, mode: int = TOP_P, p: float = 0.9, k: int = 1,
                   max_sel: int | None = None, out=None, stream=None):
        """Full-scan indexer: every key scored, top-p / top-K over keys.
        Returns (sel [walks][max_sel] int32 key indices ascending, sel_count [walks])."""
        B, Hq, nq, d = Q.shape
        W = B * Hq * nq
        if max_sel is None:
            max_sel = max(1, self.n_keys)
        if out is None:
            sel = torch.empty(W, max_sel, dtype=torch.int32, device=Q.device)
            cnt = torch.empty(W, dtype=torch.int32, device=Q.device)
        else:
            sel, cnt = out
        _check(lib().zha_dense_scan(self._h, _dev(Q, "Q"), _dtype_code(Q), Hq, nq, mode, float(p), int(k),
                                    _dev(sel, "sel"), _dev(cnt, "sel_count"), max_sel, _stream(stream)))
        return sel, cnt

    def chunk_mass(self, Q: torch.Tensor, group: int = 16, p: float = 0.9, max_sel: int | None = None, out=None,
                   stream=None):
        """Chunk-mass profile of dense attention: per walk, the fewest chunks of
        `group` keys holding p of the softmax over all keys. Returns (sel
        [walks][max_sel] int32 chunk indices ascending, count [walks] int32,
        n_chunks)."""
        B, Hq, nq, d = Q.shape
        W = B * Hq * nq
        n_chunks = (self.n_keys + group - 1) // group if group >= 1 else 0
        if max_sel is None:
            max_sel = max(1, n_chunks)
        if out is None:
            sel = torch.empty(W, max_sel, dtype=torch.int32, device=Q.device)
            cnt = torch.empty(W, dtype=torch.int32, device=Q.device)
        else:
            sel, cnt = out
        _check(lib().zha_chunk_mass(self._h, _dev(Q, "Q"), _dtype_code(Q), Hq, nq, int(group), float(p),
                                    _dev(sel, "sel"), _dev(cnt, "count"), max_sel, _stream(stream)))
        return sel, cnt, n_chunks

    def ref_grad(self, Q: torch.Tensor, stream=None):
        """The split loss (KL of the teacher's split of attention from the tree's,
        summed over levels, averaged over walks) and its gradient with respect to
        the references the tree was built with. Returns (loss [1], grad
        [H_kv][R][d]), fp32 on the device."""
        B, Hq, nq, d = Q.shape
        loss = torch.empty(1, dtype=torch.float32, device=Q.device)
        grad = torch.empty(self.cfg.n_kv_heads, self.cfg.R, d, dtype=torch.float32, device=Q.device)
        _check(lib().zha_ref_grad(self._h, _dev(Q, "Q"), _dtype_code(Q), Hq, nq, _dev(loss, "loss"),
                                  _dev(grad, "grad"), _stream(stream)))
        return loss, grad

    # -- context-parallel walk (one shard of every tree per process) ------------
    def cp_begin(self, Q: torch.Tensor, key_begin: int, global_counts, stream=None) -> int:
        """Start a context-parallel walk of Q on this shard; returns the start level."""
        B, Hq, nq, d = Q.shape
        counts = (ctypes.c_longlong * len(global_counts))(*[int(c) for c in global_counts])
        level = ctypes.c_int()
        _check(lib().zha_cp_begin(self._h, _dev(Q, "Q"), _dtype_code(Q), Hq, nq, int(key_begin), counts,
                                  len(global_counts), ctypes.byref(level), _stream(stream)))
        return level.value

    def cp_export(self, ids: torch.Tensor, scores: torch.Tensor, counts: torch.Tensor, stream=None) -> int:
        """Score this shard's frontier; ids/scores [walks][stride], counts [walks]. Returns the level."""
        level = ctypes.c_int()
        _check(lib().zha_cp_export(self._h, _dev(ids, "ids"), _dev(scores, "scores"), _dev(counts, "counts"),
                                   ids.shape[1], ctypes.byref(level), _stream(stream)))
        return level.value

    def cp_select(self, ids: torch.Tensor, scores: torch.Tensor, counts: torch.Tensor, mode: int, p: float, k: int,
                  sel: torch.Tensor, sel_count: torch.Tensor, stream=None) -> int:
        """Choose over the gathered lists (ids/scores [parts][walks][stride], counts
        [parts][walks]); returns the next level (0 when the walk is complete)."""
        level = ctypes.c_int()
        _check(lib().zha_cp_select(self._h, ids.shape[0], _dev(ids, "ids"), _dev(scores, "scores"),
                                   _dev(counts, "counts"), ids.shape[2], mode, float(p), int(k), _dev(sel, "sel"),
                                   _dev(sel_count, "sel_count"), sel.shape[1], ctypes.byref(level),
                                   _stream(stream)))
        return level.value

    def reserve(self, max_walks: int, max_sel: int) -> None:
        _check(lib().zha_reserve(self._h, int(max_walks), int(max_sel)))

    # -- diagnostics --------------------------------------------------------
    def profile(self, enable: bool) -> None:
        _check(lib().zha_profile(self._h, 1 if enable else 0))

    def profile_read(self, stream=None) -> dict:
        arr = (KernelTime * len(KERNEL_KINDS))()
        _check(lib().zha_profile_read(self._h, arr, _stream(stream)))
        return {name: (arr[i].launches, arr[i].ms) for i, name in enumerate(KERNEL_KINDS)}

    def last_search_info(self, stream=None) -> dict:
        info = SearchInfo()
        _check(lib().zha_last_search_info(self._h, ctypes.byref(info), _stream(stream)))
        return {"start_level": info.start_level, "union_nodes": list(info.union_nodes),
                "walk_nodes": list(info.walk_nodes)}

    def test_wait_limit(self, wait_ns: int, stall: bool = False) -> None:
        """Test hook: the tensor-core scorer's waits give up after wait_ns (0: the
        default 1 s); with stall, its launches first wait on a barrier nothing
        arrives at, so the search reports ZHA_ERR_TIMEOUT."""
        _check(lib().zha_test_wait_limit(self._h, int(wait_ns), 1 if stall else 0))

    def sync_status(self, stream=None) -> None:
        _check(lib().zha_sync_status(self._h, _stream(stream)))

    def close(self) -> None:
        if self._h and self._h.value:
            lib().zha_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def lse_combine(outs: torch.Tensor, lses: torch.Tensor, out_dtype=torch.float32, stream=None):
    """Attention over the union of disjoint key sets: outs [parts][walks][d] fp32,
    lses [parts][walks] fp32 -> (out [walks][d] of out_dtype, lse [walks])."""
    P, W, d = outs.shape
    out = torch.empty(W, d, dtype=out_dtype, device=outs.device)
    lse = torch.empty(W, dtype=torch.float32, device=outs.device)
    _check(lib().zha_lse_combine(P, W, d, _dev(outs, "outs"), _dev(lses, "lses"), _dev(out, "out"),
                                 _dtype_code(out), _dev(lse, "lse"), _stream(stream)))
    return out, lse


def parse_stats(st: torch.Tensor) -> list:
    """Device stats bytes -> list of dicts (host)."""
    raw = st.cpu().numpy().tobytes()
    out = []
    for w in range(st.shape[0]):
        s = Stats.from_buffer_copy(raw[w * STATS_BYTES:(w + 1) * STATS_BYTES])
        out.append({"start_level": s.start_level, "frontier": list(s.frontier), "opened": list(s.opened),
                    "keys_read": s.keys_read, "work": s.work})
    return out


def kernel_launches() -> int:
    """Kernels this library has launched in this process."""
    return int(lib().zha_kernel_launches())


def version() -> str:
    return lib().zha_version().decode()
