"""The C ABI library loads on a machine without a GPU and exports every symbol that
include/zha.h declares; calls that need no device reject bad arguments on the host."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zha.h")


@pytest.fixture(scope="module")
def zha():
    import tree_indexed_sparse_append_b200 as Z
    from tree_indexed_sparse_append_b200 import build as B

    B.build()
    return Z


def declared_symbols():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(zha_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree(zha):
    assert declared_symbols() == sorted(zha.SYMBOLS)


def test_library_exports_every_declared_symbol(zha):
    out = subprocess.run(["nm", "-D", "--defined-only", zha.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s(zha_\w+)", out))
    missing = [s for s in declared_symbols() if s not in exported]
    assert not missing, missing
    for name in declared_symbols():
        getattr(zha.lib(), name)


def test_build_targets_sm100a(zha):
    from tree_indexed_sparse_append_b200 import build as B

    assert "arch=compute_100a,code=sm_100a" in B.FLAGS


def test_host_side_argument_checks(zha):
    L = zha.lib()
    assert b"sm_100a" in L.zha_version()
    h = ctypes.c_void_p()
    assert L.zha_build(None, None, None, None, 0, None, ctypes.byref(h)) == zha.ERR_INVALID
    assert b"config" in L.zha_last_error()
    cfg = zha.Config(batch=1, n_kv_heads=1, d=100, R=4, chunk=4, depth=3, top_width=64, capacity=64,
                     sharpness=0.1, kv_dtype=zha.F32)
    assert L.zha_build(ctypes.byref(cfg), None, None, None, 0, None, ctypes.byref(h)) == zha.ERR_INVALID
    assert b"d must be" in L.zha_last_error()
    cfg.d = 64
    cfg.chunk = 1
    assert L.zha_build(ctypes.byref(cfg), None, None, None, 0, None, ctypes.byref(h)) == zha.ERR_INVALID
    cfg.chunk = 4
    cfg.depth = -1
    assert L.zha_build(ctypes.byref(cfg), None, None, None, 0, None, ctypes.byref(h)) == zha.ERR_INVALID
    assert b"depth" in L.zha_last_error()
    cfg.depth = 0  # a growing tree: the config is valid, the NULL pointers are not
    assert L.zha_build(ctypes.byref(cfg), None, None, None, 0, None, ctypes.byref(h)) == zha.ERR_INVALID
    assert b"NULL" in L.zha_last_error()
    assert h.value is None
    assert L.zha_search(None, None, 0, 1, 1, 0, 0.9, 1, None, None, 1, None, None) == zha.ERR_INVALID
    assert L.zha_attend(None, None, 0, 1, 1, None, None, 1, None, 0, None, None) == zha.ERR_INVALID
    assert L.zha_attend_noalloc(None, None, 0, 1, 1, None, None, 1, None, 0, None, None) == zha.ERR_INVALID
    assert L.zha_append(None, None, None, None) == zha.ERR_INVALID
    assert L.zha_rebuild(None, None) == zha.ERR_INVALID
    assert L.zha_test_wait_limit(None, 1000, 1) == zha.ERR_INVALID
    assert L.zha_cp_export(None, None, None, None, 1, None, None) == zha.ERR_INVALID
    assert L.zha_lse_combine(0, 1, 64, None, None, None, 0, None, None) == zha.ERR_INVALID
    assert L.zha_reserve(None, 1, 1) == zha.ERR_INVALID
    assert L.zha_dense_scan(None, None, 0, 1, 1, 0, 0.9, 1, None, None, 1, None) == zha.ERR_INVALID
    assert L.zha_chunk_mass(None, None, 0, 1, 1, 16, 0.9, None, None, 1, None) == zha.ERR_INVALID
    assert L.zha_num_keys(None) == -1
    assert L.zha_depth(None) == -1
    assert L.zha_sync_status(None, None) == zha.ERR_INVALID
    L.zha_destroy(None)


def test_binding_refuses_cpu_tensors(zha):
    import torch

    K = torch.zeros(1, 1, 64, 64)
    with pytest.raises((ValueError, zha.ZhaError)):
        zha.Tree(K, K.clone(), torch.zeros(1, 4, 64), 64, 4, 3, 0.125)
