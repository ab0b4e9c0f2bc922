"""The C-ABI library loads and exports every symbol include/csa2.h declares;
host-side argument, mode and fault-injection checks return their status
without touching a device.  Runs on the CPU (no compute calls)."""
import ctypes
import os
import re

import pytest

import kv_cache_csa2_b200 as K
from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "csa2.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(csa2_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = K.lib()
    decl = declared_functions()
    assert len(decl) >= 20
    for name in decl:
        assert hasattr(lib, name), name
    # the binding declares exactly the header's functions
    assert sorted(K.EXPORTED_SYMBOLS) == decl


def test_status_strings_and_version():
    lib = K.lib()
    assert lib.csa2_version() >= 1
    names = [lib.csa2_status_string(i).decode() for i in range(8)]
    assert names == ["CSA2_OK", "CSA2_ERR_INVALID", "CSA2_ERR_MODE", "CSA2_ERR_UNSUPPORTED",
                     "CSA2_ERR_CUDA", "CSA2_ERR_TIMEOUT", "CSA2_ERR_OOM", "CSA2_ERR_BOUNDS"]


def test_invalid_arguments_rejected_on_host():
    lib = K.lib()
    p = ctypes.c_void_p(16)
    # D not a multiple of 8, m out of range
    assert lib.csa2_compress(p, p, p, 1, 8, 7, 4, 0, p, 0, None) == 1
    assert lib.csa2_compress(p, p, p, 1, 8, 8, 0, 0, p, 0, None) == 1
    assert "m=0" in lib.csa2_last_error().decode()
    # FP4 width must be a multiple of 16
    assert lib.csa2_fp4_pack(p, 4, 24, p, p, None) == 1
    # indexer width limits
    assert lib.csa2_index_scores(p, p, p, 1, 1, 8, 12, 10, None, None, 0, 0, p, None) == 1
    # empty work is a no-op
    assert lib.csa2_compress(None, None, None, 0, 8, 8, 4, 0, None, 0, None) == 0


def test_mode_rules_rejected_on_host():
    lib = K.lib()
    p = ctypes.c_void_p(256)
    args = lambda mode, pin, pout: (mode, p, p, p, 1, 1, 8, 64, 100, None, pin, 10 if pin else 0,
                                    4, p, pout, 10 if pout else 0, 0, p, 1 << 20, None)
    assert lib.csa2_index_topk(*args(K.REUSE, None, None)) == 2          # Reuse runs no indexer
    assert lib.csa2_index_topk(*args(K.FULL, p, None)) == 2              # Full takes no pool
    assert lib.csa2_index_topk(*args(K.REINDEX, None, p)) == 2           # Reindex keeps no pool
    assert "Reuse" in lib.csa2_last_error().decode() or "pool" in lib.csa2_last_error().decode()


def test_group_descriptor_validation_on_host():
    lib = K.lib()
    modes = (ctypes.c_int * 2)(K.FULL, 7)
    desc = K.CSA2GroupDesc(1, 1, 100, 128, 16, 8, 64, 16, 0, 0.1, 0, 0, 2, modes)
    h = ctypes.c_void_p()
    assert lib.csa2_group_create(ctypes.byref(h), ctypes.byref(desc)) == 1
    assert not h.value


def test_fault_injection_returns_status_without_device():
    lib = K.lib()
    p = ctypes.c_void_p(256)
    try:
        K.set_fault("alloc")
        assert lib.csa2_fp4_pack(p, 4, 32, p, p, None) == 6
        assert "injected" in lib.csa2_last_error().decode()
        K.set_fault("launch")
        assert lib.csa2_compress(p, p, p, 1, 8, 8, 4, 0, p, 0, None) == 4
        with pytest.raises(K.CSA2Error):
            K._check(lib.csa2_sparse_attn(0, p, None, p, 1, 1, 16, 4, 1.0, p, None, None, 0, None))
        with pytest.raises(K.CSA2Error):
            K.set_fault("bogus")
    finally:
        K.set_fault("")
    assert lib.csa2_fp4_pack(p, 4, 24, p, p, None) == 1   # back to normal validation


def test_workspace_queries():
    lib = K.lib()
    ws = lib.csa2_index_topk_workspace(8, 1, 262144, 0, 2048, 16384)
    assert ws >= 8 * 262144 * 4
    assert lib.csa2_index_topk_workspace(8, 1, 262144, 16384, 2048, 0) >= 8 * 16384 * 4
    assert lib.csa2_select_topk_workspace(8, 262144, 2048) >= 0


def test_attention_workspace_covers_every_schedule():
    """The attention workspace query is the maximum over the kernels a call may
    take: entries of width 128 with several 128-row tiles keep per-tile
    partials (a 128 x heads f32 block plus m and l per head) and a counter
    per query; one tile needs none."""
    lib = K.lib()
    fp4, bf16 = 1, 0
    # 64 queries, 16 heads, k = 256: two tiles per query
    need = 64 * 2 * (128 * 16 + 2 * 16) * 4 + 64 * 4
    assert lib.csa2_sparse_attn_workspace(64, 1, 16, 128, 256, fp4) >= need
    assert lib.csa2_sparse_attn_workspace(64, 1, 16, 128, 256, bf16) >= need
    # 64 heads x 512 (the split schedule): a 128 KiB partial per CTA and a flag
    assert lib.csa2_sparse_attn_workspace(8, 1, 64, 512, 2048, bf16) >= 16 * 128 * 1024
