"""The C ABI library without a GPU: it loads, exports every function that
include/*.h declares, and rejects bad arguments on the host before any CUDA
call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fp():
    from dynamic_block_sparse_last_b200 import build
    build.build()
    from dynamic_block_sparse_last_b200 import fp as mod
    return mod


def declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if f.endswith(".h"):
            src = re.sub(r"/\*.*?\*/", "", open(os.path.join(inc, f)).read(), flags=re.S)
            names |= set(re.findall(r"\b(fp_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_every_declared_symbol_is_exported(fp):
    names = declared_functions()
    assert "fp_build_index" in names and "fp_sparse_attn" in names and "fp_prefill_run" in names
    lib = ctypes.CDLL(fp.library_path())
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) <= set(fp.SYMBOLS) | set(n for n in names if hasattr(fp, n))


def test_strerror(fp):
    assert fp.fp_strerror(fp.FP_OK) == "ok"
    assert "timed out" in fp.fp_strerror(fp.FP_ERR_TIMEOUT)


@pytest.mark.parametrize("S,Hq,Hkv,d,b", [(131073, 4, 2, 128, 128), (1024, 4, 3, 128, 128), (1024, 4, 2, 64, 128),
                                           (1024, 4, 2, 128, 32), (0, 4, 2, 128, 128), (262144, 4, 2, 128, 128),
                                           (1024, 0, 2, 128, 128)])
def test_create_rejects_unsupported_shapes(fp, S, Hq, Hkv, d, b):
    h = ctypes.c_void_p()
    assert fp.lib().fp_index_create(S, Hq, Hkv, d, b, ctypes.byref(h)) == fp.FP_ERR_ARG
    assert h.value is None


def test_calls_reject_null_and_misaligned_pointers(fp):
    L = fp.lib()
    assert L.fp_build_index(None, None, 1024, 4, 2, 128, 128, 0.9, 0.1, 0, None, None, None, None) == fp.FP_ERR_ARG
    assert L.fp_sparse_attn(None, None, None, None, None, None, None, None) == fp.FP_ERR_ARG
    assert L.fp_index_nnz(None, None, None) == fp.FP_ERR_ARG
    assert L.fp_index_export(None, None, None, None, None, None, None, None, None) == fp.FP_ERR_ARG
    assert L.fp_debug_wait_timeout(0, None) == fp.FP_ERR_ARG
    assert L.fp_debug_qk_tile_i8(8, 16, 1024, 4, 2, 128, 0, 0, 0, 16, None) == fp.FP_ERR_ARG   # q8 misaligned
    assert L.fp_debug_qk_tile_i8(16, 16, 1024, 4, 2, 128, 0, 64, 0, 16, None) == fp.FP_ERR_ARG  # p0 % 128


def test_index_info_rejects_null(fp):
    assert fp.lib().fp_index_info(None, None, None, None, None, None, None) == fp.FP_ERR_ARG


@pytest.mark.parametrize("S,Hq,Hkv,d,b,dt,groups", [(1024, 4, 2, 128, 128, 0, 3), (1024, 4, 2, 128, 128, 0, -1),
                                                   (1024, 4, 2, 128, 128, 0, 6), (1024, 6, 2, 128, 128, 0, 4),
                                                   (1024, 4, 2, 128, 128, 2, 0),
                                                   (1024, 4, 2, 64, 128, 0, 0), (131073, 4, 2, 128, 128, 0, 0)])
def test_prefill_create_rejects_bad_arguments(fp, S, Hq, Hkv, d, b, dt, groups):
    h = ctypes.c_void_p()
    assert fp.lib().fp_prefill_create(S, Hq, Hkv, d, b, dt, groups, ctypes.byref(h)) == fp.FP_ERR_ARG
    assert h.value is None


def test_prefill_run_rejects_null_before_any_cuda_call(fp):
    L = fp.lib()
    assert L.fp_prefill_run(None, 16, 16, 16, None, None, 0.9, 0.1, 16, None) == fp.FP_ERR_ARG
    assert L.fp_prefill_enqueue(None, 16, 16, 16, None, None, 0.9, 0.1, 16, None) == fp.FP_ERR_ARG
    assert L.fp_prefill_wait(None, None) == fp.FP_ERR_ARG
    assert L.fp_prefill_group_index(None, 0, None) == fp.FP_ERR_ARG
    L.fp_prefill_free(None)


def test_varlen_create_rejects_bad_offsets(fp):
    L = fp.lib()
    h = ctypes.c_void_p()
    for cu, nseq, b in [([1, 100], 1, 128), ([0, 100, 50], 2, 128), ([0, 100], 0, 128), ([0, 131073], 1, 128),
                        ([0, 0], 1, 128), ([0, 100], 1, 32), ([0, 65600], 1, 64)]:
        arr = (ctypes.c_int32 * len(cu))(*cu)
        assert L.fp_varlen_create(arr, nseq, 4, 2, 128, b, ctypes.byref(h)) == fp.FP_ERR_ARG, cu
        assert h.value is None
    assert L.fp_varlen_create(None, 1, 4, 2, 128, 128, ctypes.byref(h)) == fp.FP_ERR_ARG


def test_varlen_calls_reject_null(fp):
    L = fp.lib()
    assert L.fp_varlen_build_index(None, 16, 16, 0.9, 0.1, 0, None, None, None) == fp.FP_ERR_ARG
    assert L.fp_varlen_sparse_attn(None, 16, 16, 16, None, None, 16, None) == fp.FP_ERR_ARG
    assert L.fp_varlen_index(None, 0, None) == fp.FP_ERR_ARG
    L.fp_varlen_free(None)


def test_rope_pool_calls_reject_null(fp):
    L = fp.lib()
    assert L.fp_rope_pool(None, 16, 16, 16, 1024, 4, 2, 128, 128, 16, 16, 16, 16, None) == fp.FP_ERR_ARG
    assert L.fp_rope_pool(16, 16, 16, 16, 1024, 4, 2, 64, 128, 16, 16, 16, 16, None) == fp.FP_ERR_ARG  # d
    assert L.fp_rope_pool(16, 16, 8, 16, 1024, 4, 2, 128, 128, 16, 16, 16, 16, None) == fp.FP_ERR_ARG  # align
    assert L.fp_build_index_pooled(16, 16, None, 16, 1024, 4, 2, 128, 128, 0.9, 0.1, None, None) == fp.FP_ERR_ARG
