"""Python binding of the C ABI in include/fp_sparse.h (ctypes).

Argument marshalling only: torch tensors are passed as device pointers and
the current CUDA stream as a handle; every step of the computation runs in
the library's CUDA kernels.  Importing fails loudly when the library has not
been built -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libfpsparse.so")

FP_OK, FP_ERR_ARG, FP_ERR_CUDA, FP_ERR_TIMEOUT, FP_ERR_STATE = 0, 1, 2, 3, 4
FP_QK_BF16, FP_QK_INT8 = 0, 1
FP_PATTERN_VS, FP_PATTERN_QA = 0, 1

SYMBOLS = ("fp_index_create", "fp_index_free", "fp_build_index", "fp_sparse_attn", "fp_index_info",
           "fp_index_nnz", "fp_index_export", "fp_get_device_error", "fp_debug_wait_timeout",
           "fp_debug_qk_tile_i8", "fp_debug_capture_i8", "fp_pattern_stats_noalloc", "fp_strerror",
           "fp_index_share", "fp_index_classes", "fp_choose_block_size", "fp_index_csr",
           "fp_index_group_lists",
           "fp_prefill_create", "fp_prefill_free", "fp_prefill_enqueue", "fp_prefill_wait", "fp_prefill_run",
           "fp_prefill_group_index", "fp_varlen_create", "fp_varlen_free", "fp_varlen_build_index",
           "fp_varlen_sparse_attn", "fp_varlen_index", "fp_rope_pool", "fp_build_index_pooled")


class FpError(RuntimeError):
    def __init__(self, code, where):
        super().__init__(f"{where}: {fp_strerror(code)} (code {code})")
        self.code = code


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"CUDA library not built: {_LIB_PATH} is missing "
                          "(run python -m dynamic_block_sparse_last_b200.build)")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.fp_index_create.argtypes = [i, i, i, i, i, ctypes.POINTER(vp)]
    L.fp_index_free.argtypes = [vp]
    L.fp_index_free.restype = None
    L.fp_build_index.argtypes = [vp, vp, i, i, i, i, i, f, f, i, vp, vp, vp, vp]
    L.fp_sparse_attn.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp]
    L.fp_index_info.argtypes = [vp] + [ctypes.POINTER(i)] * 6
    L.fp_index_nnz.argtypes = [vp, ctypes.POINTER(ctypes.c_int64), vp]
    L.fp_index_export.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.fp_get_device_error.argtypes = [vp]
    L.fp_debug_wait_timeout.argtypes = [i, vp]
    L.fp_debug_qk_tile_i8.argtypes = [vp, vp, i, i, i, i, i, i, i, vp, vp]
    L.fp_debug_capture_i8.argtypes = [i, i, i, i, vp]
    L.fp_index_share.argtypes = [vp, f, vp]
    L.fp_index_csr.argtypes = [vp, vp, vp, vp]
    L.fp_index_group_lists.argtypes = [vp, vp, vp, vp, vp]
    L.fp_index_classes.argtypes = [vp, vp, vp]
    L.fp_choose_block_size.argtypes = [vp, f, ctypes.POINTER(i), ctypes.POINTER(f), vp]
    L.fp_pattern_stats_noalloc.argtypes = [vp, vp, i, i, i, i, i, f, i, vp, vp, vp, vp, vp, vp, vp, vp]
    L.fp_strerror.argtypes = [i]
    L.fp_strerror.restype = ctypes.c_char_p
    L.fp_prefill_create.argtypes = [i, i, i, i, i, i, i, ctypes.POINTER(vp)]
    L.fp_prefill_free.argtypes = [vp]
    L.fp_prefill_free.restype = None
    L.fp_prefill_run.argtypes = [vp, vp, vp, vp, vp, vp, f, f, vp, vp]
    L.fp_prefill_enqueue.argtypes = [vp, vp, vp, vp, vp, vp, f, f, vp, vp]
    L.fp_prefill_wait.argtypes = [vp, vp]
    L.fp_prefill_group_index.argtypes = [vp, i, ctypes.POINTER(vp)]
    L.fp_rope_pool.argtypes = [vp, vp, vp, vp, i, i, i, i, i, vp, vp, vp, vp, vp]
    L.fp_build_index_pooled.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, f, vp, vp]
    L.fp_varlen_create.argtypes = [vp, i, i, i, i, i, ctypes.POINTER(vp)]
    L.fp_varlen_free.argtypes = [vp]
    L.fp_varlen_free.restype = None
    L.fp_varlen_build_index.argtypes = [vp, vp, vp, f, f, i, vp, vp, vp]
    L.fp_varlen_sparse_attn.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp]
    L.fp_varlen_index.argtypes = [vp, i, ctypes.POINTER(vp)]
    for s in SYMBOLS:
        if s not in ("fp_index_free", "fp_strerror", "fp_prefill_free", "fp_varlen_free"):
            getattr(L, s).restype = i
    return L


_lib = _load()


def lib():
    return _lib


def library_path():
    return _LIB_PATH


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc, where):
    if rc != FP_OK:
        raise FpError(rc, where)


def fp_strerror(code: int) -> str:
    return _lib.fp_strerror(int(code)).decode()


class Index:
    """Owns one fp_index handle (device workspace for one layer shape)."""

    def __init__(self, handle, S, Hq, Hkv, d, b):
        self.handle = handle
        self.S, self.Hq, self.Hkv, self.d, self.b = S, Hq, Hkv, d, b
        self.n = (S + b - 1) // b

    def free(self):
        if self.handle:
            _lib.fp_index_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def fp_index_create(S, Hq, Hkv, d, b) -> Index:
    h = ctypes.c_void_p()
    _check(_lib.fp_index_create(S, Hq, Hkv, d, b, ctypes.byref(h)), "fp_index_create")
    return Index(h.value, S, Hq, Hkv, d, b)


def fp_index_free(idx: Index):
    idx.free()


def fp_build_index(q, k, S, Hq, Hkv, d, b, gamma, tau, qk_dtype, q_scale, k_scale, idx: Index, stream=None):
    _check(_lib.fp_build_index(_ptr(q), _ptr(k), S, Hq, Hkv, d, b, float(gamma), float(tau), int(qk_dtype),
                               _ptr(q_scale), _ptr(k_scale), idx.handle, _stream(stream)), "fp_build_index")


def fp_sparse_attn(q, k, v, q_scale, k_scale, idx: Index, out, stream=None):
    _check(_lib.fp_sparse_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(q_scale), _ptr(k_scale), idx.handle,
                               _ptr(out), _stream(stream)), "fp_sparse_attn")


def fp_rope_pool(q_in, k_in, rope_cos, rope_sin, S, Hq, Hkv, d, b, q_out, k_out, qbar, kbar, stream=None):
    """Rotary embedding of bf16 q_in/k_in into q_out/k_out (may alias) plus block means."""
    _check(_lib.fp_rope_pool(_ptr(q_in), _ptr(k_in), _ptr(rope_cos), _ptr(rope_sin), S, Hq, Hkv, d, b, _ptr(q_out),
                             _ptr(k_out), _ptr(qbar), _ptr(kbar), _stream(stream)), "fp_rope_pool")


def fp_build_index_pooled(q, k, qbar, kbar, S, Hq, Hkv, d, b, gamma, tau, idx: Index, stream=None):
    _check(_lib.fp_build_index_pooled(_ptr(q), _ptr(k), _ptr(qbar), _ptr(kbar), S, Hq, Hkv, d, b, float(gamma),
                                      float(tau), idx.handle, _stream(stream)), "fp_build_index_pooled")


def fp_index_info(idx: Index):
    vals = [ctypes.c_int() for _ in range(6)]
    _check(_lib.fp_index_info(idx.handle, *[ctypes.byref(v) for v in vals]), "fp_index_info")
    return dict(zip(("S", "Hq", "Hkv", "d", "b", "qk_dtype"), [v.value for v in vals]))


def fp_index_nnz(idx: Index, stream=None) -> int:
    v = ctypes.c_int64()
    _check(_lib.fp_index_nnz(idx.handle, ctypes.byref(v), _stream(stream)), "fp_index_nnz")
    return v.value


def fp_index_export(idx: Index, stream=None):
    """Host copies: CSR (row_ptr, col) over rows h*n + r, pattern, jsd, vhat, shat, pest."""
    import numpy as np
    nnz = fp_index_nnz(idx, stream)
    Hn = idx.Hq * idx.n
    row_ptr = np.zeros(Hn + 1, dtype=np.int32)
    col = np.zeros(max(nnz, 1), dtype=np.int32)
    pattern = np.zeros(idx.Hq, dtype=np.uint8)
    jsd = np.zeros(idx.Hq, dtype=np.float32)
    vhat = np.zeros(Hn, dtype=np.float32)
    shat = np.zeros(Hn, dtype=np.float32)
    pest = np.zeros(Hn, dtype=np.float32)
    _check(_lib.fp_index_export(idx.handle, row_ptr.ctypes.data, col.ctypes.data, pattern.ctypes.data,
                                jsd.ctypes.data, vhat.ctypes.data, shat.ctypes.data, pest.ctypes.data,
                                _stream(stream)), "fp_index_export")
    return {"row_ptr": row_ptr, "col": col[:nnz], "pattern": pattern, "jsd": jsd,
            "vhat": vhat.reshape(idx.Hq, idx.n), "shat": shat.reshape(idx.Hq, idx.n),
            "pest": pest.reshape(idx.Hq, idx.n), "nnz": nnz}


def fp_get_device_error(stream=None) -> int:
    return int(_lib.fp_get_device_error(_stream(stream)))


def fp_debug_wait_timeout(timeout_us: int, stream=None):
    _check(_lib.fp_debug_wait_timeout(int(timeout_us), _stream(stream)), "fp_debug_wait_timeout")


def fp_debug_qk_tile_i8(q8, k8, S, Hq, Hkv, d, h, p0, j0, out, stream=None):
    _check(_lib.fp_debug_qk_tile_i8(_ptr(q8), _ptr(k8), S, Hq, Hkv, d, h, p0, j0, _ptr(out), _stream(stream)),
           "fp_debug_qk_tile_i8")


def fp_index_share(idx, eps, stream=None):
    """Head-pattern sharing on a built index: classes by JSD of vhat < eps
    within each GQA group, every member's lists replaced by the class union."""
    _check(_lib.fp_index_share(idx.handle, float(eps), _stream(stream)), "fp_index_share")


def fp_index_csr(idx, row_ptr, col=None, stream=None):
    """Device CSR of the index into caller-owned device int32 tensors
    (row_ptr [Hq*n + 1], col [nnz] or None for the offsets only)."""
    _check(_lib.fp_index_csr(idx.handle, _ptr(row_ptr), _ptr(col), _stream(stream)), "fp_index_csr")


def fp_index_group_lists(idx, grp_ptr, grp_col=None, grp_mask=None, stream=None):
    """Per-(KV head, query block) union lists with head masks into caller-owned
    device tensors (grp_ptr int32 [Hkv*n + 1]; grp_col int32, grp_mask int32
    bit patterns [total], or both None for the offsets only)."""
    _check(_lib.fp_index_group_lists(idx.handle, _ptr(grp_ptr), _ptr(grp_col), _ptr(grp_mask), _stream(stream)),
           "fp_index_group_lists")


def fp_index_classes(idx, stream=None):
    import numpy as np
    cls = np.zeros(idx.Hq, dtype=np.int32)
    _check(_lib.fp_index_classes(idx.handle, cls.ctypes.data, _stream(stream)), "fp_index_classes")
    return cls


def fp_choose_block_size(idx, gamma, stream=None):
    """Block size chosen by the content rule from an index built at b = 128: (b, rho)."""
    b, rho = ctypes.c_int(0), ctypes.c_float(0.0)
    _check(_lib.fp_choose_block_size(idx.handle, float(gamma), ctypes.byref(b), ctypes.byref(rho), _stream(stream)),
           "fp_choose_block_size")
    return b.value, rho.value


def fp_debug_capture_i8(which, h, tile, chunk, out):
    """Arms (out a device int32 [128][128] tensor) or disarms (out None) the
    capture of one raw int8 score tile: which 0 = index pass, 1 = attention."""
    _check(_lib.fp_debug_capture_i8(int(which), int(h), int(tile), int(chunk), _ptr(out)), "fp_debug_capture_i8")


def fp_pattern_stats_noalloc(q, k, S, Hq, Hkv, d, b, tau, qk_dtype, q_scale, k_scale, vhat, shat, pest, jsd,
                             pattern, stream=None):
    """Per-head vhat/shat/pest/jsd/pattern into caller-owned device buffers,
    using the library's fixed scratch array instead of any allocation."""
    _check(_lib.fp_pattern_stats_noalloc(_ptr(q), _ptr(k), S, Hq, Hkv, d, b, float(tau), int(qk_dtype),
                                         _ptr(q_scale), _ptr(k_scale), _ptr(vhat), _ptr(shat), _ptr(pest),
                                         _ptr(jsd), _ptr(pattern), _stream(stream)), "fp_pattern_stats_noalloc")


class Prefill:
    """Owns one fp_prefill pipeline (include/fp_prefill.h): device copies of a
    layer and one index per KV-head group, for host-to-host runs."""

    def __init__(self, S, Hq, Hkv, d, b, qk_dtype=FP_QK_BF16, groups=0):
        h = ctypes.c_void_p()
        _check(_lib.fp_prefill_create(S, Hq, Hkv, d, b, int(qk_dtype), int(groups), ctypes.byref(h)),
               "fp_prefill_create")
        self.handle = h.value
        self.S, self.Hq, self.Hkv, self.d, self.b, self.qk_dtype = S, Hq, Hkv, d, b, qk_dtype
        self.groups = groups if groups else Hkv

    def run(self, h_q, h_k, h_v, h_q_scale, h_k_scale, gamma, tau, h_out, stream=None):
        """Host tensors in, host tensor out (pinned for overlap); asynchronous on `stream`."""
        _check(_lib.fp_prefill_run(self.handle, _ptr(h_q), _ptr(h_k), _ptr(h_v), _ptr(h_q_scale),
                                   _ptr(h_k_scale), float(gamma), float(tau), _ptr(h_out), _stream(stream)),
               "fp_prefill_run")

    def enqueue(self, h_q, h_k, h_v, h_q_scale, h_k_scale, gamma, tau, h_out, stream=None):
        """Queues a run; consecutive runs overlap.  h_out is ready after wait()."""
        _check(_lib.fp_prefill_enqueue(self.handle, _ptr(h_q), _ptr(h_k), _ptr(h_v), _ptr(h_q_scale),
                                       _ptr(h_k_scale), float(gamma), float(tau), _ptr(h_out), _stream(stream)),
               "fp_prefill_enqueue")

    def wait(self, stream=None):
        """Makes `stream` wait for the outputs of every queued run."""
        _check(_lib.fp_prefill_wait(self.handle, _stream(stream)), "fp_prefill_wait")

    def group_index(self, group):
        """The fp_index of KV-head group `group` of the last run (owned by the pipeline)."""
        h = ctypes.c_void_p()
        _check(_lib.fp_prefill_group_index(self.handle, int(group), ctypes.byref(h)), "fp_prefill_group_index")
        hkv = self.Hkv // self.groups if self.groups <= self.Hkv else 1
        idx = Index(h.value, self.S, self.Hq // self.groups, hkv, self.d, self.b)
        idx.free = lambda: None  # owned by the pipeline
        return idx

    def free(self):
        if self.handle:
            _lib.fp_prefill_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


class Varlen:
    """Owns one fp_varlen set (include/fp_sparse.h): one index per packed
    sequence; cu_seqlens is a host sequence of nseq + 1 offsets."""

    def __init__(self, cu_seqlens, Hq, Hkv, d, b):
        import numpy as np
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        h = ctypes.c_void_p()
        _check(_lib.fp_varlen_create(cu.ctypes.data, len(cu) - 1, Hq, Hkv, d, b, ctypes.byref(h)),
               "fp_varlen_create")
        self.handle = h.value
        self.cu, self.Hq, self.Hkv, self.d, self.b = [int(c) for c in cu], Hq, Hkv, d, b

    def build_index(self, q, k, gamma, tau, qk_dtype, q_scale=None, k_scale=None, stream=None):
        _check(_lib.fp_varlen_build_index(self.handle, _ptr(q), _ptr(k), float(gamma), float(tau), int(qk_dtype),
                                          _ptr(q_scale), _ptr(k_scale), _stream(stream)), "fp_varlen_build_index")

    def sparse_attn(self, q, k, v, out, q_scale=None, k_scale=None, stream=None):
        _check(_lib.fp_varlen_sparse_attn(self.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(q_scale), _ptr(k_scale),
                                          _ptr(out), _stream(stream)), "fp_varlen_sparse_attn")

    def index(self, seq):
        """The Index of sequence `seq` (owned by the set), or None when it is empty."""
        h = ctypes.c_void_p()
        _check(_lib.fp_varlen_index(self.handle, int(seq), ctypes.byref(h)), "fp_varlen_index")
        if not h.value:
            return None
        idx = Index(h.value, self.cu[seq + 1] - self.cu[seq], self.Hq, self.Hkv, self.d, self.b)
        idx.free = lambda: None  # owned by the set
        return idx

    def free(self):
        if self.handle:
            _lib.fp_varlen_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass
