"""ctypes wrapper of the fp64 C oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the package smoke check
and by the benchmark's CPU-baseline leg.  The product path never imports it.
The oracle is compiled with the host C compiler into ``oracle/_build`` on
first use (or by ``build()``), single-threaded, no fast-math.  The
environment variable ORACLE_LIB, when set, names another build of oracle.c
to load instead; only the mutation test of the pins sets it (to builds with
one planted mistake each).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "_build", "liboracle.so")

VS, QA = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into a shared library (gcc -O2, IEEE semantics)."""
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=gnu99",
                               "-shared", "-fPIC", SRC, "-o", tmp, "-lm"])
        os.replace(tmp, LIB)
    return LIB


class Problem(ctypes.Structure):
    _fields_ = [
        ("S", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
        ("b", ctypes.c_int), ("qk_int8", ctypes.c_int),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("q8", ctypes.c_void_p), ("k8", ctypes.c_void_p),
        ("q_scale", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
    ]


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(os.environ.get("ORACLE_LIB") or build())
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        pp = ctypes.POINTER(Problem)
        L.orc_nibble_mul.argtypes = [ctypes.c_int32, ctypes.c_int32]
        L.orc_nibble_mul.restype = ctypes.c_int32
        L.orc_qk_int.argtypes = [pp, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.orc_qk_int.restype = ctypes.c_int64
        L.orc_last_block_stats.argtypes = [pp, ctypes.c_int, dp, dp]
        L.orc_last_block_stats.restype = ctypes.c_double
        L.orc_block_means.argtypes = [pp, ctypes.c_int, ctypes.c_int, dp]
        L.orc_rope_pool.argtypes = [dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, dp, dp]
        L.orc_rope_pool.restype = None
        L.orc_block_means.restype = None
        L.orc_pest.argtypes = [dp, dp, ctypes.c_int, ctypes.c_int, dp]
        L.orc_pest.restype = None
        L.orc_jsd.argtypes = [dp, dp, ctypes.c_int]
        L.orc_jsd.restype = ctypes.c_double
        L.orc_row_scores.argtypes = [ctypes.c_int, ctypes.c_int, dp, dp, dp, dp, ctypes.c_int, dp]
        L.orc_row_scores.restype = None
        L.orc_select.argtypes = [dp, ctypes.c_int, ctypes.c_double, ip, dp]
        L.orc_select.restype = ctypes.c_int
        L.orc_build_index_head.argtypes = [pp, ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                           dp, dp, dp, dp, ip, ip, ip, dp, dp]
        L.orc_build_index_head.restype = ctypes.c_double
        L.orc_attn_rows.argtypes = [pp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ip, ctypes.c_int, dp]
        L.orc_attn_rows.restype = None
        L.orc_qk_int_tile.argtypes = [pp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ip]
        L.orc_qk_int_tile.restype = None
        L.orc_share_classes.argtypes = [dp, ctypes.c_int, ctypes.c_int, ctypes.c_double, ip]
        L.orc_share_classes.restype = None
        L.orc_union_lists.argtypes = [ctypes.POINTER(ip), ip, ctypes.c_int, ctypes.c_int, ip]
        L.orc_union_lists.restype = ctypes.c_int
        L.orc_cover_count.argtypes = [dp, ctypes.c_int, ctypes.c_double]
        L.orc_cover_count.restype = ctypes.c_int
        L.orc_choose_block_size.argtypes = [dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, dp]
        L.orc_choose_block_size.restype = ctypes.c_int
        _lib = L
    return _lib


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _np(t):
    """CPU numpy view (bf16 tensors are viewed as their uint16 bit patterns)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
        return t.numpy().view(np.uint16)
    return t.numpy()


class OracleProblem:
    """Holds host copies of one layer's inputs and the ctypes problem record."""

    def __init__(self, q, k, v, b, q8=None, k8=None, q_scale=None, k_scale=None):
        Hq, S, d = q.shape
        Hkv = k.shape[0]
        self.S, self.Hq, self.Hkv, self.d, self.b = S, Hq, Hkv, d, b
        self.n = (S + b - 1) // b
        self.int8 = q8 is not None
        self._keep = []

        def keep(x):
            if x is None:
                return None
            a = np.ascontiguousarray(_np(x))
            self._keep.append(a)
            return a.ctypes.data

        self.rec = Problem(S, Hq, Hkv, d, b, 1 if self.int8 else 0,
                           keep(q), keep(k), keep(v), keep(q8), keep(k8),
                           keep(q_scale.float() if q_scale is not None else None),
                           keep(k_scale.float() if k_scale is not None else None))

    @property
    def ptr(self):
        return ctypes.byref(self.rec)

    def last_block_stats(self, h):
        n = self.n
        vh, sh = np.zeros(n), np.zeros(n)
        err = lib().orc_last_block_stats(self.ptr, h, _dp(vh), _dp(sh))
        return vh, sh, err

    def block_means(self, which, head):
        out = np.zeros((self.n, self.d))
        lib().orc_block_means(self.ptr, 0 if which == "q" else 1, head, _dp(out))
        return out

    def build_index_head(self, h, gamma, tau, force_pattern=-1, want_scores=True):
        n = self.n
        T = n * (n + 1) // 2
        vh, sh, pe = np.zeros(n), np.zeros(n), np.zeros(n)
        jsd = np.zeros(1)
        pat = np.zeros(1, dtype=np.int32)
        counts = np.zeros(n, dtype=np.int32)
        cols = np.zeros(T, dtype=np.int32)
        scores = np.zeros(T) if want_scores else None
        info = np.zeros((n, 3))
        err = lib().orc_build_index_head(
            self.ptr, h, float(gamma), float(tau), int(force_pattern), _dp(vh), _dp(sh), _dp(pe), _dp(jsd),
            _ip(pat), _ip(counts), _ip(cols), _dp(scores) if scores is not None else None, _dp(info))
        rows = [cols[r * (r + 1) // 2: r * (r + 1) // 2 + counts[r]].copy() for r in range(n)]
        srows = [scores[r * (r + 1) // 2: r * (r + 1) // 2 + r + 1].copy() for r in range(n)] \
            if scores is not None else None
        return {"vhat": vh, "shat": sh, "pest": pe, "jsd": float(jsd[0]), "pattern": int(pat[0]),
                "rows": rows, "scores": srows, "info": info, "rowsum_err": err}

    def attn_rows(self, h, p_lo, p_hi, blocks):
        blocks = np.ascontiguousarray(np.asarray(blocks, dtype=np.int32))
        out = np.zeros((p_hi - p_lo, self.d))
        lib().orc_attn_rows(self.ptr, h, p_lo, p_hi, _ip(blocks), len(blocks), _dp(out))
        return out

    def qk_int_tile(self, h, p0, j0, rows, cols):
        out = np.zeros((rows, cols), dtype=np.int32)
        lib().orc_qk_int_tile(self.ptr, h, p0, j0, rows, cols, _ip(out))
        return out


def nibble_mul(a, b):
    return int(lib().orc_nibble_mul(int(a), int(b)))


def jsd(p, q):
    p = np.ascontiguousarray(p, dtype=np.float64)
    q = np.ascontiguousarray(q, dtype=np.float64)
    return float(lib().orc_jsd(_dp(p), _dp(q), len(p)))


def pest(qbar_last, kbar):
    qbar_last = np.ascontiguousarray(qbar_last, dtype=np.float64)
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    n, d = kbar.shape
    out = np.zeros(n)
    lib().orc_pest(_dp(qbar_last), _dp(kbar), n, d, _dp(out))
    return out


def row_scores(pattern, r, vhat, shat, qbar_r, kbar):
    vhat = np.ascontiguousarray(vhat, dtype=np.float64)
    shat = np.ascontiguousarray(shat, dtype=np.float64)
    qbar_r = np.ascontiguousarray(qbar_r, dtype=np.float64)
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    w = np.zeros(r + 1)
    lib().orc_row_scores(int(pattern), int(r), _dp(vhat), _dp(shat), _dp(qbar_r), _dp(kbar),
                         kbar.shape[1], _dp(w))
    return w


def select(w, r, gamma):
    w = np.ascontiguousarray(w, dtype=np.float64)
    sel = np.zeros(r + 1, dtype=np.int32)
    info = np.zeros(3)
    cnt = lib().orc_select(_dp(w), int(r), float(gamma), _ip(sel), _dp(info))
    return sel[:cnt].copy(), info


def rope_pool(x, cos, sin, b):
    """Rotary embedding (rotate-half, the caller's cos/sin tables [S][d/2])
    of x [H][S][d], each output rounded to bf16, and the block means of the
    rounded rows.  Returns (out [H][S][d] float64, means [H][n][d])."""
    def f64(t):  # values (not bit patterns) as float64
        if isinstance(t, torch.Tensor):
            return t.detach().cpu().to(torch.float64).contiguous().numpy()
        return np.ascontiguousarray(t, dtype=np.float64)
    x, cos, sin = f64(x), f64(cos), f64(sin)
    H, S, d = x.shape
    n = (S + b - 1) // b
    out = np.zeros_like(x)
    means = np.zeros((H, n, d))
    lib().orc_rope_pool(_dp(x), _dp(cos), _dp(sin), H, S, d, b, _dp(out), _dp(means))
    return out, means


def share_classes(vhat_group, eps):
    """Classes of the heads of one GQA group (vhat_group [g][n]): position of
    each head's class representative within the group."""
    v = np.ascontiguousarray(vhat_group, dtype=np.float64)
    g, n = v.shape
    cls = np.zeros(g, dtype=np.int32)
    lib().orc_share_classes(_dp(v), g, n, float(eps), _ip(cls))
    return cls


def union_lists(lists, r):
    """Ascending union of the given ascending block lists of query block r."""
    arrs = [np.ascontiguousarray(np.asarray(x, dtype=np.int32)) for x in lists]
    ptrs = (ctypes.POINTER(ctypes.c_int32) * len(arrs))(*[_ip(a) for a in arrs])
    counts = np.array([len(a) for a in arrs], dtype=np.int32)
    out = np.zeros(r + 1, dtype=np.int32)
    cnt = lib().orc_union_lists(ptrs, _ip(counts), len(arrs), int(r), _ip(out))
    return out[:cnt].copy()


def share_index(heads, g, eps):
    """Head-pattern sharing applied to per-head oracle results (the dicts of
    OracleProblem.build_index_head, in head order): returns (classes per head
    as absolute head indices, rows per head after the class union)."""
    Hq = len(heads)
    n = len(heads[0]["rows"])
    cls_abs = np.zeros(Hq, dtype=np.int64)
    rows = [None] * Hq
    for j in range(Hq // g):
        grp = list(range(j * g, (j + 1) * g))
        cls = share_classes(np.stack([heads[h]["vhat"] for h in grp]), eps)
        for a, h in enumerate(grp):
            cls_abs[h] = grp[int(cls[a])]
        for a, h in enumerate(grp):
            members = [grp[m] for m in range(g) if int(cls[m]) == int(cls[a])]
            rows[h] = [union_lists([heads[m]["rows"][r] for m in members], r) for r in range(n)]
    return cls_abs, rows


def cover_count(v, gamma):
    v = np.ascontiguousarray(v, dtype=np.float64)
    return int(lib().orc_cover_count(_dp(v), len(v), float(gamma)))


def choose_block_size(vhat128, S, gamma):
    """The block-size rule on the b = 128 vertical statistics of every head
    (vhat128 [Hq][n]): returns (b, rho)."""
    v = np.ascontiguousarray(vhat128, dtype=np.float64)
    Hq, n = v.shape
    rho = np.zeros(1)
    b = lib().orc_choose_block_size(_dp(v), Hq, n, int(S), float(gamma), _dp(rho))
    return int(b), float(rho[0])
