"""CPU oracle for two-stage bucketed approximate top-k (TEST INFRASTRUCTURE ONLY).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The product path (the CUDA library and its Python
binding) never does: the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, qsort, double accumulation,
OpenMP across rows only); this module compiles it with gcc and wraps it with
numpy.  The recall formulas live in ``oracle.recall``.

Source: "Approximate Top-k for Increased Parallelism" (arXiv 2412.04358),
pith.science review page, "What carries the argument" and Fig. 2.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()


def _compile(src: str, out: str) -> None:
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.check_call(
        ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra",
         "-o", tmp, src, "-lm"])
    os.replace(tmp, out)


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2 -fopenmp)."""
    with _lock:
        stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
        if force or stale:
            _compile(_SRC, _LIB)
    return _LIB


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _rows_f32(x) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    if x.ndim == 1:
        x = x[None, :]
    assert x.ndim == 2
    return x


def _bf16_bits(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return np.ascontiguousarray(a)
    if a.dtype == np.int16:
        return np.ascontiguousarray(a.view(np.uint16))
    raise TypeError("bf16 inputs are passed as their raw 16-bit patterns (uint16/int16)")


class Oracle:
    """numpy front end of one compiled copy of oracle.c."""

    def __init__(self, libpath: str):
        lib = ctypes.CDLL(libpath)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        lib.oracle_bucketed.argtypes = [p, i64, i64, i64, i64, i64, p, p, p]
        lib.oracle_exact.argtypes = [p, i64, i64, i64, p, p]
        lib.oracle_bucketed_pairs.argtypes = [p, p, i64, i64, i64, i64, p, p]
        lib.oracle_scores.argtypes = [p, i64, i64, p, i64, i64, p]
        lib.oracle_score_topk.argtypes = [p, i64, i64, p, i64, i64, i64, i64, i64, p, p, p]
        lib.oracle_rerank.argtypes = [p, i64, i64, p, i64, i64, p, i64, i64, p, p]
        lib.oracle_sample_row.argtypes = [p, p, i64, ctypes.c_double, ctypes.c_double, p, p]
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        for f in ("oracle_bucketed", "oracle_exact", "oracle_bucketed_pairs", "oracle_scores",
                  "oracle_score_topk", "oracle_sample_row", "oracle_rerank", "oracle_get_threads",
                  "oracle_max_threads"):
            getattr(lib, f).restype = ctypes.c_int
        self.lib = lib
        self.path = libpath

    def set_threads(self, t: int) -> None:
        self.lib.oracle_set_threads(int(t))

    def get_threads(self) -> int:
        return int(self.lib.oracle_get_threads())

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    def bucketed(self, x, k: int, b: int, kb: int, return_candidates: bool = False):
        """Two-stage bucketed top-k of every row of x (float32, [rows, n]).

        Returns (values [rows,k] float32, indices [rows,k] int32[, C per row]).
        """
        x = _rows_f32(x)
        rows, n = x.shape
        ov = np.empty((rows, k), np.float32)
        oi = np.empty((rows, k), np.int32)
        oc = np.empty(rows, np.int64)
        rc = self.lib.oracle_bucketed(_ptr(x), rows, n, k, b, kb, _ptr(ov), _ptr(oi), _ptr(oc))
        if rc:
            raise ValueError("oracle_bucketed failed (%d)" % rc)
        return (ov, oi, oc) if return_candidates else (ov, oi)

    def exact(self, x, k: int):
        """Exact top-k of every row (ties by lowest index), padded with -inf / -1."""
        x = _rows_f32(x)
        rows, n = x.shape
        ov = np.empty((rows, k), np.float32)
        oi = np.empty((rows, k), np.int32)
        rc = self.lib.oracle_exact(_ptr(x), rows, n, k, _ptr(ov), _ptr(oi))
        if rc:
            raise ValueError("oracle_exact failed (%d)" % rc)
        return ov, oi

    def bucketed_pairs(self, values, indices, k: int, b: int, kb: int):
        """Bucketed selection over (value, index) pairs, bucket = index mod b."""
        v = np.ascontiguousarray(np.asarray(values, np.float32).ravel())
        i = np.ascontiguousarray(np.asarray(indices, np.int32).ravel())
        assert v.shape == i.shape
        ov = np.empty(k, np.float32)
        oi = np.empty(k, np.int32)
        rc = self.lib.oracle_bucketed_pairs(_ptr(v), _ptr(i), v.size, k, b, kb, _ptr(ov),
                                            _ptr(oi))
        if rc:
            raise ValueError("oracle_bucketed_pairs failed (%d)" % rc)
        return ov, oi

    def rerank(self, q_bits, K_bits, cand, k: int):
        """Exact scores of each row's distinct candidate indices and their top-k.

        q_bits [rows, d], K_bits [rows, n, d] or [n, d] (bf16 bit patterns),
        cand [rows, c] int32 (-1 = empty).  Returns (values, indices) [rows, k].
        """
        q = _bf16_bits(q_bits)
        K = _bf16_bits(K_bits)
        rows, d = q.shape
        if K.ndim == 2:
            n, stride = K.shape[0], 0
        else:
            n, stride = K.shape[1], K.shape[1] * d
        cidx = np.ascontiguousarray(np.asarray(cand, np.int32))
        c = cidx.shape[1]
        ov = np.empty((rows, k), np.float32)
        oi = np.empty((rows, k), np.int32)
        rc = self.lib.oracle_rerank(_ptr(q), rows, d, _ptr(K), n, stride, _ptr(cidx), c, k,
                                    _ptr(ov), _ptr(oi))
        if rc:
            raise ValueError("oracle_rerank failed (%d)" % rc)
        return ov, oi

    def sample_rows(self, values, indices, temperature: float, u):
        """Top-k sampling tail per row: (tokens [rows] int32, margins [rows])."""
        v = np.ascontiguousarray(np.atleast_2d(np.asarray(values, np.float32)))
        i = np.ascontiguousarray(np.atleast_2d(np.asarray(indices, np.int32)))
        uu = np.asarray(u, np.float64).ravel()
        rows, k = v.shape
        tok = np.empty(rows, np.int32)
        mar = np.empty(rows, np.float64)
        one_t = ctypes.c_int32()
        one_m = ctypes.c_double()
        for r in range(rows):
            rc = self.lib.oracle_sample_row(_ptr(v[r]), _ptr(i[r]), k, 1.0 / float(temperature),
                                            float(uu[r]), ctypes.byref(one_t), ctypes.byref(one_m))
            if rc:
                raise ValueError("oracle_sample_row failed (%d)" % rc)
            tok[r], mar[r] = one_t.value, one_m.value
        return tok, mar

    def scores(self, q_bits, K_bits, kstride: int | None = None):
        """fp64-accumulated scores q . K_i rounded to float32.

        q_bits: [rows, d] bf16 bit patterns.  K_bits: [rows, n, d] (per-row keys)
        or [n, d] (one key matrix shared by all rows).
        """
        q = _bf16_bits(q_bits)
        K = _bf16_bits(K_bits)
        rows, d = q.shape
        if K.ndim == 2:
            n, stride = K.shape[0], 0
        else:
            assert K.shape[0] == rows
            n, stride = K.shape[1], K.shape[1] * d
        if kstride is not None:
            stride = kstride
        assert K.shape[-1] == d
        out = np.empty((rows, n), np.float32)
        rc = self.lib.oracle_scores(_ptr(q), rows, d, _ptr(K), n, stride, _ptr(out))
        if rc:
            raise ValueError("oracle_scores failed (%d)" % rc)
        return out

    def score_topk(self, q_bits, K_bits, k: int, b: int, kb: int):
        """Scores (as in `scores`) followed by bucketed selection on the floats.

        Returns (values, indices, scores).
        """
        q = _bf16_bits(q_bits)
        K = _bf16_bits(K_bits)
        rows, d = q.shape
        if K.ndim == 2:
            n, stride = K.shape[0], 0
        else:
            n, stride = K.shape[1], K.shape[1] * d
        ov = np.empty((rows, k), np.float32)
        oi = np.empty((rows, k), np.int32)
        sc = np.empty((rows, n), np.float32)
        rc = self.lib.oracle_score_topk(_ptr(q), rows, d, _ptr(K), n, stride, k, b, kb,
                                        _ptr(ov), _ptr(oi), _ptr(sc))
        if rc:
            raise ValueError("oracle_score_topk failed (%d)" % rc)
        return ov, oi, sc


_default: Oracle | None = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def variant(c_source: str, workdir: str) -> Oracle:
    """Compile a modified copy of oracle.c (used to plant mistakes in tests)."""
    src = os.path.join(workdir, "oracle_variant.c")
    out = os.path.join(workdir, "liboracle_variant.so")
    with open(src, "w") as f:
        f.write(c_source)
    _compile(src, out)
    return Oracle(out)


def source() -> str:
    with open(_SRC) as f:
        return f.read()


def set_threads(t: int) -> None:
    default().set_threads(t)


def get_threads() -> int:
    return default().get_threads()


def max_threads() -> int:
    return default().max_threads()


def bucketed(x, k, b, kb, return_candidates=False):
    return default().bucketed(x, k, b, kb, return_candidates)


def exact(x, k):
    return default().exact(x, k)


def bucketed_pairs(values, indices, k, b, kb):
    return default().bucketed_pairs(values, indices, k, b, kb)


def scores(q_bits, K_bits, kstride=None):
    return default().scores(q_bits, K_bits, kstride)


def sample_rows(values, indices, temperature, u):
    return default().sample_rows(values, indices, temperature, u)


def rerank(q_bits, K_bits, cand, k):
    return default().rerank(q_bits, K_bits, cand, k)


def score_topk(q_bits, K_bits, k, b, kb):
    return default().score_topk(q_bits, K_bits, k, b, kb)
