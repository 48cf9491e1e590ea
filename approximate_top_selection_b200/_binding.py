"""Thin Python binding of the C ABI in include/topk_b200.h.

Argument marshalling only: every step of the selection runs in the CUDA
library (libtopk_b200.so).  PyTorch provides device memory and the current
stream; there is no CPU fallback -- a missing library or a non-CUDA tensor is an
error.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

TOPK_OK, TOPK_EINVAL, TOPK_EUNSUPPORTED, TOPK_ECUDA, TOPK_EWORKSPACE, TOPK_ESCRATCH = range(6)
TOPK_OP_BUCKETED, TOPK_OP_EXACT, TOPK_OP_SCORE, TOPK_OP_BUCKETED_BF16 = range(4)

_lib = None
_lock = threading.Lock()


class TopkError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s" % (where, topk_status_string(status)))


def library_path() -> str:
    return _build.LIB


def load_library():
    """Load libtopk_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            path = _build.LIB
            if not os.path.exists(path):
                raise ImportError(
                    "libtopk_b200.so is missing: build it with "
                    "`python -m approximate_top_selection_b200.build`")
            lib = ctypes.CDLL(path)
            i64, i32, p, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
            lib.topk_workspace_bytes.argtypes = [i32, i64, i64, i32, i32, i32, i32]
            lib.topk_workspace_bytes.restype = sz
            lib.topk_bucketed.argtypes = [p, i64, i64, i32, i32, i32, p, p, p, sz, p]
            lib.topk_bucketed.restype = i32
            lib.topk_exact.argtypes = [p, i64, i64, i32, p, p, p, sz, p]
            lib.topk_exact.restype = i32
            lib.score_topk.argtypes = [p, i64, i32, p, i64, i64, i32, i32, i32, p, p, p, p, sz, p]
            lib.score_topk.restype = i32
            lib.topk_bucketed_bf16.argtypes = [p, i64, i64, i32, i32, i32, p, p, p, sz, p]
            lib.topk_bucketed_bf16.restype = i32
            lib.topk_bucketed_noalloc.argtypes = [p, i64, i64, i32, i32, i32, p, p, p]
            lib.topk_bucketed_noalloc.restype = i32
            lib.topk_bucketed_merge.argtypes = [p, p, i32, i64, i32, ctypes.POINTER(ctypes.c_int64),
                                                i64, i32, i32, i32, p, p, p]
            lib.topk_bucketed_merge.restype = i32
            lib.score_rerank.argtypes = [p, i64, i32, p, i64, i64, p, i32, i32, p, p, p, p]
            lib.score_rerank.restype = i32
            lib.topk_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, p]
            lib.topk_selftest_wait_timeout.restype = i32
            f32 = ctypes.c_float
            lib.topk_sample_rows.argtypes = [p, p, i64, i32, f32, p, p, p]
            lib.topk_sample_rows.restype = i32
            lib.topk_sample.argtypes = [p, i64, i64, i32, i32, i32, f32, p, p, p, p, p, sz, p]
            lib.topk_sample.restype = i32
            lib.topk_sample_bf16.argtypes = [p, i64, i64, i32, i32, i32, f32, p, p, p, p, p, sz, p]
            lib.topk_sample_bf16.restype = i32
            lib.topk_status_string.argtypes = [i32]
            lib.topk_status_string.restype = ctypes.c_char_p
            lib.topk_device_status.argtypes = [ctypes.POINTER(ctypes.c_int)]
            lib.topk_device_status.restype = i32
            _lib = lib
    return _lib


def topk_status_string(status: int) -> str:
    return load_library().topk_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != TOPK_OK:
        raise TopkError(status, where)


def _stream_handle(stream, device_index: int) -> int:
    """cudaStream_t of `stream`, or of the device's current stream."""
    if stream is None:
        return torch._C._cuda_getCurrentRawStream(device_index)
    return int(stream.cuda_stream)


class _OnDevice:
    """Makes the tensor's device current for a call, switching only when it
    is not current already (a device context costs microseconds per call).

    With an explicit `stream`, that stream is also made torch's current stream
    for the call, so the outputs and the zero-filled workspace the binding
    allocates are created (and the workspace zeroed) on the stream the kernel
    runs on: the kernel is ordered after the fill, and the caching allocator
    recycles those blocks only for later work of that same stream."""

    __slots__ = ("index", "prev", "stream", "stream_ctx")

    def __init__(self, device: torch.device, stream=None):
        self.index = device.index if device.index is not None else torch.cuda.current_device()
        self.prev = None
        self.stream = stream
        self.stream_ctx = None

    def __enter__(self):
        cur = torch.cuda.current_device()
        if cur != self.index:
            self.prev = cur
            torch.cuda.set_device(self.index)
        if self.stream is not None:
            self.stream_ctx = torch.cuda.stream(self.stream)
            self.stream_ctx.__enter__()
        return self

    def __exit__(self, *exc):
        if self.stream_ctx is not None:
            self.stream_ctx.__exit__(*exc)
        if self.prev is not None:
            torch.cuda.set_device(self.prev)
        return False


def _cuda(t: torch.Tensor, name: str, dtype) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


# One zero-filled workspace per (device, stream); every call leaves it zeroed.
_ws_cache: dict = {}


def _workspace(nbytes: int, device: torch.device, stream: int) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    key = (device.index, stream)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


_ws_bytes_cache: dict = {}


def topk_workspace_bytes(op: int, rows: int, n: int, k: int, b: int = 1, kb: int = 1,
                         d: int = 0) -> int:
    """Workspace bytes of a call on the current device (cached per shape)."""
    key = (torch.cuda.current_device(), op, rows, n, k, b, kb, d)
    v = _ws_bytes_cache.get(key)
    if v is None:
        v = int(load_library().topk_workspace_bytes(op, rows, n, k, b, kb, d))
        _ws_bytes_cache[key] = v
    return v


def _outputs(rows: int, k: int, device, out_vals, out_idx, dtype=torch.float32):
    if out_vals is None:
        out_vals = torch.empty(rows, k, dtype=dtype, device=device)
    if out_idx is None:
        out_idx = torch.empty(rows, k, dtype=torch.int32, device=device)
    _cuda(out_vals, "out_vals", dtype)
    _cuda(out_idx, "out_idx", torch.int32)
    if out_vals.numel() != rows * k or out_idx.numel() != rows * k:
        raise ValueError("outputs must hold rows*k elements")
    return out_vals, out_idx


def topk_bucketed(scores: torch.Tensor, k: int, b: int, kb: int, *, out_vals=None, out_idx=None,
                  workspace: torch.Tensor | None = None, stream=None):
    """Bucketed approximate top-k of every row of `scores` ([rows, n] float32
    or bfloat16, CUDA).

    Returns (values [rows, k] of the input dtype, indices [rows, k] int32),
    best-first, padded with -inf / -1.
    """
    if isinstance(scores, torch.Tensor) and scores.dtype == torch.bfloat16:
        return topk_bucketed_bf16(scores, k, b, kb, out_vals=out_vals, out_idx=out_idx,
                                  workspace=workspace, stream=stream)
    lib = load_library()
    _cuda(scores, "scores", torch.float32)
    if scores.dim() != 2:
        raise ValueError("scores must be [rows, n]")
    rows, n = scores.shape
    with _OnDevice(scores.device, stream) as on:
        sh = _stream_handle(stream, on.index)
        out_vals, out_idx = _outputs(rows, k, scores.device, out_vals, out_idx)
        need = topk_workspace_bytes(TOPK_OP_BUCKETED, rows, n, k, b, kb)
        ws = workspace if workspace is not None else _workspace(need, scores.device, sh)
        st = lib.topk_bucketed(scores.data_ptr(), rows, n, k, b, kb, out_vals.data_ptr(),
                               out_idx.data_ptr(), ws.data_ptr() if ws is not None else None,
                               ws.numel() if ws is not None else 0, sh)
    _check(st, "topk_bucketed")
    return out_vals, out_idx


def topk_bucketed_bf16(scores: torch.Tensor, k: int, b: int, kb: int, *, out_vals=None,
                       out_idx=None, workspace: torch.Tensor | None = None, stream=None):
    """Bucketed approximate top-k of bfloat16 rows; values come back as bf16."""
    lib = load_library()
    _cuda(scores, "scores", torch.bfloat16)
    if scores.dim() != 2:
        raise ValueError("scores must be [rows, n]")
    rows, n = scores.shape
    with _OnDevice(scores.device, stream) as on:
        sh = _stream_handle(stream, on.index)
        out_vals, out_idx = _outputs(rows, k, scores.device, out_vals, out_idx, torch.bfloat16)
        need = topk_workspace_bytes(TOPK_OP_BUCKETED_BF16, rows, n, k, b, kb)
        ws = workspace if workspace is not None else _workspace(need, scores.device, sh)
        st = lib.topk_bucketed_bf16(scores.data_ptr(), rows, n, k, b, kb, out_vals.data_ptr(),
                                    out_idx.data_ptr(), ws.data_ptr() if ws is not None else None,
                                    ws.numel() if ws is not None else 0, sh)
    _check(st, "topk_bucketed_bf16")
    return out_vals, out_idx


def topk_bucketed_noalloc(scores: torch.Tensor, k: int, b: int, kb: int, *, out_vals=None,
                          out_idx=None, stream=None):
    """topk_bucketed without a workspace: for callers that must not allocate
    device memory when they select (the library's built-in scratch buffer is
    used instead; see include/topk_b200.h).  Pass preallocated out_vals /
    out_idx to allocate nothing at all on this path.  Calls on different
    streams that overlap on the GPU race on the shared buffer."""
    lib = load_library()
    _cuda(scores, "scores", torch.float32)
    if scores.dim() != 2:
        raise ValueError("scores must be [rows, n]")
    rows, n = scores.shape
    with _OnDevice(scores.device, stream) as on:
        sh = _stream_handle(stream, on.index)
        out_vals, out_idx = _outputs(rows, k, scores.device, out_vals, out_idx)
        st = lib.topk_bucketed_noalloc(scores.data_ptr(), rows, n, k, b, kb, out_vals.data_ptr(),
                                       out_idx.data_ptr(), sh)
    _check(st, "topk_bucketed_noalloc")
    return out_vals, out_idx


def topk_exact(scores: torch.Tensor, k: int, *, out_vals=None, out_idx=None, stream=None):
    """Exact top-k of every row (ties by lowest index), padded with -inf / -1."""
    lib = load_library()
    _cuda(scores, "scores", torch.float32)
    if scores.dim() != 2:
        raise ValueError("scores must be [rows, n]")
    rows, n = scores.shape
    with _OnDevice(scores.device, stream) as on:
        sh = _stream_handle(stream, on.index)
        out_vals, out_idx = _outputs(rows, k, scores.device, out_vals, out_idx)
        st = lib.topk_exact(scores.data_ptr(), rows, n, k, out_vals.data_ptr(),
                            out_idx.data_ptr(), None, 0, sh)
    _check(st, "topk_exact")
    return out_vals, out_idx


def topk_bucketed_merge(vals: torch.Tensor, idx: torch.Tensor, n_total: int, k: int, b: int,
                        kb: int, *, part_offsets=None, out_vals=None, out_idx=None, stream=None):
    """Bucketed top-k over candidate lists (bucket = global index mod b).

    vals: [parts, rows, m] float32, idx: [parts, rows, m] int32 (-1 = empty),
    both on the GPU; part_offsets: `parts` integers added to each part's
    indices (default 0).  With each part's lists = topk_bucketed of a column
    slice of the same rows, the result is topk_bucketed of the whole rows.
    """
    lib = load_library()
    _cuda(vals, "vals", torch.float32)
    _cuda(idx, "idx", torch.int32)
    if vals.dim() == 2:
        vals, idx = vals[None], idx[None]
    if vals.dim() != 3 or tuple(idx.shape) != tuple(vals.shape):
        raise ValueError("vals and idx must both be [parts, rows, m]")
    if idx.device != vals.device:
        raise ValueError("vals and idx must be on the same device")
    parts, rows, m = vals.shape
    offs = [0] * parts if part_offsets is None else [int(o) for o in part_offsets]
    if len(offs) != parts:
        raise ValueError("part_offsets needs one entry per part")
    c_offs = (ctypes.c_int64 * parts)(*offs)
    with _OnDevice(vals.device, stream) as on:
        sh = _stream_handle(stream, on.index)
        out_vals, out_idx = _outputs(rows, k, vals.device, out_vals, out_idx)
        st = lib.topk_bucketed_merge(vals.data_ptr(), idx.data_ptr(), parts, rows, m, c_offs,
                                     n_total, k, b, kb, out_vals.data_ptr(), out_idx.data_ptr(), sh)
    _check(st, "topk_bucketed_merge")
    return out_vals, out_idx


def score_rerank(q: torch.Tensor, K: torch.Tensor, cand_idx: torch.Tensor, k: int, *,
                 return_scores: bool = False, out_vals=None, out_idx=None, stream=None):
    """Exact scores of each row's distinct candidate indices and their top-k.

    q: [rows, d] bf16; K: [rows, n, d] or [n, d] bf16; cand_idx: [rows, c]
    int32 (-1 = empty).  Returns (values, indices[, per-slot scores]).
    """
    lib = load_library()
    _cuda(q, "q", torch.bfloat16)
    _cuda(K, "K", torch.bfloat16)
    _cuda(cand_idx, "cand_idx", torch.int32)
    if q.dim() != 2 or cand_idx.dim() != 2 or cand_idx.shape[0] != q.shape[0]:
        raise ValueError("q must be [rows, d] and cand_idx [rows, c]")
    rows, d = q.shape
    c = cand_idx.shape[1]
    if K.dim() == 3:
        if K.shape[0] != rows or K.shape[2] != d:
            raise ValueError("K must be [rows, n, d] or [n, d]")
        n, kstride = K.shape[1], K.shape[1] * d
    elif K.dim() == 2 and K.shape[1] == d:
        n, kstride = K.shape[0], 0
    else:
        raise ValueError("K must be [rows, n, d] or [n, d]")
    with _OnDevice(q.device, stream) as on:
        sh = _stream_handle(stream, on.index)
        out_vals, out_idx = _outputs(rows, k, q.device, out_vals, out_idx)
        scores = torch.empty(rows, c, dtype=torch.float32, device=q.device) if return_scores else None
        st = lib.score_rerank(q.data_ptr(), rows, d, K.data_ptr(), n, kstride, cand_idx.data_ptr(), c,
                              k, out_vals.data_ptr(), out_idx.data_ptr(),
                              scores.data_ptr() if scores is not None else None, sh)
    _check(st, "score_rerank")
    return (out_vals, out_idx, scores) if return_scores else (out_vals, out_idx)


def topk_sample_rows(vals: torch.Tensor, idx: torch.Tensor, temperature: float, u: torch.Tensor, *,
                     out_token=None, stream=None):
    """One token per row drawn from the softmax (temperature T) of the row's
    selected logits, by inverse CDF with the given uniforms u [rows]."""
    lib = load_library()
    _cuda(vals, "vals", torch.float32)
    _cuda(idx, "idx", torch.int32)
    _cuda(u, "u", torch.float32)
    if vals.dim() != 2 or tuple(idx.shape) != tuple(vals.shape) or u.numel() != vals.shape[0]:
        raise ValueError("vals, idx must be [rows, k] and u [rows]")
    rows, k = vals.shape
    with _OnDevice(vals.device, stream) as on:
        sh = _stream_handle(stream, on.index)
        if out_token is None:
            out_token = torch.empty(rows, dtype=torch.int32, device=vals.device)
        _cuda(out_token, "out_token", torch.int32)
        st = lib.topk_sample_rows(vals.data_ptr(), idx.data_ptr(), rows, k, float(temperature),
                                  u.data_ptr(), out_token.data_ptr(), sh)
    _check(st, "topk_sample_rows")
    return out_token


def topk_sample(logits: torch.Tensor, k: int, b: int, kb: int, temperature: float, u: torch.Tensor, *,
                out_vals=None, out_idx=None, out_token=None, stream=None):
    """Bucketed top-k of float32 or bfloat16 logits [rows, n], then one
    sampled token per row.  Returns (tokens [rows], values [rows, k] of the
    logits' dtype, indices [rows, k])."""
    lib = load_library()
    bf16 = isinstance(logits, torch.Tensor) and logits.dtype == torch.bfloat16
    _cuda(logits, "logits", torch.bfloat16 if bf16 else torch.float32)
    _cuda(u, "u", torch.float32)
    if logits.dim() != 2 or u.numel() != logits.shape[0]:
        raise ValueError("logits must be [rows, n] and u [rows]")
    rows, n = logits.shape
    with _OnDevice(logits.device, stream) as on:
        sh = _stream_handle(stream, on.index)
        out_vals, out_idx = _outputs(rows, k, logits.device, out_vals, out_idx,
                                     dtype=torch.bfloat16 if bf16 else torch.float32)
        if out_token is None:
            out_token = torch.empty(rows, dtype=torch.int32, device=logits.device)
        _cuda(out_token, "out_token", torch.int32)
        nbytes = topk_workspace_bytes(TOPK_OP_BUCKETED_BF16 if bf16 else TOPK_OP_BUCKETED,
                                      rows, n, k, b, kb)
        ws = _workspace(nbytes, logits.device, sh)
        fn = lib.topk_sample_bf16 if bf16 else lib.topk_sample
        st = fn(logits.data_ptr(), rows, n, k, b, kb, float(temperature), u.data_ptr(),
                             out_token.data_ptr(), out_vals.data_ptr(), out_idx.data_ptr(),
                             ws.data_ptr() if ws is not None else None,
                             ws.numel() if ws is not None else 0, sh)
    _check(st, "topk_sample")
    return out_token, out_vals, out_idx


def score_topk(q: torch.Tensor, K: torch.Tensor, k: int, b: int, kb: int, *,
               return_scores: bool = False, out_vals=None, out_idx=None,
               workspace: torch.Tensor | None = None, stream=None):
    """Fused q.K scoring and bucketed top-k.

    q: [rows, d] bfloat16.  K: [rows, n, d] (one key matrix per row) or [n, d]
    (shared by all rows), bfloat16.  Returns (values, indices[, scores]).
    """
    lib = load_library()
    _cuda(q, "q", torch.bfloat16)
    _cuda(K, "K", torch.bfloat16)
    if q.dim() != 2:
        raise ValueError("q must be [rows, d]")
    rows, d = q.shape
    if K.dim() == 3:
        if K.shape[0] != rows:
            raise ValueError("K must be [rows, n, d] or [n, d]")
        n, stride = K.shape[1], K.shape[1] * d
    elif K.dim() == 2:
        n, stride = K.shape[0], 0
    else:
        raise ValueError("K must be [rows, n, d] or [n, d]")
    if K.shape[-1] != d:
        raise ValueError("q and K disagree on d")
    with _OnDevice(q.device, stream) as on:
        sh = _stream_handle(stream, on.index)
        out_vals, out_idx = _outputs(rows, k, q.device, out_vals, out_idx)
        scores = torch.empty(rows, n, dtype=torch.float32, device=q.device) if return_scores else None
        need = topk_workspace_bytes(TOPK_OP_SCORE, rows, n, k, b, kb, d)
        ws = workspace if workspace is not None else _workspace(need, q.device, sh)
        st = lib.score_topk(q.data_ptr(), rows, d, K.data_ptr(), n, stride, k, b, kb,
                            out_vals.data_ptr(), out_idx.data_ptr(),
                            scores.data_ptr() if scores is not None else None,
                            ws.data_ptr() if ws is not None else None,
                            ws.numel() if ws is not None else 0, sh)
    _check(st, "score_topk")
    if return_scores:
        return out_vals, out_idx, scores
    return out_vals, out_idx


def topk_selftest_wait_timeout(limit_ns: int = 1_000_000, stream=None) -> None:
    """Queue a bounded wait that is sure to expire (see the header); the next
    topk_device_status() then reports the expiry."""
    lib = load_library()
    with _OnDevice(torch.device("cuda", torch.cuda.current_device()), stream) as on:
        _check(lib.topk_selftest_wait_timeout(int(limit_ns), _stream_handle(stream, on.index)),
               "topk_selftest_wait_timeout")


def topk_device_status() -> int:
    """Read and clear the device status word (synchronises the device)."""
    v = ctypes.c_int(0)
    _check(load_library().topk_device_status(ctypes.byref(v)), "topk_device_status")
    return int(v.value)
