"""CPU oracle for paged MQA logits -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import
this package. The product path never imports it: the CUDA library and its
binding fail loudly instead of falling back here.

This module is argument marshalling around oracle.c (ctypes); every number is
computed there, in fp64, from the plain definition. The library is built on
first use (or by the package build step).

logits() and points() can spread the work over host threads (threads=N, or
threads=None for every core this process may use): each thread makes the same
C call on its own rows (or points), so every element is computed by exactly
the same code, in the same order, as in a single-threaded call; only the
assignment of rows to threads changes. ctypes releases the GIL during the
calls, so the threads run in parallel.
"""
from __future__ import annotations

import concurrent.futures
import ctypes
import os
import threading

import numpy as np

from . import build as _build

_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64


def lib() -> ctypes.CDLL:
    """The oracle library. MQA_ORACLE_LIB, if set, names another build of
    oracle.c to load instead (the test suite's planted-mistake check loads
    deliberately broken copies this way, to show that the pins catch them)."""
    global _lib
    with _lock:
        if _lib is None:
            path = os.environ.get("MQA_ORACLE_LIB") or _build.build()
            L = ctypes.CDLL(path)
            L.oracle_e4m3_to_double.restype = ctypes.c_double
            L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            L.oracle_e2m1_to_double.restype = ctypes.c_double
            L.oracle_e2m1_to_double.argtypes = [ctypes.c_uint8]
            L.oracle_bf16_to_double.restype = ctypes.c_double
            L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            L.oracle_schedule.restype = None
            L.oracle_schedule.argtypes = [_P, _I, _I, _P]
            for name in ("oracle_logits_fp8", "oracle_logits_fp4", "oracle_logits_nvfp4"):
                f = getattr(L, name)
                f.restype = None
                f.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _L, _P, _P]
            for name in ("oracle_points_fp8", "oracle_points_fp4", "oracle_points_nvfp4"):
                f = getattr(L, name)
                f.restype = None
                f.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _L, _P, _P]
            L.oracle_decode_tables.restype = None
            L.oracle_decode_tables.argtypes = [_P, _P]
            L.oracle_topk.restype = None
            L.oracle_topk.argtypes = [_P, _P, _I, _I, _I, _I, _P]
            _lib = L
    return _lib


def _np(x, dtype):
    """A C-contiguous numpy array of dtype (torch CPU tensors accepted)."""
    if hasattr(x, "numpy"):
        x = x.detach().cpu().contiguous().numpy()
    a = np.ascontiguousarray(x)
    if a.dtype != dtype:
        a = a.view(dtype) if a.dtype.itemsize == np.dtype(dtype).itemsize else a.astype(dtype)
    return np.ascontiguousarray(a)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def e4m3_to_double(code: int) -> float:
    return lib().oracle_e4m3_to_double(code)


def e2m1_to_double(nibble: int) -> float:
    return lib().oracle_e2m1_to_double(nibble)


def bf16_to_double(bits: int) -> float:
    return lib().oracle_bf16_to_double(bits & 0xFFFF)


def decode_tables():
    """(e4m3 [256], e2m1 [16]) fp64: the tables the logits loops read."""
    e4 = np.empty(256, dtype=np.float64)
    e2 = np.empty(16, dtype=np.float64)
    lib().oracle_decode_tables(_ptr(e4), _ptr(e2))
    return e4, e2


def schedule(context_lens, num_ctas: int) -> np.ndarray:
    """int32 [num_ctas + 1, 2]: (row, unit offset) per CTA start, linear scan."""
    ctx = _np(context_lens, np.int32)
    out = np.zeros((num_ctas + 1, 2), dtype=np.int32)
    lib().oracle_schedule(_ptr(ctx), ctx.size, num_ctas, _ptr(out))
    return out


_KINDS = ("fp8", "fp4", "nvfp4")


def _args(wl):
    qdt = np.uint16 if wl.kind == "fp4" else np.uint8
    return (_np(wl.q, qdt), _np(wl.kv_cache, np.uint8), _np(wl.block_table, np.int32),
            _np(wl.context_lens, np.int32), _np(wl.weights, np.float32))


def host_cores() -> int:
    """Cores this process may run on (its CPU affinity)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _nthreads(threads, work_items):
    n = host_cores() if threads is None else int(threads)
    return max(1, min(n, work_items))


def _run_parallel(nthreads, tasks):
    """Run the callables in `tasks` on nthreads threads (in order if 1)."""
    if nthreads == 1:
        for t in tasks:
            t()
        return
    with concurrent.futures.ThreadPoolExecutor(max_workers=nthreads) as ex:
        for f in [ex.submit(t) for t in tasks]:
            f.result()


def _addr(a: np.ndarray, offset_elems: int = 0):
    return ctypes.c_void_p(a.ctypes.data + offset_elems * a.itemsize)


def logits(wl, with_absw: bool = True, threads=1):
    """Whole output of a workload: (out, absw), fp64 [B, next_n, L] each;
    absw is the per-element tolerance denominator sum_h |w_h| * ReLU(s * score_h).
    threads: 1 (default), N, or None for every core; rows are spread over the
    threads, each row computed by the same C call as in the single-threaded case."""
    q, kv, bt, ctx, w = _args(wl)
    out = np.empty((wl.B, wl.next_n, wl.out_len), dtype=np.float64)
    absw = np.empty_like(out) if with_absw else None
    assert wl.kind in _KINDS, wl.kind
    fn = getattr(lib(), "oracle_logits_" + wl.kind)
    nn, L = wl.next_n, wl.out_len
    q_row = q.size // max(wl.B, 1)        # q elements per batch row (any q layout)
    mp = wl.max_pages_per_row

    def rows(b0, b1):
        def call():
            fn(_addr(q, b0 * q_row), _ptr(kv), _addr(bt, b0 * mp), _addr(ctx, b0),
               _addr(w, b0 * nn * wl.H), b1 - b0, nn, wl.H, wl.D, wl.page_size, mp, L,
               _addr(out, b0 * nn * L), _addr(absw, b0 * nn * L) if absw is not None else None)
        return call

    n = _nthreads(threads, wl.B)
    if n == 1:
        if wl.B > 0:
            rows(0, wl.B)()
    else:
        # one row per task, longest rows first, for balance
        order = np.argsort(-np.asarray(ctx, dtype=np.int64), kind="stable")
        _run_parallel(n, [rows(int(b), int(b) + 1) for b in order])
    return out, absw


def points(wl, idx, threads=1):
    """Selected elements: idx int64 [n, 3] of (b, n, t). Returns (out, absw) fp64 [n].
    threads as for logits(); the points are split into contiguous blocks."""
    q, kv, bt, ctx, w = _args(wl)
    ix = _np(idx, np.int64).reshape(-1, 3)
    out = np.empty(ix.shape[0], dtype=np.float64)
    absw = np.empty_like(out)
    assert wl.kind in _KINDS, wl.kind
    fn = getattr(lib(), "oracle_points_" + wl.kind)

    def block(i0, i1):
        def call():
            fn(_ptr(q), _ptr(kv), _ptr(bt), _ptr(ctx), _ptr(w), wl.next_n, wl.H, wl.D,
               wl.page_size, wl.max_pages_per_row, _addr(ix, 3 * i0), i1 - i0,
               _addr(out, i0), _addr(absw, i0))
        return call

    npts = ix.shape[0]
    n = _nthreads(threads, max(npts, 1))
    step = -(-npts // (4 * n)) if npts else 1
    _run_parallel(n, [block(i, min(npts, i + step)) for i in range(0, npts, step)])
    return out, absw


def topk(logits, context_lens, next_n: int, k: int, by_token: bool = False) -> np.ndarray:
    """int32 [B, next_n, k]: per row the k largest logits' tokens among
    t < ctx_{b,n} (value descending, ties by token ascending), -1 padded.
    With by_token the same tokens are listed in ascending token order.
    logits: fp32 [B, next_n, L]."""
    lg = _np(logits, np.float32)
    B, nn, L = lg.shape
    assert nn == next_n
    ctx = _np(context_lens, np.int32)
    out = np.empty((B, next_n, k), dtype=np.int32)
    lib().oracle_topk(_ptr(lg), _ptr(ctx), B, next_n, L, k, _ptr(out))
    if by_token:
        for b in range(B):
            for n in range(next_n):
                m = int((out[b, n] >= 0).sum())
                out[b, n, :m] = np.sort(out[b, n, :m])
    return out


def library_path() -> str:
    return os.path.abspath(_build.LIB)
