"""CPU oracle for paged MQA logits -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import
this package. The product path never imports it: the CUDA library and its
binding fail loudly instead of falling back here.

This module is argument marshalling around oracle.c (ctypes); every number is
computed there, in fp64, single-threaded, from the plain definition. The
library is built on first use (or by the package build step).
"""
from __future__ import annotations

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
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
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


def logits(wl, with_absw: bool = True):
    """Whole output of a workload: (out, absw), fp64 [B, next_n, L] each;
    absw is the per-element tolerance denominator sum_h |w_h| * ReLU(s * score_h)."""
    q, kv, bt, ctx, w = _args(wl)
    out = np.empty((wl.B, wl.next_n, wl.out_len), dtype=np.float64)
    absw = np.empty_like(out) if with_absw else None
    assert wl.kind in _KINDS, wl.kind
    fn = getattr(lib(), "oracle_logits_" + wl.kind)
    fn(_ptr(q), _ptr(kv), _ptr(bt), _ptr(ctx), _ptr(w), wl.B, wl.next_n, wl.H, wl.D,
       wl.page_size, wl.max_pages_per_row, wl.out_len, _ptr(out),
       _ptr(absw) if absw is not None else None)
    return out, absw


def points(wl, idx):
    """Selected elements: idx int64 [n, 3] of (b, n, t). Returns (out, absw) fp64 [n]."""
    q, kv, bt, ctx, w = _args(wl)
    ix = _np(idx, np.int64).reshape(-1, 3)
    out = np.empty(ix.shape[0], dtype=np.float64)
    absw = np.empty_like(out)
    assert wl.kind in _KINDS, wl.kind
    fn = getattr(lib(), "oracle_points_" + wl.kind)
    fn(_ptr(q), _ptr(kv), _ptr(bt), _ptr(ctx), _ptr(w), wl.next_n, wl.H, wl.D,
       wl.page_size, wl.max_pages_per_row, _ptr(ix), ix.shape[0], _ptr(out), _ptr(absw))
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
