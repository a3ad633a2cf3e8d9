"""Python binding of the B200 paged MQA-logits library (libmqa_logits.so).

Argument marshalling only: tensors become device pointers and shapes become
an mqa_logits_params struct; every step of the computation runs in the CUDA
kernels behind the C ABI (include/mqa_logits.h). There is no fallback: if the
library is missing or the device is not a B200 (compute capability 10.0),
the calls raise.

    sched = mqa_logits_schedule(context_lens, num_ctas)
    out = paged_mqa_logits_fp8(q, kv_cache, block_table, context_lens, weights, sched)
    idx = mqa_logits_topk(out, context_lens, k, by_token=True)

mqa_logits_topk_merge merges per-shard top-k lists of a row split over GPUs
by token range (shard.sharded_topk does the exchange). PyTorch is used for
device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

__all__ = [
    "MQALogitsError", "Params", "library", "library_path", "mqa_logits_num_ctas",
    "mqa_logits_schedule", "paged_mqa_logits_fp8", "paged_mqa_logits_fp4",
    "paged_mqa_logits_nvfp4",
    "mqa_logits_version", "mqa_logits_topk", "mqa_logits_topk_merge", "mqa_logits_get_status",
    "mqa_logits_clear_status", "mqa_logits_check_status", "mqa_diag_fp8_gather", "MQA_TOPK_MAX",
    "MQA_TOPK_BY_TOKEN",
    "MQA_TOPK_MERGE_MAX", "MQA_TOPK_MERGE_MAX_SHARDS", "MQA_FLAG_VALIDATE", "MQA_FLAG_NO_PDL",
    "MQA_STATUS_TIMEOUT", "MQA_STATUS_BAD_PAGE", "MQA_STATUS_BAD_CONTEXT",
    "MQA_STATUS_STALE_SCHEDULE", "MQA_STATUS_Q_RANGE", "MQA_STATUS_DEBUG_INVARIANT", "SCHEDULE_UNIT",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
# MQA_LOGITS_DEBUG=1 selects the build with the kernels' pipeline-invariant
# checks (libmqa_logits_debug.so, `python -m paged_mqa_logits_b200.build --debug`).
_LIB_PATH = os.path.join(_HERE, "libmqa_logits_debug.so" if os.environ.get("MQA_LOGITS_DEBUG") == "1"
                         else "libmqa_logits.so")

MQA_TOPK_MAX = 4096
MQA_TOPK_BY_TOKEN = 1
MQA_TOPK_MERGE_MAX = 16384
MQA_TOPK_MERGE_MAX_SHARDS = 8
MQA_FLAG_VALIDATE = 0x1
MQA_FLAG_NO_PDL = 0x2
# Test hook, not part of the stable interface (see the test-hooks section of
# include/mqa_logits.h): the producers skip one unit so a bounded wait expires.
_MQA_FLAG_TEST_DROP_ARRIVE = 0x100
MQA_STATUS_TIMEOUT = 0x1
MQA_STATUS_BAD_PAGE = 0x2
MQA_STATUS_BAD_CONTEXT = 0x4
MQA_STATUS_STALE_SCHEDULE = 0x8
MQA_STATUS_Q_RANGE = 0x10
MQA_STATUS_DEBUG_INVARIANT = 0x20
SCHEDULE_UNIT = 256

_STATUS_NAMES = {0: "MQA_OK", -1: "MQA_ERR_INVALID_ARG", -2: "MQA_ERR_ARCH",
                 -3: "MQA_ERR_CUDA", -4: "MQA_ERR_UNSUPPORTED", -5: "MQA_ERR_DEVICE_CHECK"}


class MQALogitsError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"{_STATUS_NAMES.get(code, code)}: {message}")
        self.code = code


class Params(ctypes.Structure):
    """Mirror of struct mqa_logits_params."""
    _fields_ = [
        ("batch", ctypes.c_int32), ("next_n", ctypes.c_int32), ("num_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32), ("max_pages_per_row", ctypes.c_int32),
        ("out_len", ctypes.c_int32), ("num_ctas", ctypes.c_int32), ("flags", ctypes.c_uint32),
        ("status", ctypes.c_void_p), ("timeout_ns", ctypes.c_uint64),
    ]


_lib = None
_lock = threading.Lock()


def library_path() -> str:
    return _LIB_PATH


def library() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is missing: build it with "
                    "`python -m paged_mqa_logits_b200.build` (there is no fallback path)")
            L = ctypes.CDLL(_LIB_PATH)
            P, I32 = ctypes.c_void_p, ctypes.c_int32
            L.mqa_logits_num_ctas.argtypes = [ctypes.c_int, ctypes.POINTER(I32)]
            L.mqa_logits_schedule.argtypes = [P, I32, I32, P, P]
            for f in (L.paged_mqa_logits_fp8, L.paged_mqa_logits_fp4, L.paged_mqa_logits_nvfp4,
                      L.mqa_diag_fp8_gather):
                f.argtypes = [P, P, P, P, P, P, P, ctypes.POINTER(Params), P]
            L.mqa_logits_topk.argtypes = [P, P, I32, I32, I32, I32, I32, P, P, P]
            L.mqa_logits_topk_merge.argtypes = [P, P, I32, I32, I32, ctypes.POINTER(I32),
                                                ctypes.POINTER(I32), I32, I32, P, P, P]
            L.mqa_logits_get_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), P]
            L.mqa_logits_clear_status.argtypes = [P]
            L.mqa_logits_check_status.argtypes = [P]
            for f in (L.mqa_diag_fp8_gather, L.mqa_logits_num_ctas, L.mqa_logits_schedule,
                      L.paged_mqa_logits_fp8,
                      L.paged_mqa_logits_fp4, L.paged_mqa_logits_nvfp4, L.mqa_logits_topk,
                      L.mqa_logits_topk_merge,
                      L.mqa_logits_get_status, L.mqa_logits_clear_status,
                      L.mqa_logits_check_status):
                f.restype = ctypes.c_int
            L.mqa_logits_last_error.restype = ctypes.c_char_p
            L.mqa_logits_last_error.argtypes = []
            L.mqa_logits_version.restype = ctypes.c_char_p
            L.mqa_logits_version.argtypes = []
            _lib = L
    return _lib


def _check(rc: int):
    if rc != 0:
        msg = library().mqa_logits_last_error().decode(errors="replace")
        raise MQALogitsError(rc, msg)


def _stream_ptr(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev_ptr(t: Optional[torch.Tensor], name: str, dtypes=None) -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    return t.data_ptr()


def mqa_logits_version() -> str:
    return library().mqa_logits_version().decode()


def mqa_logits_get_status(stream=None) -> int:
    """The library's own status word on the current device (MQA_STATUS_* bits
    OR-ed in by every logits kernel), read after the work queued on `stream`."""
    v = ctypes.c_uint32(0)
    _check(library().mqa_logits_get_status(ctypes.byref(v), _stream_ptr(stream)))
    return int(v.value)


def mqa_logits_check_status(stream=None) -> None:
    """Raise MQALogitsError (MQA_ERR_DEVICE_CHECK, naming the bits) if the
    library's status word on the current device has any bit set, after the
    work queued on `stream`; the word is left as it is."""
    _check(library().mqa_logits_check_status(_stream_ptr(stream)))


def mqa_logits_clear_status(stream=None) -> None:
    """Zero the library's status word on the current device (on `stream`)."""
    _check(library().mqa_logits_clear_status(_stream_ptr(stream)))


def mqa_logits_num_ctas(device: Optional[int] = None) -> int:
    """Persistent CTAs per launch on `device` (its SM count)."""
    if device is None:
        device = torch.cuda.current_device()
    n = ctypes.c_int32(0)
    _check(library().mqa_logits_num_ctas(int(device), ctypes.byref(n)))
    return int(n.value)


def mqa_logits_schedule(context_lens: torch.Tensor, num_ctas: Optional[int] = None,
                        schedule: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """GPU split schedule: int32 [num_ctas + 1, 2] of (row, unit offset)."""
    if num_ctas is None:
        num_ctas = mqa_logits_num_ctas(context_lens.device.index)
    if schedule is None:
        schedule = torch.empty(num_ctas + 1, 2, dtype=torch.int32, device=context_lens.device)
    if schedule.numel() != 2 * (num_ctas + 1):
        raise ValueError("schedule must hold (num_ctas + 1) * 2 int32")
    _check(library().mqa_logits_schedule(
        _dev_ptr(context_lens, "context_lens", (torch.int32,)), int(context_lens.numel()),
        int(num_ctas), _dev_ptr(schedule, "schedule", (torch.int32,)), _stream_ptr(stream)))
    return schedule


def _logits(fn, kind, q, kv_cache, block_table, context_lens, weights, schedule, out, page_size,
            out_len, flags, status, timeout_ns, stream, num_heads=None):
    if kind == "nvfp4":
        if q.dim() != 3 or num_heads is None:
            raise ValueError("nvfp4 q must be [B, next_n, H * (D/2 + D/16)] bytes, with num_heads")
        B, next_n, rb = (int(x) for x in q.shape)
        H = int(num_heads)
        if H <= 0 or rb % H or (rb // H) % 9:
            raise ValueError("nvfp4 q rows must hold H * (D/2 + D/16) bytes")
        D = rb // H // 9 * 16
        qt = (torch.uint8,)
        row_bytes = D // 2 + D // 16
    elif q.dim() != 4:
        raise ValueError("q must be [B, next_n, H, D]")
    else:
        B, next_n, H, D = (int(x) for x in q.shape)
    if kind == "fp8":
        qt = (torch.uint8, torch.float8_e4m3fn)
        row_bytes = D + 4
    elif kind == "fp4":
        qt = (torch.bfloat16, torch.int16)
        row_bytes = D // 2 + D // 16
    if kv_cache.dim() == 3:  # [num_pages, page_size, row_bytes]
        page_size = int(kv_cache.shape[1]) if page_size is None else page_size
    num_pages = int(kv_cache.shape[0])
    page_bytes = kv_cache.numel() // max(num_pages, 1) * kv_cache.element_size()
    if page_size is None:
        if page_bytes % row_bytes:
            raise ValueError("kv_cache page size does not match head_dim")
        page_size = page_bytes // row_bytes
    if page_size * row_bytes != page_bytes:
        raise ValueError(f"kv_cache pages hold {page_bytes} bytes, expected page_size*{row_bytes}")
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be [B, max_pages_per_row]")
    if context_lens.numel() != B:
        raise ValueError(f"context_lens must hold B = {B} entries (got {context_lens.numel()})")
    if tuple(weights.shape) != (B, next_n, H):
        raise ValueError(f"weights must be [B, next_n, H] = {[B, next_n, H]} "
                         f"(got {list(weights.shape)})")
    num_ctas = schedule.numel() // 2 - 1
    if out is None:
        if out_len is None:
            raise ValueError("give out or out_len")
        out = torch.empty(B, next_n, out_len, dtype=torch.float32, device=q.device)
    out_len = int(out.shape[-1])
    if tuple(out.shape) != (B, next_n, out_len):
        raise ValueError("out must be [B, next_n, out_len]")
    p = Params(batch=B, next_n=next_n, num_heads=H, head_dim=D, page_size=int(page_size),
               num_pages=num_pages, max_pages_per_row=int(block_table.shape[1]), out_len=out_len,
               num_ctas=int(num_ctas), flags=int(flags),
               status=_dev_ptr(status, "status", (torch.int32,)) or None,
               timeout_ns=int(timeout_ns))
    _check(fn(_dev_ptr(q, "q", qt), _dev_ptr(kv_cache, "kv_cache", (torch.uint8,)),
              _dev_ptr(block_table, "block_table", (torch.int32,)),
              _dev_ptr(context_lens, "context_lens", (torch.int32,)),
              _dev_ptr(weights, "weights", (torch.float32,)),
              _dev_ptr(schedule, "schedule", (torch.int32,)),
              _dev_ptr(out, "out", (torch.float32,)), ctypes.byref(p), _stream_ptr(stream)))
    return out


def paged_mqa_logits_fp8(q, kv_cache, block_table, context_lens, weights, schedule, out=None, *,
                         page_size: Optional[int] = None, out_len: Optional[int] = None,
                         flags: int = 0, status: Optional[torch.Tensor] = None,
                         timeout_ns: int = 0, stream=None) -> torch.Tensor:
    """FP8 logits into out [B, next_n, L] (fp32); see include/mqa_logits.h.

    q: uint8 or float8_e4m3fn [B, next_n, H, D]; kv_cache: uint8
    [num_pages, page_size * (D + 4)] (or [num_pages, page_size, D + 4]);
    block_table int32 [B, max_pages]; context_lens int32 [B]; weights fp32
    [B, next_n, H]; schedule from mqa_logits_schedule."""
    return _logits(library().paged_mqa_logits_fp8, "fp8", q, kv_cache, block_table, context_lens,
                   weights, schedule, out, page_size, out_len, flags, status, timeout_ns, stream)


def mqa_diag_fp8_gather(q, kv_cache, block_table, context_lens, weights, schedule, out=None, *,
                        page_size: Optional[int] = None, out_len: Optional[int] = None,
                        flags: int = 0, status: Optional[torch.Tensor] = None,
                        timeout_ns: int = 0, stream=None) -> torch.Tensor:
    """The FP8 path's data movement alone (include/mqa_logits_diag.h): the
    arguments of paged_mqa_logits_fp8; `out` is not written."""
    return _logits(library().mqa_diag_fp8_gather, "fp8", q, kv_cache, block_table, context_lens,
                   weights, schedule, out, page_size, out_len, flags, status, timeout_ns, stream)


def paged_mqa_logits_fp4(q, kv_cache, block_table, context_lens, weights, schedule, out=None, *,
                         page_size: Optional[int] = None, out_len: Optional[int] = None,
                         flags: int = 0, status: Optional[torch.Tensor] = None,
                         timeout_ns: int = 0, stream=None) -> torch.Tensor:
    """FP4 logits: q bf16 [B, next_n, H, D]; kv_cache uint8
    [num_pages, page_size * (D/2 + D/16)] (packed e2m1 rows, then e4m3 block
    scales). Otherwise as paged_mqa_logits_fp8."""
    return _logits(library().paged_mqa_logits_fp4, "fp4", q, kv_cache, block_table, context_lens,
                   weights, schedule, out, page_size, out_len, flags, status, timeout_ns, stream)


def paged_mqa_logits_nvfp4(q, kv_cache, block_table, context_lens, weights, schedule, out=None,
                           *, num_heads: int, page_size: Optional[int] = None,
                           out_len: Optional[int] = None, flags: int = 0,
                           status: Optional[torch.Tensor] = None, timeout_ns: int = 0,
                           stream=None) -> torch.Tensor:
    """Block-scaled FP4 logits: q uint8 [B, next_n, H * (D/2 + D/16)] (per
    (b, n) row: [H][D/2] packed e2m1 codes, then [H][D/16] e4m3 scales), K in
    the FP4 page format. Otherwise as paged_mqa_logits_fp4."""
    return _logits(library().paged_mqa_logits_nvfp4, "nvfp4", q, kv_cache, block_table,
                   context_lens, weights, schedule, out, page_size, out_len, flags, status,
                   timeout_ns, stream, num_heads=num_heads)


def _topk_outputs(shape, device, indices, values, with_values):
    if indices is None:
        indices = torch.empty(*shape, dtype=torch.int32, device=device)
    if tuple(indices.shape) != tuple(shape):
        raise ValueError(f"indices must be {list(shape)}")
    if with_values and values is None:
        values = torch.empty(*shape, dtype=torch.float32, device=device)
    if values is not None and tuple(values.shape) != tuple(shape):
        raise ValueError(f"values must be {list(shape)}")
    return indices, values


def mqa_logits_topk(logits: torch.Tensor, context_lens: torch.Tensor, k: int,
                    indices: Optional[torch.Tensor] = None, stream=None,
                    by_token: bool = False, values: Optional[torch.Tensor] = None,
                    with_values: bool = False):
    """Per row (b, n) of logits [B, next_n, L]: the k valid tokens of largest
    logit (among equal logits the lower tokens), listed by value descending
    then token ascending, or by token ascending with by_token; -1 padded;
    int32 [B, next_n, k]. Valid tokens: t < ctx_{b,n} (see mqa_logits.h).
    With with_values (or a `values` tensor) also their logits, fp32, -inf
    where the index is -1, and the result is (indices, values)."""
    if logits.dim() != 3:
        raise ValueError("logits must be [B, next_n, out_len]")
    B, next_n, L = (int(x) for x in logits.shape)
    if context_lens.numel() != B:
        raise ValueError(f"context_lens must hold B = {B} entries (got {context_lens.numel()})")
    want = with_values or values is not None
    indices, values = _topk_outputs((B, next_n, k), logits.device, indices, values, want)
    _check(library().mqa_logits_topk(
        _dev_ptr(logits, "logits", (torch.float32,)),
        _dev_ptr(context_lens, "context_lens", (torch.int32,)), B, next_n, L, int(k),
        MQA_TOPK_BY_TOKEN if by_token else 0,
        _dev_ptr(indices, "indices", (torch.int32,)),
        _dev_ptr(values, "values", (torch.float32,)) if values is not None else None,
        _stream_ptr(stream)))
    return (indices, values) if want else indices


def mqa_logits_topk_merge(cand_values: torch.Tensor, cand_tokens: torch.Tensor,
                          token_offsets, token_counts, k: int, by_token: bool = False,
                          indices: Optional[torch.Tensor] = None,
                          values: Optional[torch.Tensor] = None, with_values: bool = False,
                          stream=None):
    """Top-k of a row split by token range over shards, from the shards' own
    top-k lists: cand_values fp32 / cand_tokens int32 [shards, rows, k_in]
    (each shard's local tokens listed by token, -1 empty), token_offsets the
    shards' first global tokens and token_counts their range lengths (ranges
    must ascend without overlap; checked). Returns int32 [rows, k]
    global tokens (and fp32 values with with_values), as one top-k over the
    whole row would (see mqa_logits.h)."""
    if cand_values.dim() != 3 or tuple(cand_tokens.shape) != tuple(cand_values.shape):
        raise ValueError("cand_values and cand_tokens must both be [shards, rows, k_in]")
    S, rows, k_in = (int(x) for x in cand_values.shape)
    offs = [int(o) for o in token_offsets]
    cnts = [int(c) for c in token_counts]
    if len(offs) != S or len(cnts) != S:
        raise ValueError("one token offset and one token count per shard")
    want = with_values or values is not None
    indices, values = _topk_outputs((rows, k), cand_values.device, indices, values, want)
    arr = (ctypes.c_int32 * max(S, 1))(*offs)
    carr = (ctypes.c_int32 * max(S, 1))(*cnts)
    _check(library().mqa_logits_topk_merge(
        _dev_ptr(cand_values, "cand_values", (torch.float32,)),
        _dev_ptr(cand_tokens, "cand_tokens", (torch.int32,)), S, rows, k_in, arr, carr, int(k),
        MQA_TOPK_BY_TOKEN if by_token else 0,
        _dev_ptr(indices, "indices", (torch.int32,)),
        _dev_ptr(values, "values", (torch.float32,)) if values is not None else None,
        _stream_ptr(stream)))
    return (indices, values) if want else indices
