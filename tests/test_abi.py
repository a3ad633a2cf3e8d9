"""The C ABI library: loads without a GPU, exports every function that
include/mqa_logits.h declares, and rejects bad arguments on the host before
touching the device."""
import ctypes
import os
import re

import pytest
import torch

import paged_mqa_logits_b200 as mq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    """Every function declared in include/*.h."""
    inc = os.path.join(ROOT, "include")
    names = set()
    for f in sorted(os.listdir(inc)):
        if f.endswith(".h"):
            src = re.sub(r"/\*.*?\*/", "", open(os.path.join(inc, f)).read(), flags=re.S)
            names.update(re.findall(r"^\s*(?:int|const char\*)\s+(\w+)\s*\(", src, flags=re.M))
    return sorted(names)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("mqa_logits_schedule", "paged_mqa_logits_fp8", "paged_mqa_logits_fp4",
              "mqa_logits_topk", "mqa_logits_topk_merge", "mqa_logits_get_status",
              "mqa_logits_clear_status", "mqa_logits_check_status", "mqa_diag_fp8_gather",
              "mqa_logits_num_ctas", "mqa_logits_last_error", "mqa_logits_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = mq.library()
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_params_struct_layout_matches_header():
    # int32 x 10, pointer, uint64 -> 56 bytes on LP64
    assert ctypes.sizeof(mq.Params) == 56
    assert mq.Params.status.offset == 40 and mq.Params.timeout_ns.offset == 48


def test_version():
    assert re.match(r"^\d+\.\d+\.\d+$", mq.mqa_logits_version())


def _params(**kw):
    base = dict(batch=2, next_n=1, num_heads=64, head_dim=128, page_size=64, num_pages=4,
                max_pages_per_row=2, out_len=128, num_ctas=148, flags=0, status=None,
                timeout_ns=0)
    base.update(kw)
    return mq.Params(**base)


@pytest.mark.parametrize("kw,code,needle", [
    (dict(next_n=0), -1, "next_n"),
    (dict(next_n=5), -1, "next_n"),
    (dict(num_heads=48), -4, "num_heads"),
    (dict(num_heads=128, next_n=4), -4, "num_heads * next_n"),
    (dict(head_dim=96), -4, "head_dim"),
    (dict(page_size=48), -1, "page_size"),
    (dict(page_size=4), -1, "page_size"),
    (dict(out_len=130), -1, "out_len"),
    (dict(num_ctas=0), -1, "num_ctas"),
    (dict(batch=-1), -1, "batch"),
])
def test_host_checks_reject_bad_params(kw, code, needle):
    lib = mq.library()
    p = _params(**kw)
    fake = 1 << 20  # never dereferenced: checks fail before any launch
    rc = lib.paged_mqa_logits_fp8(fake, fake, fake, fake, fake, fake, fake, ctypes.byref(p), None)
    assert rc == code
    assert needle in lib.mqa_logits_last_error().decode()


def test_host_checks_reject_null_and_misaligned_pointers():
    lib = mq.library()
    p = _params()
    rc = lib.paged_mqa_logits_fp8(None, 16, 16, 16, 16, 16, 16, ctypes.byref(p), None)
    assert rc == -1 and "NULL" in lib.mqa_logits_last_error().decode()
    rc = lib.paged_mqa_logits_fp8(8, 16, 16, 16, 16, 16, 16, ctypes.byref(p), None)
    assert rc == -1 and "aligned" in lib.mqa_logits_last_error().decode()
    rc = lib.paged_mqa_logits_fp8(16, 16, 16, 16, 16, 16, 16, None, None)
    assert rc == -1 and "params" in lib.mqa_logits_last_error().decode()


def test_schedule_host_checks():
    lib = mq.library()
    assert lib.mqa_logits_schedule(16, -1, 148, 16, None) == -1
    assert lib.mqa_logits_schedule(16, 40000, 148, 16, None) == -1
    assert lib.mqa_logits_schedule(16, 4, 0, 16, None) == -1
    assert lib.mqa_logits_schedule(16, 4, 148, None, None) == -1


def test_topk_host_checks():
    lib = mq.library()
    # k out of range, bad next_n, unknown flags, NULL and misaligned pointers:
    # rejected before any launch
    assert lib.mqa_logits_topk(16, 16, 4, 1, 64, 0, 0, 16, None, None) == -1
    assert lib.mqa_logits_topk(16, 16, 4, 1, 64, mq.MQA_TOPK_MAX + 1, 0, 16, None, None) == -1
    assert "k must be" in lib.mqa_logits_last_error().decode()
    assert lib.mqa_logits_topk(16, 16, 4, 0, 64, 8, 0, 16, None, None) == -1
    assert lib.mqa_logits_topk(16, 16, 4, 1, 64, 8, 2, 16, None, None) == -1
    assert "flag" in lib.mqa_logits_last_error().decode()
    assert lib.mqa_logits_topk(None, 16, 4, 1, 64, 8, 0, 16, None, None) == -1
    assert lib.mqa_logits_topk(18, 16, 4, 1, 64, 8, mq.MQA_TOPK_BY_TOKEN, 16, None, None) == -1
    assert "aligned" in lib.mqa_logits_last_error().decode()
    assert lib.mqa_logits_topk(16, 16, 4, 1, 64, 8, 0, 16, 18, None) == -1  # values misaligned
    assert lib.mqa_logits_topk(None, None, 0, 1, 64, 8, 0, None, None, None) == 0  # empty batch


def test_topk_merge_host_checks():
    lib = mq.library()
    offs = (ctypes.c_int32 * 9)(*range(0, 900, 100))
    cnts = (ctypes.c_int32 * 9)(*([100] * 9))
    bad = (ctypes.c_int32 * 2)(100, 50)

    def ok(v, t, S, rows, k_in, o, k, flags, idx, val, stream):
        return lib.mqa_logits_topk_merge(v, t, S, rows, k_in, o, cnts, k, flags, idx, val, stream)
    # shards out of range, too many candidates, k out of range, unknown flags,
    # NULL or decreasing offsets, NULL / misaligned arrays: rejected before any launch
    assert ok(16, 16, 0, 4, 8, offs, 8, 0, 16, None, None) == -1
    assert ok(16, 16, mq.MQA_TOPK_MERGE_MAX_SHARDS + 1, 4, 8, offs, 8, 0, 16, None, None) == -1
    assert ok(16, 16, 2, 4, mq.MQA_TOPK_MERGE_MAX // 2 + 1, offs, 8, 0, 16, None, None) == -1
    assert "k_in" in lib.mqa_logits_last_error().decode()
    assert ok(16, 16, 2, 4, 8, offs, 0, 0, 16, None, None) == -1
    assert ok(16, 16, 2, 4, 8, offs, 8, 4, 16, None, None) == -1
    assert ok(16, 16, 2, 4, 8, None, 8, 0, 16, None, None) == -1
    assert ok(16, 16, 2, 4, 8, bad, 8, 0, 16, None, None) == -1
    assert "overlap" in lib.mqa_logits_last_error().decode()
    # ranges that overlap by one token, or a NULL count array: rejected
    over = (ctypes.c_int32 * 2)(0, 99)
    assert ok(16, 16, 2, 4, 8, over, 8, 0, 16, None, None) == -1
    assert "overlap" in lib.mqa_logits_last_error().decode()
    assert lib.mqa_logits_topk_merge(16, 16, 2, 4, 8, offs, None, 8, 0, 16, None, None) == -1
    touching = (ctypes.c_int32 * 2)(0, 100)
    assert ok(None, None, 2, 0, 8, touching, 8, 0, None, None, None) == 0  # adjacent ranges: fine
    assert ok(None, 16, 2, 4, 8, offs, 8, 0, 16, None, None) == -1
    assert ok(16, 18, 2, 4, 8, offs, 8, 0, 16, None, None) == -1
    assert ok(None, None, 2, 0, 8, offs, 8, 0, None, None, None) == 0  # no rows


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_no_gpu_is_an_error_not_a_fallback():
    lib = mq.library()
    p = _params()
    rc = lib.paged_mqa_logits_fp8(16, 16, 16, 16, 16, 16, 16, ctypes.byref(p), None)
    assert rc in (-2, -3)  # arch or CUDA error: never a silent success
    assert lib.mqa_logits_check_status(None) in (-2, -3)  # no status word to read: an error


def test_logits_bindings_check_shapes_on_the_host():
    """Mismatched context_lens or weights are rejected before any pointer is
    taken: the kernels would otherwise read past those buffers."""
    B, nn, H, D, ps = 3, 2, 64, 128, 64
    q = torch.zeros(B, nn, H, D, dtype=torch.uint8)
    kv = torch.zeros(4, ps * (D + 4), dtype=torch.uint8)
    bt = torch.zeros(B, 2, dtype=torch.int32)
    ctx = torch.zeros(B, dtype=torch.int32)
    w = torch.zeros(B, nn, H)
    sched = torch.zeros(149, 2, dtype=torch.int32)
    with pytest.raises(ValueError, match="context_lens"):
        mq.paged_mqa_logits_fp8(q, kv, bt, ctx[:2], w, sched, out_len=128)
    with pytest.raises(ValueError, match="weights"):
        mq.paged_mqa_logits_fp8(q, kv, bt, ctx, w[:, :1], sched, out_len=128)
    with pytest.raises(ValueError, match="weights"):
        mq.paged_mqa_logits_fp8(q, kv, bt, ctx, w[:, :, :32], sched, out_len=128)
    qb = torch.zeros(B, nn, H, D, dtype=torch.bfloat16)
    kv4 = torch.zeros(4, ps * (D // 2 + D // 16), dtype=torch.uint8)
    with pytest.raises(ValueError, match="context_lens"):
        mq.paged_mqa_logits_fp4(qb, kv4, bt, ctx[:1], w, sched, out_len=128)


def test_status_word_entry_points_reject_bad_args_without_a_gpu():
    lib = mq.library()
    assert lib.mqa_logits_get_status(None, None) == -1
    assert "bits" in lib.mqa_logits_last_error().decode()


def test_topk_bindings_check_shapes_and_devices_on_the_host():
    lg = torch.zeros(2, 1, 16)
    ctx = torch.zeros(2, dtype=torch.int32)
    with pytest.raises(ValueError):
        mq.mqa_logits_topk(torch.zeros(2, 16), ctx, 4)  # not [B, next_n, L]
    with pytest.raises(ValueError):
        mq.mqa_logits_topk(lg, ctx, 4, indices=torch.zeros(2, 1, 5, dtype=torch.int32))
    with pytest.raises(ValueError, match="context_lens"):
        mq.mqa_logits_topk(lg, ctx[:1], 4)  # one context length per batch row
    with pytest.raises(ValueError):
        mq.mqa_logits_topk(lg, ctx, 4)  # host tensors: no CPU path
    v = torch.zeros(2, 3, 4)
    t = torch.zeros(2, 3, 4, dtype=torch.int32)
    with pytest.raises(ValueError):
        mq.mqa_logits_topk_merge(v, t[:, :, :3], [0, 10], [10, 10], 4)  # shapes differ
    with pytest.raises(ValueError):
        mq.mqa_logits_topk_merge(v, t, [0], [10], 4)  # one offset per shard
    with pytest.raises(ValueError):
        mq.mqa_logits_topk_merge(v, t, [0, 10], [10], 4)  # one count per shard
    with pytest.raises(ValueError):
        mq.mqa_logits_topk_merge(v, t, [0, 10], [10, 10], 4)  # host tensors: no CPU path
