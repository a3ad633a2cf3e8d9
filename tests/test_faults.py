"""Failure detection without a GPU fault: every failure here is made on the
host (bad arguments, a corrupt page index, a stale schedule, a test-only
dropped arrive) and must come back as an error code or a status bit, with
the next call succeeding."""
import numpy as np
import pytest
import torch

import oracle
import paged_mqa_logits_b200 as mq
import workloads
from tests.helpers import compare, run, to_device

pytestmark = pytest.mark.gpu


def _wl(seed=5):
    return workloads.make_workload("fp8", 4, 1, 64, 128, 64, 1024, [1000, 0, 513, 700],
                                   seed=seed)


def _healthy_call_after():
    wl = _wl(seed=9)
    out, _ = run(wl)
    torch.cuda.synchronize()
    ref, absw = oracle.logits(wl)
    compare(out.cpu().numpy(), ref, absw)


def test_bad_args_raise_before_launch():
    wl = _wl()
    d = to_device(wl)
    sched = mq.mqa_logits_schedule(d["ctx"])
    with pytest.raises(mq.MQALogitsError, match="num_heads"):
        mq.paged_mqa_logits_fp8(d["q"][:, :, :48].contiguous(), d["kv"], d["bt"], d["ctx"],
                                d["w"][:, :, :48].contiguous(), sched, page_size=64, out_len=1024)
    with pytest.raises(mq.MQALogitsError, match="out_len"):
        mq.paged_mqa_logits_fp8(d["q"], d["kv"], d["bt"], d["ctx"], d["w"], sched, page_size=64,
                                out_len=1022)
    _healthy_call_after()


def test_validate_flags_bad_page_without_faulting():
    wl = _wl()
    wl.block_table = wl.block_table.clone()
    wl.block_table[0, 3] = wl.num_pages + 1000
    wl.block_table[3, 0] = -7
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mq.mqa_logits_clear_status()
    mq.mqa_logits_check_status()  # a clean word is no error
    run(wl, flags=mq.MQA_FLAG_VALIDATE, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & mq.MQA_STATUS_BAD_PAGE
    # the library's own word as an error code, naming the bit; reading leaves it set
    for _ in range(2):
        with pytest.raises(mq.MQALogitsError, match=r"MQA_ERR_DEVICE_CHECK.*BAD_PAGE"):
            mq.mqa_logits_check_status()
    mq.mqa_logits_clear_status()
    mq.mqa_logits_check_status()
    _healthy_call_after()
    mq.mqa_logits_check_status()


def test_validate_flags_context_beyond_out_len():
    wl = _wl()
    d = to_device(wl)
    d["ctx"][0] = 5000  # > out_len and > max_pages * page_size
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    run(wl, dev=d, flags=mq.MQA_FLAG_VALIDATE, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & mq.MQA_STATUS_BAD_CONTEXT
    _healthy_call_after()


def test_validate_flags_stale_schedule():
    wl = workloads.make_workload("fp8", 4, 1, 64, 128, 64, 1024, [1000, 0, 513, 700], seed=5,
                                 reserve_lens=[1000, 0, 900, 700])
    d = to_device(wl)
    sched = mq.mqa_logits_schedule(d["ctx"])
    d["ctx"][2] = 900  # 513 -> 900 crosses 256-token boundaries
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    run(wl, dev=d, flags=mq.MQA_FLAG_VALIDATE, status=status, schedule=sched)
    torch.cuda.synchronize()
    assert int(status.item()) & mq.MQA_STATUS_STALE_SCHEDULE
    # a fresh schedule for the same lengths is not flagged
    status.zero_()
    run(wl, dev=d, flags=mq.MQA_FLAG_VALIDATE, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


@pytest.mark.parametrize("kind", ["fp8", "fp4"])
@pytest.mark.parametrize("caller_word", [True, False], ids=["caller-status", "null-status"])
def test_dropped_arrive_times_out_and_reports(kind, caller_word):
    """Test hook: the producers never fill one unit, so a consumer's bounded
    wait must expire (50 ms), raise MQA_STATUS_TIMEOUT and let the kernel
    exit; the context stays usable. The bit reaches the library's own status
    word whether or not the caller passed a status pointer."""
    wl = workloads.make_workload(kind, 2, 1, 32 if kind == "fp4" else 64, 128, 64, 2048,
                                 [2048, 1500], seed=11)
    d = to_device(wl)
    sched = mq.mqa_logits_schedule(d["ctx"], 1)  # one CTA: it owns every tile
    mq.mqa_logits_clear_status()
    assert mq.mqa_logits_get_status() == 0
    status = torch.zeros(1, dtype=torch.int32, device="cuda") if caller_word else None
    fn = mq.paged_mqa_logits_fp8 if kind == "fp8" else mq.paged_mqa_logits_fp4
    fn(d["q"], d["kv"], d["bt"], d["ctx"], d["w"], sched, page_size=64, out_len=2048,
       flags=mq._MQA_FLAG_TEST_DROP_ARRIVE, status=status, timeout_ns=50_000_000)
    torch.cuda.synchronize()
    if caller_word:
        assert int(status.item()) & mq.MQA_STATUS_TIMEOUT
    assert mq.mqa_logits_get_status() & mq.MQA_STATUS_TIMEOUT
    mq.mqa_logits_clear_status()
    assert mq.mqa_logits_get_status() == 0
    _healthy_call_after()
    assert mq.mqa_logits_get_status() == 0  # a healthy call raises nothing
