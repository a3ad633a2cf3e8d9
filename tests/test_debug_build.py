"""The -DMQA_DEBUG build (libmqa_logits_debug.so): the kernels check their
pipeline invariants -- every work-table entry against its row, context and
schedule range, the roles' unit and tile counts against each other, and the
phase every pipeline barrier ends in -- and raise MQA_STATUS_DEBUG_INVARIANT
when one fails. The CPU test checks that the build exists and exports the
C ABI; the GPU test runs parity cases through it (in a child process, which
loads the debug library instead of the product one) and requires both
oracle-matching logits and a clean status word."""
import ctypes
import os
import subprocess
import sys

import pytest

from paged_mqa_logits_b200 import build as lib_build
from tests.test_abi import declared_functions

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_library_exports_the_abi():
    lib = ctypes.CDLL(lib_build.build(debug=True))
    for n in declared_functions():
        assert hasattr(lib, n), n
    lib.mqa_logits_version.restype = ctypes.c_char_p
    assert lib.mqa_logits_version().decode().endswith("-debug")


CHILD = r"""
import sys
sys.path.insert(0, ROOT)
import torch
import oracle
import paged_mqa_logits_b200 as mq
import workloads
from tests.helpers import compare, run

assert mq.library_path().endswith("libmqa_logits_debug.so"), mq.library_path()
assert mq.mqa_logits_version().endswith("-debug")
mw = workloads.make_workload
cases = [
    (workloads.make_config("tiny"), None),
    # several tiles, ragged tails, every page size and draft count
    (mw("fp8", 5, 1, 64, 128, 64, 1504, [1, 127, 128, 129, 1500], seed=11), None),
    (mw("fp8", 4, 2, 64, 128, 64, 1028, [1, 2, 255, 1027], seed=12), None),
    (mw("fp8", 3, 3, 32, 128, 16, 700, [700, 0, 257], seed=13), None),
    (mw("fp8", 3, 4, 16, 64, 32, 520, [513, 4, 300], seed=14), None),
    (mw("fp8", 3, 1, 128, 128, 128, 900, [899, 384, 1], seed=15), None),
    (mw("fp8", 2, 2, 128, 128, 256, 1100, [1100, 640], seed=16), None),
    (mw("fp8", 4, 1, 8, 32, 8, 400, [399, 33, 0, 256], seed=17), None),
    # one CTA walking several table chunks; many short and empty rows per CTA
    (mw("fp8", 3, 1, 8, 32, 8, 12800, [12800, 9001, 4097], seed=18), 2),
    (mw("fp8", 2, 2, 16, 64, 64, 20000, [20000, 17777], seed=19), 1),
    (mw("fp8", 150, 1, 16, 64, 16, 600, [(37 * i) % 600 if i % 7 else 0 for i in range(150)],
        seed=20), 3),
    # the other two kernels (their table checks)
    (mw("fp4", 3, 1, 32, 128, 64, 1300, [1300, 0, 520], seed=21), None),
    (mw("nvfp4", 3, 1, 32, 128, 64, 1300, [1300, 0, 520], seed=22), None),
    # full-size decode and scheduler-stress workloads
    (workloads.make_config("decode"), None),
    (workloads.make_config("stress"), None),
]
mq.mqa_logits_clear_status()
for wl, S in cases:
    out, _ = run(wl, num_ctas=S)
    torch.cuda.synchronize()
    ref, absw = oracle.logits(wl)
    compare(out.cpu().numpy(), ref, absw)
    st = mq.mqa_logits_get_status()
    assert st == 0, (wl.kind, wl.B, wl.next_n, wl.H, wl.D, wl.page_size, S, hex(st))
print("DEBUG-BUILD-OK", len(cases))
"""


@pytest.mark.gpu
def test_debug_build_keeps_every_invariant():
    lib_build.build(debug=True)
    env = dict(os.environ, MQA_LOGITS_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", CHILD.replace("ROOT", repr(ROOT), 1)], env=env,
                       cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "DEBUG-BUILD-OK" in r.stdout
