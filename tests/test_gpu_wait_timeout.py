"""The kernels' bounded waits run out, report, and leave the context usable.

Every wait inside the library's kernels gives up after a time limit and
records GQA_ERR_TIMEOUT in the caller's status word instead of hanging.
gqa_selftest_wait_timeout runs the two wait routines the kernels use (the
suspending and the polling one) on mbarriers that no thread arrives on, with
a short limit, in a kernel that has no copy or MMA in flight.  The test
checks that the kernel returns after about the limit with the status set
and both waits counted as given up, that the control case (barriers
completed first) reports nothing, and that a decode on the same context
afterwards still matches the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, f64
from grouped_query_attention_03_b200 import synthetic

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
GQA_ERR_TIMEOUT = 11


def _timed(fn):
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    out = fn()
    b.record()
    torch.cuda.synchronize(DEV)
    return out, a.elapsed_time(b)


def test_completed_barriers_report_nothing(cuda_lib):
    torch.cuda.set_device(DEV)
    (status, gave_up), ms = _timed(lambda: cuda_lib.selftest_wait_timeout(
        200000, arrive=True, device=DEV))
    assert int(status.item()) == 0
    assert gave_up.tolist() == [0, 0]
    assert ms < 100.0  # no wait ran anywhere near its 200 ms limit


@pytest.mark.parametrize("limit_us", [2000, 50000])
def test_wait_with_no_arrival_times_out_and_reports(cuda_lib, limit_us):
    torch.cuda.set_device(DEV)
    (status, gave_up), ms = _timed(lambda: cuda_lib.selftest_wait_timeout(
        limit_us, arrive=False, device=DEV))
    assert int(status.item()) == GQA_ERR_TIMEOUT
    assert gave_up.tolist() == [1, 1]  # the suspending and the polling wait
    assert ms >= limit_us / 1e3 * 0.95
    assert ms < limit_us / 1e3 + 1000.0


def test_status_keeps_the_first_error(cuda_lib):
    status = torch.full((1,), 5, dtype=torch.int32, device=DEV)  # an earlier error
    st, gave_up = cuda_lib.selftest_wait_timeout(1000, device=DEV, status=status)
    torch.cuda.synchronize(DEV)
    assert int(st.item()) == 5 and gave_up.tolist() == [1, 1]


def test_context_is_usable_after_a_timeout(cuda_lib):
    cuda_lib.selftest_wait_timeout(1000, device=DEV)
    torch.cuda.synchronize(DEV)
    B, Hq, Hkv, C, d = 2, 8, 2, 700, 128
    q, kc, vc = synthetic.decode_inputs(B, Hq, Hkv, C, d, seed=9)
    lens = [700, 333]
    status = cuda_lib.new_status(DEV)
    o = cuda_lib.decode(q.to(DEV), kc.to(DEV), vc.to(DEV),
                        torch.tensor(lens, dtype=torch.int32, device=DEV), status=status)
    torch.cuda.synchronize(DEV)
    assert int(status.item()) == 0
    want = oracle.decode(f64(q), f64(kc), f64(vc), np.array(lens))
    assert_close(o, want, torch.bfloat16, "decode after a timed-out wait")
