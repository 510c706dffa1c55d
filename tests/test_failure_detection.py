"""Failure detection without a GPU fault.

Every kernel that waits on an mbarrier (the attention kernels, the pool and
block-sum rings) waits through one bounded function: after its cycle limit it
gives up, records LH_ERR_TIMEOUT in the device error word and lets the kernel
wind down and return. lh_selftest_timeout runs that function on an mbarrier
nothing ever arrives on (a flag that nothing sets), with a short limit; the
host must then read the timeout, the word must be cleared by the read, and
the context must still run the path correctly.
"""

import pytest
import torch

from long_context_symmetric_b200 import lh

LH_ERR_NULL, LH_ERR_SHAPE, LH_ERR_TIMEOUT = 1, 2, 8


def test_selftest_validates_arguments():
    """Bad arguments are rejected before anything touches the device."""
    f = lh.lib().lh_selftest_timeout
    assert f(1000, None, None) == LH_ERR_NULL
    assert f(0, 1 << 20, None) == LH_ERR_SHAPE
    assert f(3_000_000_000, 1 << 20, None) == LH_ERR_SHAPE


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_context_survives():
    from lhtest import Case, compare_head, run_gpu
    from long_context_symmetric_b200 import synth

    assert lh.get_device_error() == (0, 0)
    gave_up = torch.zeros(1, dtype=torch.int32, device="cuda")
    lh.selftest_timeout(2_000_000, gave_up)          # about 1 ms of SM clock
    torch.cuda.synchronize()
    assert int(gave_up.item()) == 1
    assert lh.get_device_error() == (LH_ERR_TIMEOUT, 900)
    assert lh.get_device_error() == (0, 0)           # the read cleared it

    # the context is still usable: a small forward + backward matches the oracle
    case = Case("after_timeout", 1, 2, 1024, 64, "bf16", 4, 3, 32)
    w = case.workload()
    q, k, v = (x.cuda() for x in synth.make_inputs(w))
    do = synth.make_dout(w).cuda()
    res = run_gpu(case, q, k, v, do)
    for h in range(case.H):
        compare_head(case, res, q, k, v, do, 0, h)
