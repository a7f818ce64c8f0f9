"""The failure path of the decode kernel's bounded waits, on the GPU, without
a fault: a test hook (include/aq_testing.h) shortens every wait to 2 ms and
holds the TMA warp back for 50 ms, so the other roles' waits run out.  The
kernel must stop, let nothing in flight outlive it, set bit 0 of
aq_device_errors() and return; the context stays usable, and after the error
is cleared (and the workspace zeroed, as aq.h asks after a device error) the
next call is correct."""
import pytest
import torch

import oracle
from group_wise_affine_quant_b200 import api, inputs
from group_wise_affine_quant_b200._lib import AQ_OK, lib
from tests.gpu_util import dev_u16, dev_u8, to_dev
from tests.util import check_matmul

pytestmark = pytest.mark.gpu


def _case(M, N, K, seed):
    g = inputs.gen(seed)
    w = inputs.normal((N, K), 0.02, 1, g)
    x = to_dev(inputs.normal((M, K), 1.0, 1, g))
    wq, s, b = api.aq_quantize(to_dev(w), 4, 64)
    return x, wq, s, b


@pytest.mark.parametrize("M,N,K", [(1, 2048, 2048), (16, 8192, 2048)])
def test_wait_runs_out_then_next_call_is_correct(M, N, K):
    x, wq, s, b = _case(M, N, K, seed=77 + M)
    torch.cuda.synchronize()
    assert lib().aq_device_errors() == 0
    ws = api.Workspace()
    try:
        lib().aq_testing_set_qmv_kernel(1)                    # the warp-MMA kernel
        lib().aq_testing_set_wait_limit_ns(2_000_000)         # 2 ms
        lib().aq_testing_set_start_delay_ns(50_000_000)       # 50 ms
        api.aq_qmv(x, wq, s, b, 4, 64, workspace=ws)          # the launch itself succeeds
        torch.cuda.synchronize()                               # and the kernel returns
    finally:
        lib().aq_testing_set_wait_limit_ns(0)
        lib().aq_testing_set_start_delay_ns(0)
        lib().aq_testing_set_qmv_kernel(0)
    assert lib().aq_device_errors() & 1, "the bounded waits did not report running out"
    assert lib().aq_testing_clear_device_errors() == AQ_OK
    assert lib().aq_device_errors() == 0
    # the next call, with a fresh workspace, is correct
    y = api.aq_qmv(x, wq, s, b, 4, 64, workspace=api.Workspace())
    torch.cuda.synchronize()
    assert lib().aq_device_errors() == 0
    yr, den = oracle.qmm(dev_u16(x), dev_u8(wq), dev_u16(s), dev_u16(b), N, 4, 64, 0, 1)
    check_matmul(dev_u16(y), yr, den, 1, what="y after a timed-out call")
