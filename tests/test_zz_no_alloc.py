"""aq_qmv_noalloc (the no-allocation decode entry point) against aq_qmv.

Called through the C ABI with raw device pointers; two calls in a row, so the
second one also checks that the first left the shared scratch's counters at
zero.  Both results must match aq_qmv within the matmul tolerance
|y - y_ref| <= 2e-3 * sum_k |x_k w_hat_k| + 1 ulp_T(y_ref), with y_ref the
oracle's fp64 product, and aq_qmv's own output is compared the same way.
This file is collected last so that it also runs after every other test.
"""
import pytest
import torch

import oracle
from group_wise_affine_quant_b200 import api, inputs
from group_wise_affine_quant_b200._lib import AQ_ERR_UNSUPPORTED, AQ_OK, lib
from tests.gpu_util import dev_u16, dev_u8, to_dev
from tests.util import check_matmul

pytestmark = pytest.mark.gpu


def _noalloc(x, wq, s, b, y, gs):
    M, K = x.shape
    N = wq.shape[0]
    dt = 1 if x.dtype == torch.bfloat16 else 0
    return lib().aq_qmv_noalloc(x.data_ptr(), wq.data_ptr(), s.data_ptr(), b.data_ptr(),
                                y.data_ptr(), M, N, K, 4, gs, 0, dt,
                                torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M,N,K,gs", [(1, 2048, 2048, 64), (16, 8192, 2048, 64),
                                      (5, 640, 8192, 32), (9, 300, 1024, 128)])
def test_noalloc_matches_qmv_twice(M, N, K, gs):
    g = inputs.gen(1000 + M)
    w = inputs.normal((N, K), 0.02, 1, g)
    x = to_dev(inputs.normal((M, K), 1.0, 1, g))
    wq, s, b = api.aq_quantize(to_dev(w), 4, gs)
    lib().aq_testing_set_qmv_kernel(1)            # aq_qmv on the warp-MMA kernel too
    try:
        y_ref_gpu = api.aq_qmv(x, wq, s, b, 4, gs)
    finally:
        lib().aq_testing_set_qmv_kernel(0)
    ys = []
    for _ in range(2):
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
        assert _noalloc(x, wq, s, b, y, gs) == AQ_OK, lib().aq_last_error()
        ys.append(y)
    torch.cuda.synchronize()
    assert lib().aq_device_errors() == 0
    yr, den = oracle.qmm(dev_u16(x), dev_u8(wq), dev_u16(s), dev_u16(b), N, 4, gs, 0, 1)
    check_matmul(dev_u16(y_ref_gpu), yr, den, 1, what="aq_qmv")
    for i, y in enumerate(ys):
        check_matmul(dev_u16(y), yr, den, 1, what="aq_qmv_noalloc call %d" % i)
        # the same kernel on the same plan: identical to aq_qmv
        assert torch.equal(y, y_ref_gpu)


def test_noalloc_rejects_what_it_cannot_hold():
    # 8-bit weights do not run the warp-MMA decode kernel
    g = inputs.gen(7)
    x = to_dev(inputs.normal((1, 2048), 1.0, 1, g))
    wq, s, b = api.aq_quantize(to_dev(inputs.normal((256, 2048), 0.02, 1, g)), 8, 64)
    y = torch.empty((1, 256), dtype=torch.bfloat16, device=x.device)
    st = lib().aq_qmv_noalloc(x.data_ptr(), wq.data_ptr(), s.data_ptr(), b.data_ptr(),
                              y.data_ptr(), 1, 256, 2048, 8, 64, 0, 1,
                              torch.cuda.current_stream().cuda_stream)
    assert st == AQ_ERR_UNSUPPORTED
    # a shape whose split-K partials exceed the 4 MiB scratch: N = 65536,
    # K = 16384, M = 16 (the weights need not exist: nothing is launched)
    x2 = torch.empty((16, 16384), dtype=torch.bfloat16, device=x.device)
    st = lib().aq_qmv_noalloc(x2.data_ptr(), wq.data_ptr(), s.data_ptr(), b.data_ptr(),
                              y.data_ptr(), 16, 65536, 16384, 4, 64, 0, 1,
                              torch.cuda.current_stream().cuda_stream)
    assert st == AQ_ERR_UNSUPPORTED
    assert b"scratch" in lib().aq_last_error()
