"""GPU parity: activation fake quantization (aq_quantize_dequantize_fp) is
bit-exact with the oracle, and the W4A4 matmul (aq_qqmm) meets the matmul
bound over the oracle's fake-quantized x and FP4 weights.  Also runs each of
aq_qmv's kernels on the same shapes through the kernel-choice test hook."""
import numpy as np
import pytest
import torch

import oracle
from group_wise_affine_quant_b200 import _lib, api, inputs
from group_wise_affine_quant_b200.inputs import gen, normal
from tests.gpu_util import DEV, TDT, assert_equal_bits, dev_u16, dev_u8, to_dev
from tests.test_gpu_quantize_fp4 import _weights
from tests.util import check_matmul

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dt", [0, 1])
@pytest.mark.parametrize("gs", [16, 32])
@pytest.mark.parametrize("bits", [4, 8])
def test_fake_quant_bit_exact(dt, gs, bits):
    N, K = 43, 5 * 64
    w = _weights(N, K, dt, seed=3 * gs + bits + dt)
    out = api.aq_quantize_dequantize_fp(to_dev(w), bits, gs)
    torch.cuda.synchronize()
    ref = oracle.quantize_dequantize_fp(dev_u16(w), bits, gs, dt)
    assert_equal_bits(dev_u16(out), ref, "fake-quantized", nan_dt=dt)


def test_fake_quant_in_place_and_large():
    """In place (out = x) on a 4096 x 14336 bf16 activation block."""
    x = to_dev(normal((4096, 14336), 1.0, 1, gen(3)))
    ref = oracle.quantize_dequantize_fp(dev_u16(x), 4, 32, 1)
    api.aq_quantize_dequantize_fp(x, 4, 32, out=x)
    torch.cuda.synchronize()
    assert_equal_bits(dev_u16(x), ref, "in place")


def _qqmm_ref(x, codes, scales, gs, dt):
    N = codes.shape[0]
    return oracle.qqmm(dev_u16(x), dev_u8(codes), dev_u8(scales), N, gs, dt)


@pytest.mark.parametrize("gs", [16, 32])
@pytest.mark.parametrize("M", [1, 5, 16, 17, 64, 300])
def test_qqmm(gs, M):
    dt = M % 2
    N, K = 256, 1024 + 2 * gs
    codes, scales = inputs.fp4(N, K, gs, seed=gs + M)
    x = to_dev(normal((M, K), 1.0, dt, gen(M)))
    y = api.aq_qqmm(x, codes.to(DEV), scales.to(DEV), gs)
    torch.cuda.synchronize()
    yr, den = _qqmm_ref(x, codes, scales, gs, dt)
    check_matmul(dev_u16(y), yr, den, dt)
    assert api.lib().aq_device_errors() == 0


@pytest.mark.parametrize("gs", [16, 32])
@pytest.mark.parametrize("M", [1, 16])
def test_qqmm_full_size_decode(gs, M):
    """The FP4 workload's shape, K = N = 4096, with weights from the FP4
    quantizer and x ~ N(0, 1)."""
    w = to_dev(normal((4096, 4096), 0.02, 1, gen(70 + gs)))
    codes, scales = api.aq_quantize_fp4(w, gs)
    x = to_dev(inputs.fp4_x(M, 4096))
    y = api.aq_qqmm(x, codes, scales, gs)
    torch.cuda.synchronize()
    yr, den = _qqmm_ref(x, codes, scales, gs, 1)
    check_matmul(dev_u16(y), yr, den, 1)


@pytest.mark.parametrize("gs", [16, 32])
def test_qqmm_full_size_m256_sampled(gs):
    codes, scales = inputs.fp4(4096, 4096, gs, seed=9)
    x = to_dev(inputs.fp4_x(256, 4096))
    y = api.aq_qqmm(x, codes.to(DEV), scales.to(DEV), gs)
    torch.cuda.synchronize()
    xh = oracle.quantize_dequantize_fp(dev_u16(x), 4, gs, 1)
    rng = np.random.default_rng(gs)
    ms = np.concatenate([[0, 255], rng.integers(0, 256, 400)])
    ns = np.concatenate([[4095, 0], rng.integers(0, 4096, 400)])
    yr, den = oracle.qmm_sampled(xh, dev_u8(codes), dev_u8(scales), None, 4096, 4, gs, oracle.FP4,
                                 1, ms, ns)
    check_matmul(dev_u16(y)[ms, ns], yr, den, 1)


def test_qqmm_shares_a_workspace_with_qmv():
    """One zero-filled buffer serves aq_qmv and aq_qqmm calls in turn (the
    qmv counters stay where every call keeps them)."""
    ws = api.Workspace()
    N, K = 2048, 4096
    codes, scales = inputs.fp4(N, K, 32, seed=4)
    codes, scales = codes.to(DEV), scales.to(DEV)
    wq, s, b = api.aq_quantize(to_dev(normal((N, K), 0.02, 1, gen(5))), 4, 64)
    x = to_dev(normal((4, K), 1.0, 1, gen(6)))
    for _ in range(3):
        y1 = api.aq_qqmm(x, codes, scales, 32, workspace=ws)
        y2 = api.aq_qmv(x, wq, s, b, 4, 64, workspace=ws)
    # a call whose matmul needs no workspace still keeps x out of the counters
    x1 = to_dev(normal((1, 1056), 1.0, 1, gen(7)))
    c1, s1 = inputs.fp4(256, 1056, 16, seed=8)
    api.aq_qqmm(x1, c1.to(DEV), s1.to(DEV), 16, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws.get(x.device, 1)[:65536].count_nonzero()) == 0
    yr, den = _qqmm_ref(x, codes, scales, 32, 1)
    check_matmul(dev_u16(y1), yr, den, 1)
    yr2, den2 = oracle.qmm(dev_u16(x), dev_u8(wq), dev_u16(s), dev_u16(b), N, 4, 64, 0, 1)
    check_matmul(dev_u16(y2), yr2, den2, 1)
    assert api.lib().aq_device_errors() == 0


@pytest.mark.parametrize("kernel", [0, 1, 2, 3])
@pytest.mark.parametrize("M", [1, 4, 16])
def test_each_qmv_kernel_on_the_decode_shapes(kernel, M):
    """aq_qmv's kernels (automatic choice, warp-MMA, tcgen05 decode, fp32) on
    the same 4-bit g64 projections, each against the exact w_hat product."""
    try:
        _lib.lib().aq_testing_set_qmv_kernel(kernel)
        for name, N, K in inputs.LLAMA_1B_PROJ[:2] + inputs.LLAMA_1B_PROJ[-1:]:
            g = gen(N + K + M + kernel)
            x = to_dev(normal((M, K), 1.0, 1, g))
            wq, s, b = api.aq_quantize(to_dev(normal((N, K), 0.02, 1, g)), 4, 64)
            y = api.aq_qmv(x, wq, s, b, 4, 64)
            torch.cuda.synchronize()
            yr, den = oracle.qmm(dev_u16(x), dev_u8(wq), dev_u16(s), dev_u16(b), N, 4, 64, 0, 1)
            check_matmul(dev_u16(y), yr, den, 1, what="%s kernel %d" % (name, kernel))
    finally:
        _lib.lib().aq_testing_set_qmv_kernel(0)
    assert api.lib().aq_device_errors() == 0
