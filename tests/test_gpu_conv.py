"""GPU parity for aq_qconv2d_nhwc (implicit GEMM on the tcgen05 kernel)
against the oracle's explicit-im2col convolution, within
|y - y_ref| <= 2e-3 * sum_k |x_k w_hat_k| + 1 ulp_T(y_ref), with w_hat rounded
once to T in the reference (the kernel multiplies T-valued weight tiles)."""
import numpy as np
import pytest
import torch

import oracle
from group_wise_affine_quant_b200 import api, inputs
from tests.gpu_util import DEV, dev_u16, dev_u8, to_dev
from tests.util import check_matmul

pytestmark = pytest.mark.gpu


def _conv_case(B, H, W, Cin, Cout, k, stride, pad, groups, bits, gs, dt, seed):
    x, w = inputs.conv(groups, seed=seed, B=B, H=H, W=W, C=Cin, Cout=Cout, kh=k, kw=k, dt=dt)
    w2 = inputs.flatten_pad_conv_weight(w, gs)
    wq, s, b = api.aq_quantize(to_dev(w2), bits, gs)
    xd = to_dev(x)
    y = api.aq_qconv2d_nhwc(xd, wq, s, b, Cout, k, k, (stride, stride), (pad, pad), groups,
                            bits, gs)
    torch.cuda.synchronize()
    return xd, wq, s, b, y


def _check_full(xd, wq, s, b, y, Cout, k, stride, pad, groups, bits, gs, dt):
    yr, den = oracle.qconv2d_nhwc(dev_u16(xd), dev_u8(wq), dev_u16(s), dev_u16(b), Cout, k, k,
                                  (stride, stride), (pad, pad), groups, bits, gs, dt, w_in_t=True)
    return check_matmul(dev_u16(y).reshape(yr.shape), yr, den, dt)


@pytest.mark.parametrize("B,H,W,Cin,Cout,k,stride,pad,groups", [
    (1, 8, 8, 16, 16, 3, 1, 1, 1),      # pixel tiles are whole rows: TMA boxes
    (2, 8, 16, 32, 32, 3, 1, 1, 2),     # TMA boxes, two conv groups
    (1, 16, 16, 64, 128, 3, 1, 1, 4),   # TMA boxes, Cg = 16
    (1, 9, 7, 16, 24, 3, 1, 1, 1),      # ragged rows: gather path
    (2, 9, 9, 16, 16, 3, 2, 1, 1),      # stride 2: gather path
    (1, 6, 5, 24, 48, 1, 1, 0, 3),      # 1x1, Cg = 8: gather path
    (1, 10, 10, 16, 200, 3, 1, 0, 1),   # no padding, several weight tiles
    (1, 8, 8, 64, 64, 3, 1, 1, 1),      # Cg = 64: one 64-channel box per K-stage
    (2, 8, 16, 128, 96, 3, 1, 1, 2),    # Cg = 64, two conv groups, two images
    (1, 16, 8, 192, 80, 3, 1, 1, 1),    # Cg = 192, ragged weight tile
    (1, 8, 8, 64, 20, 3, 1, 1, 1),      # Cout = 20: rows not a multiple of 8, 2-byte y stores
    (2, 8, 8, 128, 36, 3, 1, 1, 2),     # Cg = 64, 18 rows per group: 2-byte y stores
])
@pytest.mark.parametrize("bits,gs,dt", [(4, 64, 1), (8, 32, 0), (3, 64, 1)])
def test_conv_small(B, H, W, Cin, Cout, k, stride, pad, groups, bits, gs, dt):
    xd, wq, s, b, y = _conv_case(B, H, W, Cin, Cout, k, stride, pad, groups, bits, gs, dt,
                                 seed=Cin + Cout + k)
    _check_full(xd, wq, s, b, y, Cout, k, stride, pad, groups, bits, gs, dt)


@pytest.mark.parametrize("groups", [1, 4])
@pytest.mark.parametrize("bits", [4, 8])
def test_conv_full_size(groups, bits):
    """Conv workload: batch 2, 64x64, Cin = Cout = 320, 3x3, stride 1, pad 1,
    bf16, group 64; sampled outputs against the oracle."""
    gs, dt = 64, 1
    xd, wq, s, b, y = _conv_case(2, 64, 64, 320, 320, 3, 1, 1, groups, bits, gs, dt, seed=groups)
    M = 2 * 64 * 64
    rng = np.random.default_rng(groups * 10 + bits)
    ms = np.concatenate([[0, M - 1, 63, 64, 4095, 4096], rng.integers(0, M, 600)])
    cos = np.concatenate([[0, 319, 79, 80, 160, 240], rng.integers(0, 320, 600)])
    yr, den = oracle.qconv2d_nhwc(dev_u16(xd), dev_u8(wq), dev_u16(s), dev_u16(b), 320, 3, 3,
                                  (1, 1), (1, 1), groups, bits, gs, dt, ms=ms, cos=cos,
                                  w_in_t=True)
    ys = dev_u16(y).reshape(M, 320)[ms, cos]
    check_matmul(ys, yr, den, dt)


def test_conv_matches_qmm_on_explicit_im2col():
    """A 1x1 stride-1 conv is a plain matmul over pixels: the conv and aq_qmm
    on the pixels-by-channels matrix both meet the matmul bound against the
    oracle's product of that matrix (w_hat rounded to T, as both kernels
    dequantize into T)."""
    B, H, W, C, Co, gs, bits = 2, 16, 16, 64, 96, 64, 4
    xd, wq, s, b, y = _conv_case(B, H, W, C, Co, 1, 1, 0, 1, bits, gs, 1, seed=5)
    x2 = xd.reshape(B * H * W, C)
    y2 = api.aq_qmm(x2, wq, s, b, bits, gs)
    torch.cuda.synchronize()
    yr, den = oracle.qmm(dev_u16(x2), dev_u8(wq), dev_u16(s), dev_u16(b), Co, bits, gs, 0, 1,
                         w_in_t=True)
    check_matmul(dev_u16(y).reshape(-1, Co), yr, den, 1, what="1x1 conv")
    check_matmul(dev_u16(y2), yr, den, 1, what="aq_qmm")


@pytest.fixture(autouse=True)
def _no_device_errors():
    """Every conv case must finish without a bounded wait running out."""
    yield
    torch.cuda.synchronize()
    assert api.lib().aq_device_errors() == 0


def test_conv_rejects_unaligned_channels():
    x = torch.zeros((1, 4, 4, 12), dtype=torch.bfloat16, device=DEV)
    wq = torch.zeros((12, 64 * 4 // 8), dtype=torch.uint8, device=DEV)
    s = torch.zeros((12, 1), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(api.AqError) as e:
        api.aq_qconv2d_nhwc(x, wq, s, s, 12, 3, 3, (1, 1), (1, 1), 1, 4, 64)
    assert e.value.status == 2
