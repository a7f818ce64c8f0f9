"""GPU parity: aq_quantize_fp4 is bit-exact with the oracle's FP4 quantizer
(codes and scale bytes), including the special values, and its output
dequantizes exactly as the oracle's does."""
import numpy as np
import pytest
import torch

import oracle
from group_wise_affine_quant_b200 import _lib, api
from group_wise_affine_quant_b200.inputs import gen, normal
from tests.gpu_util import DEV, TDT, assert_equal_bits, dev_u16, dev_u8, to_dev
from tests.util import check_matmul

pytestmark = pytest.mark.gpu


def _weights(N, K, dt, seed):
    """Rows of log-normal scale, then rows built to hit the edges: all zeros,
    -0, the E2M1 thresholds exactly (absmax 6, so the scale is exactly 1),
    E8M0 scales on both sides of a sqrt(2) mantissa, values so small that the
    scale underflows, so large that E4M3 saturates, and NaN / inf elements."""
    g = gen(seed)
    w = normal((N, K), 1.0, dt, g).float() * torch.exp(torch.randn((N, 1), generator=g) * 2)
    edge = [
        torch.zeros(K),
        -torch.zeros(K),
        torch.tensor([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0,
                      -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, -6.0] * (K // 16)),
        torch.full((K,), 6.0 * 1.4140625),              # mantissa just below sqrt(2)
        torch.full((K,), 6.0 * 1.4150390625),           # just above
        torch.full((K,), 6e-5) * torch.linspace(-1, 1, K),
        torch.full((K,), 3.0e4 if dt == 0 else 1.0e30),
        torch.linspace(-7.0, 7.0, K),
    ]
    for i, r in enumerate(edge[:N]):
        w[i] = r
    w = w.to(TDT[dt])
    if N > len(edge):
        w[len(edge), 5] = float("nan")                  # NaN in a group: ignored by absmax
    if N > len(edge) + 1:
        w[len(edge) + 1, 40] = float("inf")             # inf absmax: E8M0 0xFF / E4M3 448
        w[len(edge) + 1, 41] = -float("inf")
    return w


@pytest.mark.parametrize("dt", [0, 1])
@pytest.mark.parametrize("gs", [16, 32])
def test_quantize_fp4_bit_exact(dt, gs):
    N, K = 41, 7 * 64
    w = _weights(N, K, dt, seed=gs + dt)
    codes, scales = api.aq_quantize_fp4(to_dev(w), gs)
    torch.cuda.synchronize()
    rc, rs = oracle.quantize_fp4(dev_u16(w), gs, dt)
    assert_equal_bits(dev_u8(scales), rs, "scales")
    assert_equal_bits(dev_u8(codes), rc, "codes")
    # the quantizer's output through the GPU dequantizer and the oracle's
    out = api.aq_dequantize(codes, scales, None, K, 4, gs, dtype=TDT[dt])
    torch.cuda.synchronize()
    _, rt = oracle.dequantize(rc, rs, None, N, K, 4, gs, oracle.FP4, dt)
    assert_equal_bits(dev_u16(out), rt, "dequantized", nan_dt=dt)


@pytest.mark.parametrize("gs", [16, 32])
def test_quantize_fp4_error_bound(gs):
    """Finite rows whose scale is not clamped: every element lies within half a
    table step (the E2M1 gaps 0.5 / 1 / 2, times the decoded scale) of its
    code's value, or beyond 6 * scale when the scale byte rounded down."""
    N, K = 64, 1024
    w = normal((N, K), 1.0, 1, gen(7)).float() * torch.exp(torch.randn((N, 1), generator=gen(8)))
    w = w.to(torch.bfloat16)
    codes, scales = api.aq_quantize_fp4(to_dev(w), gs)
    # bf16 holds every E2M1 value times a decoded scale of this range exactly
    wh = api.aq_dequantize(codes, scales, None, K, 4, gs, dtype=torch.bfloat16).cpu().double()
    s = torch.from_numpy(
        oracle.dequantize(np.ones((N, K // 2), np.uint8) * 0x22, dev_u8(scales), None, N, K, 4, gs,
                          oracle.FP4, 1)[0]).double()           # code 2 is 1.0: the decoded scale
    wf = w.double()
    err = (wf - wh).abs()
    step = torch.where(wf.abs() / s < 2, 0.25, torch.where(wf.abs() / s < 4, 0.5, 1.0)) * s
    ok = (err <= step * (1 + 1e-6)) | (wf.abs() >= 6 * s)
    assert bool(ok.all()), err[~ok][:8]


@pytest.mark.parametrize("gs", [16, 32])
def test_quantize_fp4_large_bit_exact(gs):
    """A 4096 x 14336 bf16 weight (a projection of the decode layers)."""
    N, K = 4096, 14336
    w = normal((N, K), 0.02, 1, gen(11 + gs))
    codes, scales = api.aq_quantize_fp4(to_dev(w), gs)
    torch.cuda.synchronize()
    rc, rs = oracle.quantize_fp4(dev_u16(w), gs, 1)
    assert_equal_bits(dev_u8(scales), rs, "scales")
    assert_equal_bits(dev_u8(codes), rc, "codes")


def test_quantize_fp4_feeds_qmv():
    """Quantize, then decode with the FP4 matvec: the result matches the
    oracle's matvec over the oracle's codes."""
    N, K, M = 512, 2048, 3
    w = normal((N, K), 1.0, 1, gen(21))
    x = normal((M, K), 1.0, 1, gen(22))
    codes, scales = api.aq_quantize_fp4(to_dev(w), 32)
    y = api.aq_qmv(to_dev(x), codes, scales, None, 4, 32)
    torch.cuda.synchronize()
    rc, rs = oracle.quantize_fp4(dev_u16(w), 32, 1)
    wh, _ = oracle.dequantize(rc, rs, None, N, K, 4, 32, oracle.FP4, 1)
    xf = x.double().numpy()
    check_matmul(dev_u16(y), xf @ wh.T, np.abs(xf) @ np.abs(wh).T, 1)


def test_quantize_fp4_empty_and_errors():
    w = torch.zeros((0, 64), dtype=torch.bfloat16, device=DEV)
    codes, scales = api.aq_quantize_fp4(w, 32)
    assert codes.shape == (0, 32) and scales.shape == (0, 2)
    with pytest.raises(_lib.AqError):
        api.aq_quantize_fp4(torch.zeros((4, 48), dtype=torch.bfloat16, device=DEV), 16)
    with pytest.raises(_lib.AqError):
        api.aq_quantize_fp4(torch.zeros((4, 64), dtype=torch.bfloat16, device=DEV), 64)
