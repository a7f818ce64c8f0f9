"""GPU parity: aq_quantize and aq_dequantize are bit-exact with the oracle."""
import numpy as np
import pytest
import torch

import oracle
from group_wise_affine_quant_b200 import api
from group_wise_affine_quant_b200.inputs import fp4 as fp4_weights, gen, normal
from tests.gpu_util import DEV, assert_equal_bits, dev_u16, dev_u8, to_dev
from tests.util import f64_to_u16

pytestmark = pytest.mark.gpu

BITS = (2, 3, 4, 5, 6, 8)


def _weights(N, K, dt, seed):
    """Mixed-scale rows with zeros, constant runs and a few exact ties."""
    g = gen(seed)
    w = normal((N, K), 1.0, dt, g).float()
    scale = torch.exp(torch.randn((N, 1), generator=g) * 3)
    w = w * scale
    w[0, :] = 0.0
    if N > 1:
        w[1, :] = 0.375
    if N > 2:
        w[2, ::3] = 0.0
    if N > 3:
        w[3, :] = w[3, :].round()
    return w.to({0: torch.float16, 1: torch.bfloat16}[dt])


@pytest.mark.parametrize("dt", [0, 1])
@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_quantize_bit_exact(dt, bits, gs):
    N, K = 37, 3 * 128
    w = _weights(N, K, dt, seed=bits * 7 + gs)
    wq, s, b = api.aq_quantize(to_dev(w), bits, gs)
    torch.cuda.synchronize()
    rq, rs, rb = oracle.quantize(dev_u16(w), bits, gs, dt)
    assert_equal_bits(dev_u8(wq), rq, "w_q")
    assert_equal_bits(dev_u16(s), rs, "scales")
    assert_equal_bits(dev_u16(b), rb, "biases")
    # dequantize of the same weights
    out = api.aq_dequantize(wq, s, b, K, bits, gs)
    torch.cuda.synchronize()
    _, rt = oracle.dequantize(rq, rs, rb, N, K, bits, gs, oracle.AFFINE, dt)
    assert_equal_bits(dev_u16(out), rt, "dequantized")


@pytest.mark.parametrize("dt", [0, 1])
@pytest.mark.parametrize("bits", BITS)
def test_dequantize_arbitrary_scales_bit_exact(dt, bits):
    """Caller-supplied scales/biases (not from the quantizer): still one rounding."""
    rng = np.random.default_rng(bits)
    N, K, gs = 16, 256, 64
    codes = rng.integers(0, 256, size=(N, K * bits // 8)).astype(np.uint8)
    s = f64_to_u16(rng.standard_normal((N, K // gs)) * 0.01, dt)
    b = f64_to_u16(rng.standard_normal((N, K // gs)) * 0.1, dt)
    from tests.gpu_util import u16_to_dev
    out = api.aq_dequantize(torch.from_numpy(codes).to(DEV), u16_to_dev(s, dt), u16_to_dev(b, dt),
                            K, bits, gs)
    torch.cuda.synchronize()
    _, rt = oracle.dequantize(codes, s, b, N, K, bits, gs, oracle.AFFINE, dt)
    assert_equal_bits(dev_u16(out), rt, "dequantized")


@pytest.mark.parametrize("dt", [0, 1])
@pytest.mark.parametrize("gs", [16, 32])
@pytest.mark.parametrize("scale_range", ["finite", "literal"])
def test_dequantize_fp4_bit_exact(dt, gs, scale_range):
    N, K = 24, 512
    codes, scales = fp4_weights(N, K, gs, scale_range=scale_range, seed=gs)
    out = api.aq_dequantize(codes.to(DEV), scales.to(DEV), None, K, 4, gs,
                            dtype={0: torch.float16, 1: torch.bfloat16}[dt])
    torch.cuda.synchronize()
    _, rt = oracle.dequantize(codes.numpy(), scales.numpy(), None, N, K, 4, gs, oracle.FP4, dt)
    # 0 * inf (a zero code under an infinite fp16 scale) is NaN on both sides
    assert_equal_bits(dev_u16(out), rt, "fp4 dequantized", nan_dt=dt)


@pytest.mark.parametrize("bits", BITS)
def test_quantize_full_size_decode_projection(bits):
    """The largest decode-sweep projection shape, bf16, 8192 x 2048."""
    g = gen(11)
    w = normal((8192, 2048), 0.02, 1, g)
    wq, s, b = api.aq_quantize(to_dev(w), bits, 64)
    torch.cuda.synchronize()
    rq, rs, rb = oracle.quantize(dev_u16(w), bits, 64, 1)
    assert_equal_bits(dev_u8(wq), rq, "w_q")
    assert_equal_bits(dev_u16(s), rs, "scales")
    assert_equal_bits(dev_u16(b), rb, "biases")


def test_quantize_empty_and_guard_bands():
    """N = 0 and K = 0 enqueue nothing; outputs never write past their end."""
    w = torch.zeros((0, 64), dtype=torch.float16, device=DEV)
    api.aq_quantize(w, 4, 64)
    N, K, bits, gs = 5, 64, 3, 32
    w = to_dev(_weights(N, K, 0, 3))
    guard = 0xA5
    wq = torch.full((N * K * bits // 8 + 64,), guard, dtype=torch.uint8, device=DEV)
    s = torch.full((N * 2 + 16,), 7.0, dtype=torch.float16, device=DEV)
    b = torch.full((N * 2 + 16,), 7.0, dtype=torch.float16, device=DEV)
    api.aq_quantize(w, bits, gs, out=(wq[:N * K * bits // 8].view(N, -1), s[:N * 2].view(N, 2),
                                      b[:N * 2].view(N, 2)))
    torch.cuda.synchronize()
    assert torch.all(wq[N * K * bits // 8:] == guard)
    assert torch.all(s[N * 2:] == 7.0) and torch.all(b[N * 2:] == 7.0)
