"""GPU parity for aq_qmv and aq_qmv_batched against the oracle, within
|y - y_ref| <= 2e-3 * sum_k |x_k w_hat_k| + 1 ulp_T(y_ref), where y_ref is the
oracle's fp64 product over the EXACT w_hat = s q + b (LUT q * s_T for FP4):
every aq_qmv kernel applies scale and bias in fp32 and never rounds w_hat to
T, for every M from 1 to 16."""
import numpy as np
import pytest
import torch

import oracle
from group_wise_affine_quant_b200 import api, inputs
from tests.gpu_util import DEV, TDT, dev_u16, dev_u8, to_dev
from tests.util import check_matmul, qmv_w_in_t

pytestmark = pytest.mark.gpu

BITS = (2, 3, 4, 5, 6, 8)


def _case(M, N, K, bits, gs, dt, seed, wstd=0.05):
    g = inputs.gen(seed)
    w = inputs.normal((N, K), wstd, dt, g)
    x = inputs.normal((M, K), 1.0, dt, g)
    wq, s, b = api.aq_quantize(to_dev(w), bits, gs)
    return to_dev(x), wq, s, b


def _check(x, wq, s, b, y, bits, gs, dt, mode=0, **kw):
    N = wq.shape[0]
    sc = dev_u8(s) if mode == 1 else dev_u16(s)
    bi = None if b is None else dev_u16(b)
    M, K = x.shape
    yr, den = oracle.qmm(dev_u16(x), dev_u8(wq), sc, bi, N, bits, gs, mode, dt,
                         w_in_t=qmv_w_in_t(M, K, bits, gs, mode))
    return check_matmul(dev_u16(y), yr, den, dt, **kw)


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 13, 16])
@pytest.mark.parametrize("bits", BITS)
def test_qmv_affine_small(M, bits):
    dt = 1 if M % 2 else 0
    gs = {1: 32, 2: 64, 3: 128}[M % 3 + 1]
    x, wq, s, b = _case(M, 100, 5 * 128, bits, gs, dt, seed=M * 10 + bits)
    y = api.aq_qmv(x, wq, s, b, bits, gs)
    torch.cuda.synchronize()
    _check(x, wq, s, b, y, bits, gs, dt)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("K", [32 * 3, 64 * 7, 4096 + 128, 16384])
def test_qmv_ragged_and_split_k(bits, K):
    """K slices that end mid-warp, and long K that splits across CTAs."""
    gs = 32
    M, N = 4, 72
    x, wq, s, b = _case(M, N, K, bits, gs, 1, seed=K + bits)
    y = api.aq_qmv(x, wq, s, b, bits, gs)
    torch.cuda.synchronize()
    _check(x, wq, s, b, y, bits, gs, 1)


@pytest.mark.parametrize("M", [1, 2, 16])
@pytest.mark.parametrize("K", [8192, 8192 + 64])
def test_qmv_split_k_twice_in_a_row(M, K):
    """Long K splits over a cluster of CTAs; two calls give identical results
    (K = 8256 gives rows of scales that are not 16-byte multiples: the fp32
    kernel for M <= 2)."""
    bits, gs, dt = 4, 64, 1
    x, wq, s, b = _case(M, 512, K, bits, gs, dt, seed=5)
    y1 = api.aq_qmv(x, wq, s, b, bits, gs)
    y2 = api.aq_qmv(x, wq, s, b, bits, gs)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    _check(x, wq, s, b, y2, bits, gs, dt)


@pytest.mark.parametrize("M", [1, 3, 16])
@pytest.mark.parametrize("K", [65536, 65536 + 128])
def test_qmv_very_long_k_chunked(M, K):
    """Very long K: 64 stages per slice on the tensor-core decode kernel
    (K = 65536), x staged in chunks on the other kernels (K = 65664)."""
    bits, gs, dt = 4, 128, 0
    x, wq, s, b = _case(M, 40, K, bits, gs, dt, seed=9, wstd=0.01)
    y = api.aq_qmv(x, wq, s, b, bits, gs)
    torch.cuda.synchronize()
    _check(x, wq, s, b, y, bits, gs, dt)


@pytest.mark.parametrize("M", [1, 8])
def test_qmv_tiny_config_fp16(M):
    """Tiny correctness workload: 512 x 512, 4-bit g64, fp16, seed 0."""
    x, w = inputs.tiny(M)
    wq, s, b = api.aq_quantize(to_dev(w), 4, 64)
    torch.cuda.synchronize()
    rq, rs, rb = oracle.quantize(inputs.as_u16(w), 4, 64, 0)
    assert np.array_equal(dev_u8(wq), rq)
    y = api.aq_qmv(to_dev(x), wq, s, b, 4, 64)
    torch.cuda.synchronize()
    _check(to_dev(x), wq, s, b, y, 4, 64, 0)


@pytest.mark.parametrize("name,N,K", inputs.LLAMA_1B_PROJ)
@pytest.mark.parametrize("M", [1, 16])
def test_qmv_decode_projection_full(name, N, K, M):
    """Decode-sweep projections at full size, bf16 4-bit g64."""
    x, wq, s, b = _case(M, N, K, 4, 64, 1, seed=N + K + M, wstd=0.02)
    y = api.aq_qmv(x, wq, s, b, 4, 64)
    torch.cuda.synchronize()
    _check(x, wq, s, b, y, 4, 64, 1)


@pytest.mark.parametrize("gs", [16, 32])
@pytest.mark.parametrize("M", [1, 16])
@pytest.mark.parametrize("dt", [0, 1])
def test_qmv_fp4(gs, M, dt):
    N, K = 96, 1024
    codes, scales = inputs.fp4(N, K, gs, seed=gs + M)
    x = inputs.normal((M, K), 1.0, dt, inputs.gen(M))
    xd, wq, sc = to_dev(x), codes.to(DEV), scales.to(DEV)
    y = api.aq_qmv(xd, wq, sc, None, 4, gs)
    torch.cuda.synchronize()
    _check(xd, wq, sc, None, y, 4, gs, dt, mode=1)


def test_qmv_fp4_literal_scales_nonfinite():
    """E8M0 scales over 0..254: where the exact result overflows bf16 the
    device gives a non-finite value; every other output is within the bound."""
    N, K, gs, M = 64, 1024, 32, 1
    codes, scales = inputs.fp4(N, K, gs, scale_range="literal", seed=3)
    x = inputs.fp4_x(M, K)
    xd, wq, sc = to_dev(x), codes.to(DEV), scales.to(DEV)
    y = api.aq_qmv(xd, wq, sc, None, 4, gs)
    torch.cuda.synchronize()
    _check(xd, wq, sc, None, y, 4, gs, 1, mode=1, overflow_any_nonfinite=True)


def test_qmv_k_zero_and_n_zero():
    x = torch.zeros((3, 0), dtype=torch.float16, device=DEV)
    wq = torch.zeros((5, 0), dtype=torch.uint8, device=DEV)
    s = torch.zeros((5, 0), dtype=torch.float16, device=DEV)
    y = torch.full((3, 5), 9.0, dtype=torch.float16, device=DEV)
    api.aq_qmv(x, wq, s, s, 4, 64, out=y)
    torch.cuda.synchronize()
    assert torch.all(y == 0)
    x = torch.zeros((3, 64), dtype=torch.float16, device=DEV)
    wq = torch.zeros((0, 32), dtype=torch.uint8, device=DEV)
    s = torch.zeros((0, 1), dtype=torch.float16, device=DEV)
    api.aq_qmv(x, wq, s, s, 4, 64)


@pytest.mark.parametrize("gs,scale_range", [(32, "finite"), (16, "finite"), (32, "literal"),
                                            (16, "literal")])
@pytest.mark.parametrize("M", [1, 16])
def test_qmv_fp4_full_size(gs, scale_range, M):
    """FP4 weights at full size, K = N = 4096: E8M0 (group 32) and E4M3
    (group 16) scales over the finite and the literal ranges."""
    N = K = 4096
    codes, scales = inputs.fp4(N, K, gs, scale_range=scale_range, seed=11 + gs + M)
    x = inputs.fp4_x(M, K)
    xd, wq, sc = to_dev(x), codes.to(DEV), scales.to(DEV)
    y = api.aq_qmv(xd, wq, sc, None, 4, gs)
    torch.cuda.synchronize()
    _check(xd, wq, sc, None, y, 4, gs, 1, mode=1,
           overflow_any_nonfinite=scale_range == "literal")


@pytest.mark.parametrize("M", [1, 3, 16])
@pytest.mark.parametrize("bits", BITS)
def test_qmv_batched_matches_single(M, bits):
    """A batch of problems of different shapes (N not a multiple of 128,
    long K that splits) in one call: every output equals the single-problem
    call bit for bit (same fp32 arithmetic, same slice order) and is within
    the bound of the oracle."""
    gs = 64 if bits != 6 else 128
    dt = 1 if M % 2 else 0
    shapes = [(200, 1024), (512, 2048), (72, 4096), (128, 8192), (1000, 1024)]
    cases = [_case(M, n, k, bits, gs, dt, seed=100 * i + bits + M) for i, (n, k) in enumerate(shapes)]
    xs = [c[0] for c in cases]
    ys = api.aq_qmv_batched(xs, [c[1] for c in cases], [c[2] for c in cases],
                            [c[3] for c in cases], bits, gs)
    torch.cuda.synchronize()
    assert api.lib().aq_device_errors() == 0
    for (x, wq, s, b), y in zip(cases, ys):
        _check(x, wq, s, b, y, bits, gs, dt)


@pytest.mark.parametrize("gs", [16, 32])
def test_qmv_batched_fp4(gs):
    shapes = [(256, 1024), (96, 2048), (130, 4096)]
    xs, ws, ss = [], [], []
    for i, (n, k) in enumerate(shapes):
        codes, scales = inputs.fp4(n, k, gs, seed=40 + i + gs)
        xs.append(to_dev(inputs.fp4_x(4, k)))
        ws.append(codes.to(DEV))
        ss.append(scales.to(DEV))
    ys = api.aq_qmv_batched(xs, ws, ss, None, 4, gs)
    torch.cuda.synchronize()
    for x, wq, sc, y in zip(xs, ws, ss, ys):
        _check(x, wq, sc, None, y, 4, gs, 1, mode=1)


def test_qmv_batched_many_problems_two_launches():
    """More problems than one launch holds: the library splits the batch and
    reuses the workspace across launches."""
    M, bits, gs, dt = 2, 4, 64, 1
    cases = [_case(M, 256, 4096, bits, gs, dt, seed=200 + i) for i in range(45)]
    ys = api.aq_qmv_batched([c[0] for c in cases], [c[1] for c in cases], [c[2] for c in cases],
                            [c[3] for c in cases], bits, gs)
    torch.cuda.synchronize()
    for c, y in zip(cases, ys):
        _check(*c, y, bits, gs, dt)


def test_qmv_deterministic_and_workspace_left_zero():
    """Split-K partials meet in the workspace; the slices are added in slice
    order, so repeated calls agree bit for bit, and every call leaves the
    counters (the first 64 KB of the workspace) zero."""
    M, bits, gs, dt = 16, 4, 64, 1
    x, wq, s, b = _case(M, 2048, 8192, bits, gs, dt, seed=77, wstd=0.02)
    ws = api.Workspace()
    y1 = api.aq_qmv(x, wq, s, b, bits, gs, workspace=ws)
    y2 = api.aq_qmv(x, wq, s, b, bits, gs, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    buf = ws.get(x.device, 1)
    assert buf is not None and int(buf[:65536].count_nonzero()) == 0
    _check(x, wq, s, b, y2, bits, gs, dt)


def test_qmv_workspace_required():
    x, wq, s, b = _case(16, 2048, 8192, 4, 64, 1, seed=3)
    need = api.aq_workspace_size(api.AQ_OP_QMV, 16, 2048, 8192, 4, 64)
    assert need > 0
    y = torch.empty((16, 2048), dtype=torch.bfloat16, device=DEV)
    st = api.lib().aq_qmv(x.data_ptr(), wq.data_ptr(), s.data_ptr(), b.data_ptr(), y.data_ptr(),
                          16, 2048, 8192, 4, 64, 0, 1, None, 0, None)
    assert st == 5   # AQ_ERR_WORKSPACE


@pytest.mark.parametrize("M", [1, 5, 16])
def test_qmv_odd_shapes_fp32_kernel(M):
    """Shapes the tensor-core kernel cannot stream (scale rows that are not
    16-byte multiples, 3-bit rows of 8-byte multiples) run the fp32 kernel,
    for every M up to 16."""
    for (N, K, bits, gs) in [(40, 96, 4, 32), (33, 64 * 3, 3, 64), (17, 448, 5, 32)]:
        x, wq, s, b = _case(M, N, K, bits, gs, 0, seed=N + K + M)
        y = api.aq_qmv(x, wq, s, b, bits, gs)
        torch.cuda.synchronize()
        _check(x, wq, s, b, y, bits, gs, 0)
