"""GPU parity for aq_qmm (tcgen05 tensor-core path) against the oracle, within
|y - y_ref| <= 2e-3 * sum_k |x_k w_hat_k| + 1 ulp_T(y_ref).

The kernel dequantizes each weight tile into T (the values aq_dequantize
writes, as the pages' kernels do) before the tensor-core product, so y_ref is
the oracle's fp64 product with w_hat rounded once to T (w_in_t)."""
import numpy as np
import pytest
import torch

import oracle
from group_wise_affine_quant_b200 import api, inputs
from tests.gpu_util import DEV, dev_u16, dev_u8, to_dev
from tests.util import check_matmul

pytestmark = pytest.mark.gpu

BITS = (2, 3, 4, 5, 6, 8)


def _case(M, N, K, bits, gs, dt, seed, wstd=0.05, xstd=1.0):
    g = inputs.gen(seed)
    w = inputs.normal((N, K), wstd, dt, g)
    x = inputs.normal((M, K), xstd, dt, g)
    wq, s, b = api.aq_quantize(to_dev(w), bits, gs)
    return to_dev(x), wq, s, b


def _check(x, wq, s, b, y, bits, gs, dt, mode=0, w_in_t=True, **kw):
    N = wq.shape[0]
    sc = dev_u8(s) if mode == 1 else dev_u16(s)
    bi = None if b is None else dev_u16(b)
    yr, den = oracle.qmm(dev_u16(x), dev_u8(wq), sc, bi, N, bits, gs, mode, dt, w_in_t=w_in_t)
    return check_matmul(dev_u16(y), yr, den, dt, **kw)


def _check_sampled(x, wq, s, b, y, bits, gs, dt, n_samples=512, seed=0, mode=0, w_in_t=True,
                   **kw):
    M, N = y.shape
    rng = np.random.default_rng(seed)
    ms = np.concatenate([[0, M - 1, M - 1, 0], rng.integers(0, M, n_samples)])
    ns = np.concatenate([[0, N - 1, 0, N - 1], rng.integers(0, N, n_samples)])
    sc = dev_u8(s) if mode == 1 else dev_u16(s)
    bi = None if b is None else dev_u16(b)
    yr, den = oracle.qmm_sampled(dev_u16(x), dev_u8(wq), sc, bi, N, bits, gs, mode, dt, ms, ns,
                                 w_in_t=w_in_t)
    ys = dev_u16(y)[ms, ns]
    return check_matmul(ys, yr, den, dt, **kw)


def test_qmm_smallest():
    """One 128 x 16 tile, one K-step."""
    x, wq, s, b = _case(16, 128, 64, 4, 64, 0, seed=1)
    y = api.aq_qmm(x, wq, s, b, 4, 64)
    torch.cuda.synchronize()
    assert api.aq_last_error() == ""
    _check(x, wq, s, b, y, 4, 64, 0)
    assert api.lib().aq_device_errors() == 0


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("dt", [0, 1])
def test_qmm_all_widths(bits, dt):
    """Several weight tiles, ragged N and M, K with a 32-element tail."""
    gs = 32
    x, wq, s, b = _case(37, 200, 64 * 5 + 32, bits, gs, dt, seed=bits + 10 * dt)
    y = api.aq_qmm(x, wq, s, b, bits, gs)
    torch.cuda.synchronize()
    _check(x, wq, s, b, y, bits, gs, dt)


@pytest.mark.parametrize("M", [1, 2, 15, 16, 17, 32, 33, 64, 65, 127, 128, 129, 255, 256, 300])
def test_qmm_m_sweep(M):
    """Every token-tile size and its edges (16/32/64/128/256 rows of x)."""
    dt = M % 2
    x, wq, s, b = _case(M, 256, 512, 4, 64, dt, seed=M)
    y = api.aq_qmm(x, wq, s, b, 4, 64)
    torch.cuda.synchronize()
    _check(x, wq, s, b, y, 4, 64, dt)


@pytest.mark.parametrize("gs", [32, 64, 128])
@pytest.mark.parametrize("bits", [3, 4, 8])
def test_qmm_groups(gs, bits):
    x, wq, s, b = _case(48, 384, 1024, bits, gs, 1, seed=gs + bits)
    y = api.aq_qmm(x, wq, s, b, bits, gs)
    torch.cuda.synchronize()
    _check(x, wq, s, b, y, bits, gs, 1)


@pytest.mark.parametrize("M,N,K", [(16, 128, 8192), (1, 256, 4096), (64, 384, 2048 + 32)])
def test_qmm_split_k_cluster(M, N, K):
    """Few output tiles: K splits over a cluster and reduces through DSMEM."""
    x, wq, s, b = _case(M, N, K, 4, 32, 0, seed=K, wstd=0.02)
    y1 = api.aq_qmm(x, wq, s, b, 4, 32)
    y2 = api.aq_qmm(x, wq, s, b, 4, 32)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    _check(x, wq, s, b, y1, 4, 32, 0)


@pytest.mark.parametrize("M,N,K,bits", [
    (1024, 5120, 1024, 4),       # 160 tiles of 256 x 128: last 12 tiles in 4 K-slices
    (1024, 5120, 1088, 3),       # odd width, 17 k-tiles: slices of an even k-tile count
    (16, 44288, 1024, 4),        # light tiles, 346 of them: last 50 in 2 K-slices
])
def test_qmm_split_last_wave(M, N, K, bits):
    """More tiles than resident CTAs with a last wave at most half full: the
    remaining tiles launch apart with K split over a cluster."""
    x, wq, s, b = _case(M, N, K, bits, 64, 1, seed=N + K + bits, wstd=0.02)
    y1 = api.aq_qmm(x, wq, s, b, bits, 64)
    y2 = api.aq_qmm(x, wq, s, b, bits, 64)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    rng = np.random.default_rng(bits)
    tail_rows = np.arange(N - 128 * 13, N)          # columns of the tail tiles
    ms = np.concatenate([[0, M - 1], rng.integers(0, M, 800), rng.integers(max(0, M - 256), M, 400)])
    ns = np.concatenate([[0, N - 1], rng.integers(0, N, 800), rng.choice(tail_rows, 400)])
    yr, den = oracle.qmm_sampled(dev_u16(x), dev_u8(wq), dev_u16(s), dev_u16(b), N, bits, 64, 0,
                                 1, ms, ns, w_in_t=True)
    check_matmul(dev_u16(y1)[ms, ns], yr, den, 1)


@pytest.mark.parametrize("bits", [2, 3, 5, 6])
def test_qmm_narrow_rows(bits):
    """K % 64 == 32: row strides that are not 16-byte multiples."""
    x, wq, s, b = _case(20, 130, 32 * 9, bits, 32, 1, seed=bits)
    y = api.aq_qmm(x, wq, s, b, bits, 32)
    torch.cuda.synchronize()
    _check(x, wq, s, b, y, bits, 32, 1)


@pytest.mark.parametrize("gs", [16, 32])
@pytest.mark.parametrize("M", [1, 16, 100, 256])
@pytest.mark.parametrize("dt", [0, 1])
def test_qmm_fp4(gs, M, dt):
    N, K = 256, 1024 + (16 if gs == 16 else 32) * 2
    codes, scales = inputs.fp4(N, K, gs, seed=gs + M)
    x = inputs.normal((M, K), 1.0, dt, inputs.gen(M))
    xd, wq, sc = to_dev(x), codes.to(DEV), scales.to(DEV)
    y = api.aq_qmm(xd, wq, sc, None, 4, gs)
    torch.cuda.synchronize()
    _check(xd, wq, sc, None, y, 4, gs, dt, mode=1)


@pytest.mark.parametrize("M", [32, 64])
@pytest.mark.parametrize("name,N,K", inputs.LLAMA_1B_PROJ)
def test_qmm_decode_projection(M, name, N, K):
    """Decode sweep rows M = 32, 64 at full projection size (bf16 4-bit g64)."""
    x, wq, s, b = _case(M, N, K, 4, 64, 1, seed=N + K + M, wstd=0.02)
    y = api.aq_qmm(x, wq, s, b, 4, 64)
    torch.cuda.synchronize()
    _check(x, wq, s, b, y, 4, 64, 1)


@pytest.mark.parametrize("bits", [2, 3, 4, 6, 8])
def test_qmm_chained_first_products(bits):
    """Chained workload, fp16 g64: x[1024,1024] . W1^T (W1 4096x1024) then
    . W2^T (W2 1024x4096), each checked on sampled outputs against the oracle
    fed with the device's own input to that product."""
    x, w1, w2 = inputs.chained()
    q1 = api.aq_quantize(to_dev(w1), bits, 64)
    q2 = api.aq_quantize(to_dev(w2), bits, 64)
    xd = to_dev(x)
    h = api.aq_qmm(xd, *q1, bits, 64)
    o = api.aq_qmm(h, *q2, bits, 64)
    torch.cuda.synchronize()
    _check_sampled(xd, *q1, h, bits, 64, 0, seed=bits)
    fin = torch.isfinite(h).all().item()
    if fin:
        _check_sampled(h, *q2, o, bits, 64, 0, seed=bits + 1)


@pytest.mark.parametrize("gs,scale_range", [(32, "finite"), (16, "finite"), (32, "literal")])
@pytest.mark.parametrize("M", [256, 4096])
def test_qmm_fp4_full_size(gs, scale_range, M):
    """FP4 workload, bf16, K = N = 4096, sampled outputs."""
    codes, scales = inputs.fp4(4096, 4096, gs, scale_range=scale_range, seed=7)
    x = inputs.fp4_x(M, 4096)
    xd, wq, sc = to_dev(x), codes.to(DEV), scales.to(DEV)
    y = api.aq_qmm(xd, wq, sc, None, 4, gs)
    torch.cuda.synchronize()
    _check_sampled(xd, wq, sc, None, y, 4, gs, 1, mode=1,
                   overflow_any_nonfinite=(scale_range == "literal"))


@pytest.mark.parametrize("bits", [4, 8])
def test_qmm_chained_meets_bound_over_exact_w(bits):
    """The literal tolerance over the EXACT w_hat (not w_hat rounded to T) at
    the chained workload's size (fp16, K = 1024): the tensor-core product of
    the T-rounded tile stays within 2e-3 * sum |x w_hat| + 1 ulp."""
    x, w1, _ = inputs.chained()
    q1 = api.aq_quantize(to_dev(w1), bits, 64)
    xd = to_dev(x)
    h = api.aq_qmm(xd, *q1, bits, 64)
    torch.cuda.synchronize()
    _check_sampled(xd, *q1, h, bits, 64, 0, seed=40 + bits, w_in_t=False)


@pytest.mark.parametrize("M", [32, 64])
def test_qmm_decode_projection_meets_bound_over_exact_w(M):
    """The same at the decode sweep's gate projection through aq_qmm (bf16,
    8192 x 2048, the coarser T)."""
    g = inputs.gen(60 + M)
    w = inputs.normal((8192, 2048), 0.02, 1, g)
    x = to_dev(inputs.normal((M, 2048), 1.0, 1, g))
    wq, s, b = api.aq_quantize(to_dev(w), 4, 64)
    y = api.aq_qmm(x, wq, s, b, 4, 64)
    torch.cuda.synchronize()
    _check_sampled(x, wq, s, b, y, 4, 64, 1, seed=M, w_in_t=False)


def test_qmm_matches_qmv_small_m():
    """For M <= 16 both paths agree within twice the bound."""
    x, wq, s, b = _case(8, 512, 2048, 4, 64, 1, seed=3)
    y1 = api.aq_qmm(x, wq, s, b, 4, 64)
    y2 = api.aq_qmv(x, wq, s, b, 4, 64)
    torch.cuda.synchronize()
    _check(x, wq, s, b, y1, 4, 64, 1)
    _check(x, wq, s, b, y2, 4, 64, 1)


@pytest.mark.parametrize("prefetch", [False, True])
def test_dependent_chain_under_pdl(prefetch):
    """Back-to-back dependent calls on one stream (each kernel may start
    before the previous one ends): y feeds the next call's x and is
    overwritten by a later call.  Results equal the same calls separated by
    device synchronisation."""
    bits, gs = 4, 64
    g = inputs.gen(21)
    ws = [api.aq_quantize(to_dev(inputs.normal((512, 512), 0.05, 1, g)), bits, gs) for _ in range(4)]
    x = to_dev(inputs.normal((8, 512), 1.0, 1, g))
    torch.cuda.synchronize()
    ref = []
    cur = x
    for i in range(6):
        fn = api.aq_qmv if i % 2 else api.aq_qmm
        cur = fn(cur, *ws[i % 4], bits, gs)
        torch.cuda.synchronize()
        ref.append(cur.clone())
    old = api.aq_get_weight_prefetch()
    api.aq_set_weight_prefetch(prefetch)
    try:
        a = torch.empty_like(x)
        b = torch.empty_like(x)
        a.copy_(x)
        outs = []
        for i in range(6):
            fn = api.aq_qmv if i % 2 else api.aq_qmm
            dst = b if i % 2 == 0 else a
            src = a if i % 2 == 0 else b
            fn(src, *ws[i % 4], bits, gs, out=dst)
            outs.append(dst)
            if i in (1, 3, 5):
                outs[-1] = dst.clone()
        torch.cuda.synchronize()
    finally:
        api.aq_set_weight_prefetch(old)
    for i in (1, 3, 5):
        assert torch.equal(outs[i], ref[i]), i


def test_independent_calls_under_input_prefetch():
    """Calls whose x were all written before the first launch, each into its
    own y, with weight and input prefetch on (each kernel may read its
    weights and x while the previous one runs): results equal the same calls
    separated by device synchronisation."""
    bits, gs = 4, 64
    g = inputs.gen(33)
    ws = [api.aq_quantize(to_dev(inputs.normal((n, 1024), 0.05, 1, g)), bits, gs)
          for n in (512, 128, 2048, 384)]
    xs = [to_dev(inputs.normal((m, 1024), 1.0, 1, g)) for m in (1, 4, 16, 40)]
    torch.cuda.synchronize()
    calls = [(api.aq_qmv if x.shape[0] <= 16 else api.aq_qmm, x, w) for x in xs for w in ws]
    ref = []
    for fn, x, w in calls:
        ref.append(fn(x, *w, bits, gs))
        torch.cuda.synchronize()
    old_w, old_x = api.aq_get_weight_prefetch(), api.aq_get_input_prefetch()
    api.aq_set_weight_prefetch(True)
    api.aq_set_input_prefetch(True)
    try:
        outs = [fn(x, *w, bits, gs) for fn, x, w in calls]
        torch.cuda.synchronize()
    finally:
        api.aq_set_weight_prefetch(old_w)
        api.aq_set_input_prefetch(old_x)
    for i, (a, b) in enumerate(zip(outs, ref)):
        assert torch.equal(a, b), i
    assert api.lib().aq_device_errors() == 0


def test_quantize_then_matmul_default_order():
    """Weights written by the kernel just before (prefetch off by default)."""
    assert not api.aq_get_weight_prefetch()
    w = to_dev(inputs.normal((256, 1024), 0.05, 1, inputs.gen(5)))
    x = to_dev(inputs.normal((4, 1024), 1.0, 1, inputs.gen(6)))
    q = api.aq_quantize(w, 4, 64)
    y = api.aq_qmm(x, *q, 4, 64)
    torch.cuda.synchronize()
    _check(x, *q, y, 4, 64, 1)


def test_qmm_empty():
    x = torch.zeros((0, 64), dtype=torch.float16, device=DEV)
    wq = torch.zeros((128, 32), dtype=torch.uint8, device=DEV)
    s = torch.zeros((128, 1), dtype=torch.float16, device=DEV)
    y = api.aq_qmm(x, wq, s, s, 4, 64)
    assert y.shape == (0, 128)
