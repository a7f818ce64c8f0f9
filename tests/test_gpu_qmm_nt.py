"""GPU parity: aq_qmm_nt, y = x . w_hat with the weight stored [N, K] as for
aq_qmv (the transpose = false product), against the oracle over the exact
w_hat: every width, both dtypes, FP4, one and many row splits, M over the
16-row chunk, and the down projection at full size."""
import pytest
import torch

import oracle
from group_wise_affine_quant_b200 import api, inputs
from group_wise_affine_quant_b200.inputs import gen, normal
from tests.gpu_util import DEV, dev_u16, dev_u8, to_dev
from tests.util import check_matmul

pytestmark = pytest.mark.gpu


def _check(x, wq, s, b, y, K, bits, gs, dt, mode=0):
    sc = dev_u8(s) if mode == 1 else dev_u16(s)
    yr, den = oracle.qmm_nt(dev_u16(x), dev_u8(wq), sc, None if b is None else dev_u16(b), K, bits,
                            gs, mode, dt)
    check_matmul(dev_u16(y), yr, den, dt)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 8])
@pytest.mark.parametrize("M,N", [(1, 640), (3, 48), (16, 640), (40, 200)])
def test_qmm_nt_affine(bits, M, N):
    dt = (M + bits) % 2
    gs = {2: 32, 3: 64, 4: 64, 5: 128, 6: 128, 8: 32}[bits]
    K = 1024 + 2 * gs
    g = gen(bits * 100 + M)
    wq, s, b = api.aq_quantize(to_dev(normal((N, K), 0.02, dt, g)), bits, gs)
    x = to_dev(normal((M, N), 1.0, dt, g))
    y = api.aq_qmm_nt(x, wq, s, b, bits, gs)
    torch.cuda.synchronize()
    assert api.lib().aq_device_errors() == 0
    _check(x, wq, s, b, y, K, bits, gs, dt)


@pytest.mark.parametrize("gs", [16, 32])
@pytest.mark.parametrize("M", [1, 7])
def test_qmm_nt_fp4(gs, M):
    N, K = 384, 2048
    codes, scales = inputs.fp4(N, K, gs, seed=gs + M)
    x = to_dev(normal((M, N), 1.0, 1, gen(M)))
    y = api.aq_qmm_nt(x, codes.to(DEV), scales.to(DEV), None, 4, gs)
    torch.cuda.synchronize()
    _check(x, codes.to(DEV), scales.to(DEV), None, y, K, 4, gs, 1, mode=1)


@pytest.mark.parametrize("M", [1, 16])
def test_qmm_nt_down_projection_full_size(M):
    """dy . W for the decode stack's down projection (W 2048 x 8192, bf16,
    4-bit g64): y [M, 8192] from x [M, 2048]."""
    g = gen(900 + M)
    wq, s, b = api.aq_quantize(to_dev(normal((2048, 8192), 0.02, 1, g)), 4, 64)
    x = to_dev(normal((M, 2048), 1.0, 1, g))
    y = api.aq_qmm_nt(x, wq, s, b, 4, 64)
    torch.cuda.synchronize()
    _check(x, wq, s, b, y, 8192, 4, 64, 1)


def test_qmm_nt_shares_workspace_and_is_deterministic():
    """Partials stay out of the counter area: aq_qmv calls on the same buffer
    stay correct, and repeated calls agree bit for bit."""
    ws = api.Workspace()
    g = gen(5)
    wq, s, b = api.aq_quantize(to_dev(normal((2048, 4096), 0.02, 1, g)), 4, 64)
    xn = to_dev(normal((4, 2048), 1.0, 1, g))
    xt = to_dev(normal((4, 4096), 1.0, 1, g))
    y1 = api.aq_qmm_nt(xn, wq, s, b, 4, 64, workspace=ws)
    y2 = api.aq_qmv(xt, wq, s, b, 4, 64, workspace=ws)
    y3 = api.aq_qmm_nt(xn, wq, s, b, 4, 64, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y3)
    assert int(ws.get(xn.device, 1)[:65536].count_nonzero()) == 0
    _check(xn, wq, s, b, y1, 4096, 4, 64, 1)
    yr, den = oracle.qmm(dev_u16(xt), dev_u8(wq), dev_u16(s), dev_u16(b), 2048, 4, 64, 0, 1)
    check_matmul(dev_u16(y2), yr, den, 1)
