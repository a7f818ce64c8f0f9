"""GPU parity: aq_gather_qmm against the oracle's gather_qmm, on the batched
decode path (M <= 16), the per-pair path (other shapes, M > 16), FP4
weights, repeated and permuted indices, and more pairs than one launch
holds."""
import numpy as np
import pytest
import torch

import oracle
from group_wise_affine_quant_b200 import api, inputs
from group_wise_affine_quant_b200.inputs import gen, normal
from tests.gpu_util import DEV, dev_u16, dev_u8, to_dev
from tests.util import check_matmul

pytestmark = pytest.mark.gpu


def _experts(E, N, K, bits, gs, dt, seed):
    qs = [api.aq_quantize(to_dev(normal((N, K), 0.02, dt, gen(seed + e))), bits, gs)
          for e in range(E)]
    return tuple(torch.stack([q[j] for q in qs]) for j in range(3))


def _check(x, wq, s, b, lhs, rhs, y, bits, gs, dt, mode=0):
    N = wq.shape[1]
    yr, den = oracle.gather_qmm(dev_u16(x), dev_u8(wq), dev_u8(s) if mode else dev_u16(s),
                                None if b is None else dev_u16(b), lhs, rhs, N, bits, gs, mode, dt)
    check_matmul(dev_u16(y), yr, den, dt)


@pytest.mark.parametrize("M", [1, 4, 16, 17, 64])
def test_gather_affine(M):
    dt, bits, gs = 1, 4, 64
    Bx, E, N, K = 3, 5, 512, 2048
    wq, s, b = _experts(E, N, K, bits, gs, dt, seed=10 * M)
    x = to_dev(normal((Bx, M, K), 1.0, dt, gen(M)))
    lhs = [2, 0, 1, 1, 0, 2, 2]
    rhs = [4, 4, 0, 3, 1, 2, 4]
    y = api.aq_gather_qmm(x, wq, s, b, lhs, rhs, bits, gs)
    torch.cuda.synchronize()
    assert api.lib().aq_device_errors() == 0
    _check(x, wq, s, b, lhs, rhs, y, bits, gs, dt)


@pytest.mark.parametrize("bits", [3, 8])
def test_gather_other_widths_and_identity(bits):
    """Other widths (the tcgen05 decode kernel's batch), identity indices."""
    dt, gs, M = 0, 64, 2
    E, N, K = 4, 256, 1024
    wq, s, b = _experts(E, N, K, bits, gs, dt, seed=bits)
    x = to_dev(normal((E, M, K), 1.0, dt, gen(bits)))
    y = api.aq_gather_qmm(x, wq, s, b, None, None, bits, gs)
    torch.cuda.synchronize()
    _check(x, wq, s, b, list(range(E)), list(range(E)), y, bits, gs, dt)


def test_gather_per_pair_fallback_shape():
    """Scale rows that are not 16-byte multiples (K = 96 at group 32): no
    batch, one call per pair."""
    dt, bits, gs, M = 1, 4, 32, 3
    E, N, K = 3, 40, 96
    wq, s, b = _experts(E, N, K, bits, gs, dt, seed=5)
    x = to_dev(normal((2, M, K), 1.0, dt, gen(5)))
    lhs, rhs = [1, 0, 1], [2, 2, 0]
    y = api.aq_gather_qmm(x, wq, s, b, lhs, rhs, bits, gs)
    torch.cuda.synchronize()
    _check(x, wq, s, b, lhs, rhs, y, bits, gs, dt)


def test_gather_fp4_experts():
    gs, M = 32, 1
    E, N, K = 6, 256, 1024
    cs, ss = zip(*[inputs.fp4(N, K, gs, seed=50 + e) for e in range(E)])
    wq, s = torch.stack(cs).to(DEV), torch.stack(ss).to(DEV)
    x = to_dev(inputs.fp4_x(2 * M, K).reshape(2, M, K))
    lhs, rhs = [0, 1, 1, 0], [5, 0, 3, 5]
    y = api.aq_gather_qmm(x, wq, s, None, lhs, rhs, 4, gs)
    torch.cuda.synchronize()
    _check(x, wq, s, None, lhs, rhs, y, 4, gs, 1, mode=1)


def test_gather_moe_decode_many_pairs():
    """A decode step of a mixture-of-experts layer: 8 experts of 1408 x 2048,
    48 token rows each routed to 2 experts (96 pairs > 40 per launch)."""
    dt, bits, gs, M = 1, 4, 64, 1
    E, N, K, T = 8, 1408, 2048, 48
    wq, s, b = _experts(E, N, K, bits, gs, dt, seed=700)
    x = to_dev(normal((T, M, K), 1.0, dt, gen(701)))
    rng = np.random.default_rng(3)
    lhs = [t for t in range(T) for _ in range(2)]
    rhs = [int(e) for t in range(T) for e in rng.choice(E, 2, replace=False)]
    y = api.aq_gather_qmm(x, wq, s, b, lhs, rhs, bits, gs)
    torch.cuda.synchronize()
    assert api.lib().aq_device_errors() == 0
    _check(x, wq, s, b, lhs, rhs, y, bits, gs, dt)


@pytest.mark.parametrize("M", [1, 2, 5])
def test_gather_grouped_by_expert(M):
    """Pairs that share an expert run as one problem (x rows gathered, y rows
    scattered back): one expert with more pairs than a problem holds (split
    into several groups, the last padded with zero rows), a permuted x order,
    and the counter area of the workspace left zero."""
    dt, bits, gs = 1, 4, 64
    Bx, E, N, K = 6, 3, 384, 1024
    wq, s, b = _experts(E, N, K, bits, gs, dt, seed=300 + M)
    x = to_dev(normal((Bx, M, K), 1.0, dt, gen(400 + M)))
    rng = np.random.default_rng(M)
    rhs = [0] * 20 + [2] * 3 + [1]
    lhs = [int(v) for v in rng.integers(0, Bx, len(rhs))]
    ws = api.Workspace()
    y = api.aq_gather_qmm(x, wq, s, b, lhs, rhs, bits, gs, workspace=ws)
    torch.cuda.synchronize()
    assert api.lib().aq_device_errors() == 0
    assert int(ws.get(x.device, 1)[:65536].count_nonzero()) == 0
    _check(x, wq, s, b, lhs, rhs, y, bits, gs, dt)
