"""Two host threads calling the library at the same time, each on its own
stream with its own workspace and its own per-thread settings (weight
prefetch on in one, off in the other): every result still matches the
oracle, and neither thread's setting leaks into the other's calls."""
import threading

import pytest
import torch

import oracle
from group_wise_affine_quant_b200 import api, inputs
from group_wise_affine_quant_b200._lib import lib
from tests.gpu_util import dev_u16, dev_u8, to_dev
from tests.util import check_matmul

pytestmark = pytest.mark.gpu


def _problem(seed, M, N, K):
    g = inputs.gen(seed)
    w = inputs.normal((N, K), 0.02, 1, g)
    x = to_dev(inputs.normal((M, K), 1.0, 1, g))
    wq, s, b = api.aq_quantize(to_dev(w), 4, 64)
    return x, wq, s, b


def test_two_threads_streams_and_settings():
    torch.cuda.synchronize()
    probs = {0: [_problem(300 + i, M, 2048, 2048) for i, M in enumerate((1, 16, 64))],
             1: [_problem(400 + i, M, 1024, 4096) for i, M in enumerate((4, 8, 128))]}
    torch.cuda.synchronize()
    outs, seen, errs = {0: [], 1: []}, {}, []

    def run(tid):
        try:
            lib().aq_set_weight_prefetch(1 if tid == 0 else 0)
            seen[tid] = lib().aq_get_weight_prefetch()
            ws = api.Workspace()
            st = torch.cuda.Stream()
            with torch.cuda.stream(st):
                for _ in range(20):
                    res = []
                    for x, wq, s, b in probs[tid]:
                        fn = api.aq_qmv if x.shape[0] <= 16 else api.aq_qmm
                        res.append(fn(x, wq, s, b, 4, 64, workspace=ws))
                st.synchronize()
            outs[tid] = res
        except Exception as e:          # reported by the main thread
            errs.append(e)

    th = [threading.Thread(target=run, args=(i,)) for i in (0, 1)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errs, errs
    assert seen == {0: 1, 1: 0}
    assert lib().aq_get_weight_prefetch() == 0          # the main thread's default
    torch.cuda.synchronize()
    assert lib().aq_device_errors() == 0
    for tid in (0, 1):
        for (x, wq, s, b), y in zip(probs[tid], outs[tid]):
            M, N = y.shape
            w_in_t = M > 16                             # aq_qmm rounds w_hat to T
            yr, den = oracle.qmm(dev_u16(x), dev_u8(wq), dev_u16(s), dev_u16(b), N, 4, 64, 0, 1,
                                 w_in_t=w_in_t)
            check_matmul(dev_u16(y), yr, den, 1, what="thread %d, M=%d" % (tid, M))
