"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every symbol the header declares, and rejects bad arguments before it touches
the device.  Pointers here are fake addresses that validation must refuse
without dereferencing."""
import ctypes

import pytest

from group_wise_affine_quant_b200 import _lib

OK, INVALID, UNSUPPORTED, MISALIGNED, CUDA, WORKSPACE = range(6)
A = 0x10000  # a 16- and 256-byte aligned fake device address


def L():
    return _lib.lib()


def test_exports_every_declared_symbol():
    names = _lib.declared_symbols()
    assert set(names) == set(_lib.SIGNATURES), names
    for n in names:
        assert hasattr(L(), n), n
    assert L().aq_version() >= 100


def _qmv(**kw):
    a = dict(x=A, w_q=A, s=A, b=A, y=A, M=1, N=64, K=128, bits=4, gs=64, mode=0, dt=0,
             ws=A, wsb=1 << 30)
    a.update(kw)
    return L().aq_qmv(a["x"], a["w_q"], a["s"], a["b"], a["y"], a["M"], a["N"], a["K"], a["bits"],
                      a["gs"], a["mode"], a["dt"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("bits", [0, 1, 7, 9, 16])
def test_unsupported_bits(bits):
    assert _qmv(bits=bits) == UNSUPPORTED
    assert b"bits" in L().aq_last_error()


@pytest.mark.parametrize("gs", [0, 8, 16, 48, 256])
def test_unsupported_group_affine(gs):
    assert _qmv(gs=gs) == UNSUPPORTED


def test_fp4_rules():
    assert _qmv(mode=1, gs=64, b=None) == UNSUPPORTED
    assert _qmv(mode=1, bits=8, gs=32, b=None) == UNSUPPORTED
    assert _qmv(mode=1, gs=32, b=A) == INVALID        # FP4 takes no biases
    assert _qmv(mode=2) == UNSUPPORTED


def test_dtype_and_shape_errors():
    assert _qmv(dt=2) == UNSUPPORTED
    assert _qmv(K=96) == INVALID                       # not a multiple of 64
    assert _qmv(M=0) == INVALID and _qmv(M=17) == INVALID
    assert _qmv(N=-1) == INVALID
    assert _qmv(b=None) == INVALID                     # affine needs biases
    assert _qmv(x=None) == INVALID and _qmv(y=None) == INVALID


def test_alignment_errors():
    assert _qmv(x=A + 2) == MISALIGNED
    assert _qmv(y=A + 8) == MISALIGNED
    assert _qmv(w_q=A + 4) == MISALIGNED
    assert _qmv(s=A + 1) == MISALIGNED


def test_qmv_workspace_sizes():
    """The tensor-core qmv splits K through the workspace when a row tile's
    K is long enough to split; shapes it does not take need none."""
    ws = lambda M, N, K, bits=4, gs=64, mode=0: L().aq_workspace_size(0, M, N, K, bits, gs, mode, 1)
    assert ws(16, 2048, 8192) > 0                     # 16 row tiles, K split over slices
    assert ws(1, 2048, 8192) < ws(16, 2048, 8192)     # partials scale with M
    assert ws(1, 64, 0) == 0
    assert ws(1, 4096, 64) == 0                       # one 64-column stage: no split
    assert ws(4, 40, 96, 4, 32) == 0                  # scale rows of 6 bytes: fp32 kernel
    assert ws(17, 2048, 8192) == 0                    # not a qmv size
    # a too-small workspace is refused before anything is launched
    assert _qmv(M=16, N=2048, K=8192, ws=None, wsb=0) == WORKSPACE
    assert _qmv(M=16, N=2048, K=8192, ws=A, wsb=16) == WORKSPACE
    assert _qmv(M=16, N=2048, K=8192, ws=A + 16, wsb=1 << 30) == MISALIGNED


def _problems(n, **kw):
    arr = (_lib.QmvProblem * n)()
    for i in range(n):
        f = dict(x=A, w_q=A, scales=A, biases=A, y=A, N=256, K=2048)
        f.update(kw)
        arr[i] = _lib.QmvProblem(f["x"], f["w_q"], f["scales"], f["biases"], f["y"], f["N"], f["K"])
    return arr


def test_qmv_batched_validation():
    b = L().aq_qmv_batched
    assert b(None, 0, 1, 4, 64, 0, 1, None, 0, None) == OK               # nothing to do
    assert b(None, 2, 1, 4, 64, 0, 1, None, 0, None) == INVALID
    assert b(_problems(2), 2, 0, 4, 64, 0, 1, A, 1 << 30, None) == INVALID   # M = 0
    assert b(_problems(2), 2, 17, 4, 64, 0, 1, A, 1 << 30, None) == INVALID
    assert b(_problems(2), 2, 1, 7, 64, 0, 1, A, 1 << 30, None) == UNSUPPORTED
    assert b(_problems(2, y=A + 2), 2, 1, 4, 64, 0, 1, A, 1 << 30, None) == MISALIGNED
    assert b"problem 0" in L().aq_last_error()
    assert b(_problems(2, K=96), 2, 1, 4, 32, 0, 1, A, 1 << 30, None) == UNSUPPORTED
    assert b(_problems(2, N=0), 2, 1, 4, 64, 0, 1, A, 1 << 30, None) == INVALID
    assert b(_problems(1, scales=A + 2), 1, 1, 4, 64, 0, 1, A, 1 << 30, None) == UNSUPPORTED
    # workspace: sized for the batch, refused when missing
    p = _problems(3, N=2048, K=8192)
    need = L().aq_qmv_batched_workspace_size(p, 3, 16, 4, 64, 0)
    assert need > 0
    assert b(p, 3, 16, 4, 64, 0, 1, None, 0, None) == WORKSPACE
    # K = 2048: one K-slice per row tile, so only the 64 KB counter area (the
    # unit scheduler's counters) and no partial sums
    assert L().aq_qmv_batched_workspace_size(_problems(3), 3, 16, 4, 64, 0) == 65536


def test_prefetch_settings_are_per_thread():
    """aq_set_weight_prefetch / aq_set_input_prefetch change only the calling
    thread's later calls: another thread still sees the default."""
    import threading
    seen = {}

    def other():
        seen["w"] = L().aq_get_weight_prefetch()
        seen["x"] = L().aq_get_input_prefetch()
        L().aq_set_input_prefetch(1)
        seen["x_after"] = L().aq_get_input_prefetch()

    L().aq_set_weight_prefetch(1)
    L().aq_set_input_prefetch(0)
    try:
        t = threading.Thread(target=other)
        t.start()
        t.join()
        assert seen == {"w": 0, "x": 0, "x_after": 1}
        assert L().aq_get_weight_prefetch() == 1
        assert L().aq_get_input_prefetch() == 0       # the other thread's setting stayed there
    finally:
        L().aq_set_weight_prefetch(0)


def test_quantize_validation():
    q = L().aq_quantize
    assert q(A, A, A, A, 4, 64, 7, 64, 0, None) == UNSUPPORTED
    assert q(A, A, A, A, 4, 96, 4, 64, 0, None) == INVALID
    assert q(A + 2, A, A, A, 4, 64, 4, 64, 0, None) == MISALIGNED
    assert q(None, A, A, A, 4, 64, 4, 64, 0, None) == INVALID
    assert q(A, A, A, A, 0, 64, 4, 64, 0, None) == OK          # empty: nothing to do


def test_dequantize_validation():
    d = L().aq_dequantize
    assert d(A, A, A, A + 8, 4, 64, 4, 64, 0, 0, None) == MISALIGNED
    assert d(A, A, None, A, 4, 64, 4, 64, 0, 0, None) == INVALID
    assert d(A, A, A, A, 4, 64, 4, 16, 0, 0, None) == UNSUPPORTED


def test_error_message_is_thread_local_and_cleared():
    assert _qmv(bits=7) == UNSUPPORTED
    assert L().aq_last_error() != b""
    assert L().aq_quantize(A, A, A, A, 0, 64, 4, 64, 0, None) == OK
    assert L().aq_last_error() == b""


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        _lib.lib()


def test_quantize_fp4_validation():
    q = L().aq_quantize_fp4
    assert q(A, A, A, 4, 64, 64, 1, None) == UNSUPPORTED        # scales are for 16 or 32
    assert q(A, A, A, 4, 64, 32, 2, None) == UNSUPPORTED        # fp16 / bf16 only
    assert q(A, A, A, 4, 48, 16, 1, None) == INVALID            # K a multiple of 32
    assert q(A + 1, A, A, 4, 64, 32, 1, None) == MISALIGNED
    assert q(None, A, A, 4, 64, 32, 1, None) == INVALID
    assert q(None, None, None, 0, 64, 32, 1, None) == OK        # empty: nothing to do


def test_quantize_dequantize_fp_validation():
    f = L().aq_quantize_dequantize_fp
    assert f(A, A, 4, 64, 6, 32, 1, None) == UNSUPPORTED         # bits 4 or 8
    assert f(A, A, 4, 64, 4, 64, 1, None) == UNSUPPORTED         # group 16 or 32
    assert f(A, A, 4, 64, 8, 16, 2, None) == UNSUPPORTED
    assert f(A, A, 4, 40, 4, 16, 1, None) == INVALID
    assert f(A, A + 1, 4, 64, 4, 32, 1, None) == MISALIGNED
    assert f(None, None, 0, 64, 4, 32, 1, None) == OK


def test_qqmm_validation_and_workspace():
    q = L().aq_qqmm
    need = L().aq_workspace_size(3, 4, 256, 1024, 4, 32, 1, 1)
    assert need >= 4 * 1024 * 2 and need % 2 == 0
    # the qmv workspace comes first, 256-byte aligned, then x, never inside
    # the first 64 KB (the counters every call leaves zero)
    qmv = L().aq_workspace_size(0, 4, 256, 1024, 4, 32, 1, 1)
    assert need == max(65536, ((qmv + 255) // 256) * 256) + 4 * 1024 * 2
    big = L().aq_workspace_size(0, 16, 4096, 65536, 4, 32, 1, 1)
    assert big > 65536
    assert (L().aq_workspace_size(3, 16, 4096, 65536, 4, 32, 1, 1) ==
            ((big + 255) // 256) * 256 + 16 * 65536 * 2)
    assert L().aq_workspace_size(3, 64, 256, 1024, 4, 32, 1, 1) == 65536 + 64 * 1024 * 2
    assert q(A, A, A, A, 4, 256, 1024, 64, 1, A, 1 << 30, None) == UNSUPPORTED  # FP4 group
    assert q(A, A, A, A, 4, 256, 1024, 32, 1, None, 0, None) == WORKSPACE
    assert q(A, A, A, A, 4, 256, 1024, 32, 1, A + 16, 1 << 30, None) == MISALIGNED
    assert q(A + 2, A, A, A, 4, 256, 1024, 32, 1, A, 1 << 30, None) == MISALIGNED
    assert q(A, A, A, A, 0, 256, 1024, 32, 1, None, 0, None) == OK             # M = 0


def test_gather_qmm_validation():
    g = L().aq_gather_qmm
    I32 = ctypes.c_int32 * 3

    def call(lhs=None, rhs=None, n=3, M=1, xb=3, wb=3, **kw):
        a = dict(x=A, w=A, s=A, b=A, y=A, N=256, K=2048, bits=4, gs=64, mode=0, dt=1, ws=A,
                 wsb=1 << 30)
        a.update(kw)
        return g(a["x"], a["w"], a["s"], a["b"], lhs, rhs, a["y"], n, M, a["N"], a["K"], xb, wb,
                 a["bits"], a["gs"], a["mode"], a["dt"], a["ws"], a["wsb"], None)
    assert call(n=0) == OK
    assert call(lhs=I32(0, 1, 3)) == INVALID                      # x batch 3 out of range
    assert b"pair 2" in L().aq_last_error()
    assert call(rhs=I32(0, -1, 1)) == INVALID
    assert call(n=4) == INVALID                                   # identity needs 4 batches
    assert call(xb=0) == INVALID
    assert call(bits=7) == UNSUPPORTED
    assert call(b=None) == INVALID                                # affine needs biases
    ws = L().aq_gather_qmm_workspace_size
    assert ws(3, 16, 2048, 8192, 4, 64, 0) > 0
    assert ws(3, 17, 2048, 8192, 4, 64, 0) == 0                   # qmm pairs need none
    assert ws(0, 1, 2048, 8192, 4, 64, 0) == 0


def test_qmm_nt_validation_and_workspace():
    f = L().aq_qmm_nt

    def call(**kw):
        a = dict(x=A, w=A, s=A, b=A, y=A, M=1, N=640, K=1024, bits=4, gs=64, mode=0, dt=1, ws=A,
                 wsb=1 << 30)
        a.update(kw)
        return f(a["x"], a["w"], a["s"], a["b"], a["y"], a["M"], a["N"], a["K"], a["bits"], a["gs"],
                 a["mode"], a["dt"], a["ws"], a["wsb"], None)
    assert call(bits=7) == UNSUPPORTED
    assert call(K=96, gs=64) == INVALID
    assert call(y=A + 8) == MISALIGNED
    assert call(x=A + 1) == MISALIGNED
    assert call(M=0) == OK
    need = L().aq_workspace_size(4, 1, 640, 1024, 4, 64, 0, 1)
    assert need > 65536                                       # partials after the counters
    assert call(M=1, ws=None, wsb=0) == WORKSPACE
    assert L().aq_workspace_size(4, 16, 640, 1024, 4, 64, 0, 1) > need   # partials grow with M
    assert L().aq_workspace_size(4, 1, 32, 1024, 4, 64, 0, 1) == 0   # one split: no partials
