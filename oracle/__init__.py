"""CPU oracle for group-wise affine quantized matmul — TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``aq_oracle.cpp`` (plain C++,
fp32 quantizer, fp64 dequant and accumulation) through ctypes and numpy, and it
shares nothing with the CUDA library.

T values (fp16 / bf16) travel as their raw 16-bit patterns in uint16 arrays.
dtype codes: 0 = fp16, 1 = bf16.  mode codes: 0 = affine, 1 = FP4 (E2M1 codes
with E8M0 scales at group 32 or FP8 E4M3 scales at group 16).
"""
import ctypes
import os

import numpy as np

from .build_oracle import build as _build

F16, BF16 = 0, 1
AFFINE, FP4, MXFP8 = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        _lib.orc_num_threads.restype = I
        _lib.orc_set_num_threads.argtypes = [I]
        _lib.orc_set_num_threads.restype = None
        _lib.orc_t_to_double.argtypes = [ctypes.c_uint16, I]
        _lib.orc_t_to_double.restype = ctypes.c_double
        _lib.orc_round_to_t.argtypes = [ctypes.c_double, I]
        _lib.orc_round_to_t.restype = ctypes.c_uint16
        for name in ("orc_e2m1", "orc_e8m0", "orc_e4m3"):
            getattr(_lib, name).argtypes = [I]
            getattr(_lib, name).restype = ctypes.c_double
        for name in ("orc_e8m0_encode", "orc_e4m3_encode", "orc_e2m1_encode"):
            getattr(_lib, name).argtypes = [ctypes.c_float]
            getattr(_lib, name).restype = I
        _lib.orc_quantize_fp4.argtypes = [P, I64, I64, I, I, P, P]
        _lib.orc_quantize_fp4.restype = I
        _lib.orc_quantize_mxfp8.argtypes = [P, I64, I64, I, P, P]
        _lib.orc_quantize_mxfp8.restype = I
        _lib.orc_quantize_dequantize_fp.argtypes = [P, I64, I64, I, I, I, P]
        _lib.orc_quantize_dequantize_fp.restype = I
        _lib.orc_quantize.argtypes = [P, I64, I64, I, I, I, P, P, P]
        _lib.orc_unpack.argtypes = [P, I64, I64, I, P]
        _lib.orc_dequantize.argtypes = [P, P, P, I64, I64, I, I, I, I, P, P]
        _lib.orc_qmm.argtypes = [P, P, P, P, I64, I64, I64, I, I, I, I, I, P, P]
        _lib.orc_qmm_sampled.argtypes = [P, P, P, P, I64, I64, I64, I, I, I, I, I,
                                         P, P, I64, P, P]
        _lib.orc_qconv2d_nhwc.argtypes = [P, P, P, P] + [I] * 16 + [P, P, I64, P, P]
        for name in ("orc_quantize", "orc_unpack", "orc_dequantize", "orc_qmm",
                     "orc_qmm_sampled", "orc_qconv2d_nhwc"):
            getattr(_lib, name).restype = I
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s rejected its arguments" % what)


def num_threads() -> int:
    return lib().orc_num_threads()


def set_num_threads(n: int) -> None:
    """Threads of the oracle's parallel loops (results do not depend on it)."""
    lib().orc_set_num_threads(int(n))


def t_to_double(bits16, dt):
    return lib().orc_t_to_double(int(bits16), dt)


def round_to_t(v, dt):
    return lib().orc_round_to_t(float(v), dt)


def e2m1(code):
    return lib().orc_e2m1(int(code))


def e8m0(s):
    return lib().orc_e8m0(int(s))


def e4m3(s):
    return lib().orc_e4m3(int(s))


def row_bytes(K, bits):
    return K * bits // 8


def quantize(w16, bits, gs, dt):
    """w16: [N, K] uint16 T patterns -> (w_q [N, K*bits/8] u8, scales, biases [N, K/gs] u16)."""
    w16 = _c(w16, np.uint16)
    N, K = w16.shape
    wq = np.zeros((N, row_bytes(K, bits)), np.uint8)
    G = K // gs if gs else 0
    s = np.zeros((N, G), np.uint16)
    b = np.zeros((N, G), np.uint16)
    _check(lib().orc_quantize(_p(w16), N, K, bits, gs, dt, _p(wq), _p(s), _p(b)), "quantize")
    return wq, s, b


def e8m0_encode(x):
    """[P4] to_fp8_e8m0 of a float (the exact log-scale reading)."""
    return lib().orc_e8m0_encode(float(x))


def e4m3_encode(x):
    """E4M3FN encoding of a float: ties to even, saturating at 448."""
    return lib().orc_e4m3_encode(float(x))


def e2m1_encode(x):
    """[P4] to_fp4_e2m1 of a float."""
    return lib().orc_e2m1_encode(float(x))


def quantize_fp4(w16, gs, dt):
    """w16: [N, K] uint16 T patterns -> (codes [N, K/2] u8, scales [N, K/gs] u8);
    E8M0 scales for gs = 32, E4M3 for gs = 16."""
    w16 = _c(w16, np.uint16)
    N, K = w16.shape
    codes = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // gs), np.uint8)
    _check(lib().orc_quantize_fp4(_p(w16), N, K, gs, dt, _p(codes), _p(scales)), "quantize_fp4")
    return codes, scales


def quantize_mxfp8(w16, dt):
    """MXFP8 weights: w16 [N, K] uint16 T patterns -> (codes [N, K] E4M3
    bytes, scales [N, K/32] E8M0 bytes)."""
    w16 = _c(w16, np.uint16)
    N, K = w16.shape
    codes = np.zeros((N, K), np.uint8)
    scales = np.zeros((N, K // 32), np.uint8)
    _check(lib().orc_quantize_mxfp8(_p(w16), N, K, dt, _p(codes), _p(scales)), "quantize_mxfp8")
    return codes, scales


def quantize_dequantize_fp(w16, bits, gs, dt):
    """[P4] fp_quantize_dequantize: w16 [N, K] uint16 T patterns -> the fake-
    quantized [N, K] T patterns (E2M1 elements for bits 4, E4M3 for bits 8;
    E8M0 scales for gs = 32, E4M3 for gs = 16)."""
    w16 = _c(w16, np.uint16)
    N, K = w16.shape
    out = np.zeros((N, K), np.uint16)
    _check(lib().orc_quantize_dequantize_fp(_p(w16), N, K, bits, gs, dt, _p(out)),
           "quantize_dequantize_fp")
    return out


def qqmm(x16, wq, scales, N, gs, dt, w_in_t=False):
    """[P4] QQMatmul: x fake-quantized to FP4 (quantize_dequantize_fp, bits 4)
    times the FP4 weights' transpose -> (y [M, N], den [M, N]) as qmm."""
    xh = quantize_dequantize_fp(x16, 4, gs, dt)
    return qmm(xh, wq, scales, None, N, 4, gs, FP4, dt, w_in_t=w_in_t)


def unpack(wq, N, K, bits):
    wq = _c(wq, np.uint8)
    codes = np.zeros((N, K), np.uint8)
    _check(lib().orc_unpack(_p(wq), N, K, bits, _p(codes)), "unpack")
    return codes


def dequantize(wq, scales, biases, N, K, bits, gs, mode, dt):
    """-> (w_hat fp64 exact [N, K], w_t uint16 T patterns [N, K])."""
    wq = _c(wq, np.uint8)
    scales = _c(scales, np.uint8 if mode in (FP4, MXFP8) else np.uint16)
    biases = None if biases is None else _c(biases, np.uint16)
    wh = np.zeros((N, K), np.float64)
    wt = np.zeros((N, K), np.uint16)
    _check(lib().orc_dequantize(_p(wq), _p(scales), _p(biases), N, K, bits, gs, mode, dt,
                                _p(wh), _p(wt)), "dequantize")
    return wh, wt


def qmm(x16, wq, scales, biases, N, bits, gs, mode, dt, w_in_t=False):
    """y = x . w_hat^T in fp64 -> (y [M, N], den [M, N] = sum |x w_hat|).
    w_in_t: multiply by w_hat rounded once to T (the dequantize output)."""
    x16 = _c(x16, np.uint16)
    M, K = x16.shape
    wq = _c(wq, np.uint8)
    scales = _c(scales, np.uint8 if mode in (FP4, MXFP8) else np.uint16)
    biases = None if biases is None else _c(biases, np.uint16)
    y = np.zeros((M, N), np.float64)
    den = np.zeros((M, N), np.float64)
    _check(lib().orc_qmm(_p(x16), _p(wq), _p(scales), _p(biases), M, N, K, bits, gs, mode, dt,
                         int(w_in_t), _p(y), _p(den)), "qmm")
    return y, den


def qmm_nt(x16, wq, scales, biases, K, bits, gs, mode, dt):
    """The non-transposed product of quantized_matmul (transpose = false; the
    product its VJP forms for x): with the weight stored as [N, K] rows
    quantized along K, y [M, K] = x [M, N] . w_hat [N, K], in fp64 over the
    exact w_hat.  -> (y [M, K], den [M, K] = sum_n |x w_hat|)."""
    x16 = _c(x16, np.uint16)
    M, N = x16.shape
    wh, _ = dequantize(wq, scales, biases, N, K, bits, gs, mode, dt)
    x = np.array([[t_to_double(int(v), dt) for v in row] for row in x16], np.float64).reshape(M, N)
    return x @ wh, np.abs(x) @ np.abs(wh)


def gather_qmm(x16, wq, scales, biases, lhs, rhs, N, bits, gs, mode, dt, w_in_t=False):
    """gather_qmm ("Add the 3bit packed qmm_t", ops and GatherQMM; the batch
    offsets of adjust_matrix_offsets): x16 [Bx, M, K], wq [E, N, row bytes],
    scales / biases [E, N, K/gs]; pair i multiplies x batch lhs[i] by the
    transpose of weight matrix rhs[i].  -> (y [P, M, N], den [P, M, N])."""
    ys, dens = [], []
    for l, r in zip(lhs, rhs):
        y, den = qmm(x16[int(l)], wq[int(r)], scales[int(r)],
                     None if biases is None else biases[int(r)], N, bits, gs, mode, dt,
                     w_in_t=w_in_t)
        ys.append(y)
        dens.append(den)
    return np.stack(ys), np.stack(dens)


def qmm_sampled(x16, wq, scales, biases, N, bits, gs, mode, dt, ms, ns, w_in_t=False):
    x16 = _c(x16, np.uint16)
    M, K = x16.shape
    wq = _c(wq, np.uint8)
    scales = _c(scales, np.uint8 if mode in (FP4, MXFP8) else np.uint16)
    biases = None if biases is None else _c(biases, np.uint16)
    ms = _c(ms, np.int64)
    ns = _c(ns, np.int64)
    y = np.zeros(len(ms), np.float64)
    den = np.zeros(len(ms), np.float64)
    _check(lib().orc_qmm_sampled(_p(x16), _p(wq), _p(scales), _p(biases), M, N, K, bits, gs,
                                 mode, dt, int(w_in_t), _p(ms), _p(ns), len(ms), _p(y), _p(den)),
           "qmm_sampled")
    return y, den


def conv_out_hw(H, W, kh, kw, sh, sw, ph, pw):
    return (H + 2 * ph - kh) // sh + 1, (W + 2 * pw - kw) // sw + 1


def qconv2d_nhwc(x16, wq, scales, biases, Cout, kh, kw, stride, pad, groups, bits, gs, dt,
                 ms=None, cos=None, w_in_t=False):
    """x16 [B, H, W, Cin] -> (y, den) as [B, Ho, Wo, Cout] fp64, or at sampled (m, co)."""
    x16 = _c(x16, np.uint16)
    B, H, W, Cin = x16.shape
    sh, sw = stride
    ph, pw = pad
    Ho, Wo = conv_out_hw(H, W, kh, kw, sh, sw, ph, pw)
    wq = _c(wq, np.uint8)
    scales = _c(scales, np.uint16)
    biases = _c(biases, np.uint16)
    if ms is not None:
        ms = _c(ms, np.int64)
        cos = _c(cos, np.int64)
        y = np.zeros(len(ms), np.float64)
        den = np.zeros(len(ms), np.float64)
        cnt = len(ms)
    else:
        y = np.zeros((B, Ho, Wo, Cout), np.float64)
        den = np.zeros((B, Ho, Wo, Cout), np.float64)
        cnt = 0
    _check(lib().orc_qconv2d_nhwc(_p(x16), _p(wq), _p(scales), _p(biases), B, H, W, Cin, Cout,
                                  kh, kw, sh, sw, ph, pw, groups, bits, gs, dt, int(w_in_t),
                                  _p(ms), _p(cos), cnt, _p(y), _p(den)), "qconv2d_nhwc")
    return y, den
