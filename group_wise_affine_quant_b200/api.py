"""Thin Python binding over the C ABI (include/aq.h), one function per entry
point with the same name.  It only marshals arguments: torch tensors supply
device memory and the current CUDA stream; every step of the computation runs
in libaq.so's kernels.

Tensors: x / w / y are fp16 or bf16 CUDA tensors; w_q is uint8 [N, K*bits/8];
affine scales / biases are T [N, K/group_size]; FP4 scales are uint8.
"""
import torch

from . import _lib
from ._lib import (AQ_BF16, AQ_F16, AQ_MODE_AFFINE, AQ_MODE_FP4, AQ_OP_QCONV2D, AQ_OP_QMM,
                   AQ_OP_QMM_NT, AQ_OP_QMV, AQ_OP_QQMM, AqError, check, lib)

__all__ = ["aq_quantize", "aq_quantize_fp4", "aq_quantize_dequantize_fp", "aq_qqmm", "aq_dequantize", "aq_qmv", "aq_qmv_batched", "aq_qmm", "aq_qmm_nt", "aq_gather_qmm", "aq_qconv2d_nhwc",
           "aq_workspace_size", "aq_qmv_noalloc", "aq_last_error", "aq_set_weight_prefetch",
           "aq_get_weight_prefetch", "aq_set_input_prefetch", "aq_get_input_prefetch", "AqError", "AQ_MODE_AFFINE", "AQ_MODE_FP4", "Workspace"]

_DT = {torch.float16: AQ_F16, torch.bfloat16: AQ_BF16}
_TORCH_DT = {AQ_F16: torch.float16, AQ_BF16: torch.bfloat16}


def _dt(t):
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError("expected an fp16 or bf16 tensor, got %s" % t.dtype) from None


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(device):
    return torch.cuda.current_stream(device).cuda_stream


def _mode(scales):
    return AQ_MODE_FP4 if scales.dtype == torch.uint8 else AQ_MODE_AFFINE


class Workspace:
    """Per-device zero-initialised scratch buffer for the ABI's workspace
    argument, grown on demand (a grown buffer is zero-filled again).  The
    tensor-core qmv kernels keep split-K partials and counters there and leave
    it zero-filled after every call; one Workspace serves calls issued on one
    stream at a time."""

    def __init__(self):
        self._bufs = {}

    def get(self, device, nbytes):
        if nbytes == 0:
            return None
        buf = self._bufs.get(device)
        if buf is None or buf.numel() < nbytes:
            buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
            self._bufs[device] = buf
        return buf


_default_ws = Workspace()


def aq_set_weight_prefetch(enable):
    """Stream weights before waiting on the previous kernel (see include/aq.h)."""
    lib().aq_set_weight_prefetch(1 if enable else 0)


def aq_get_weight_prefetch():
    return bool(lib().aq_get_weight_prefetch())


def aq_set_input_prefetch(enable):
    """Read x before waiting on the previous kernel (see include/aq.h)."""
    lib().aq_set_input_prefetch(1 if enable else 0)


def aq_get_input_prefetch():
    return bool(lib().aq_get_input_prefetch())


def aq_last_error():
    return lib().aq_last_error().decode()


def aq_workspace_size(op, M, N, K, bits, group_size, mode=AQ_MODE_AFFINE, groups=1):
    return lib().aq_workspace_size(op, M, N, K, bits, group_size, mode, groups)


def aq_quantize(w, bits=4, group_size=64, out=None):
    """w [N, K] T -> (w_q uint8 [N, K*bits/8], scales T [N, G], biases T [N, G])."""
    N, K = w.shape
    if out is None:
        G = K // group_size if group_size > 0 else 0
        out = (torch.empty((N, K * bits // 8), dtype=torch.uint8, device=w.device),
               torch.empty((N, G), dtype=w.dtype, device=w.device),
               torch.empty((N, G), dtype=w.dtype, device=w.device))
    w_q, s, b = out
    check(lib().aq_quantize(_ptr(w), _ptr(w_q), _ptr(s), _ptr(b), N, K, bits, group_size, _dt(w),
                            _stream(w.device)), "aq_quantize")
    return w_q, s, b


def aq_quantize_fp4(w, group_size=32, out=None):
    """w [N, K] fp16/bf16 -> (codes [N, K/2] uint8, scales [N, K/group_size]
    uint8): E2M1 codes with E8M0 (group 32) or E4M3 (group 16) scales."""
    N, K = w.shape
    if out is None:
        out = (torch.empty((N, K // 2), dtype=torch.uint8, device=w.device),
               torch.empty((N, K // group_size), dtype=torch.uint8, device=w.device))
    check(lib().aq_quantize_fp4(_ptr(w), _ptr(out[0]), _ptr(out[1]), N, K, group_size, _dt(w),
                                _stream(w.device)), "aq_quantize_fp4")
    return out


def aq_quantize_dequantize_fp(x, bits=4, group_size=32, out=None):
    """Fake quantization of x [N, K] fp16/bf16: E2M1 (bits 4) or E4M3 (bits 8)
    elements under E8M0 (group 32) or E4M3 (group 16) scales, back in T."""
    N, K = x.shape
    if out is None:
        out = torch.empty_like(x)
    check(lib().aq_quantize_dequantize_fp(_ptr(x), _ptr(out), N, K, bits, group_size, _dt(x),
                                          _stream(x.device)), "aq_quantize_dequantize_fp")
    return out


def aq_qqmm(x, w_q, scales, group_size=32, out=None, workspace=None):
    """W4A4: y = fq(x) . dequant(w)^T with FP4 weights and x fake-quantized to
    the weights' FP4 format."""
    M, K = x.shape
    N = w_q.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=x.dtype, device=x.device)
    ws_bytes = aq_workspace_size(AQ_OP_QQMM, M, N, K, 4, group_size, AQ_MODE_FP4)
    ws = (workspace or _default_ws).get(x.device, ws_bytes)
    check(lib().aq_qqmm(_ptr(x), _ptr(w_q), _ptr(scales), _ptr(out), M, N, K, group_size, _dt(x),
                        _ptr(ws), 0 if ws is None else ws.numel(), _stream(x.device)), "aq_qqmm")
    return out


def aq_dequantize(w_q, scales, biases, K, bits=4, group_size=64, dtype=None, out=None):
    """-> w_out T [N, K].  dtype defaults to the affine scales' dtype (bf16 for FP4)."""
    mode = _mode(scales)
    N = w_q.shape[0]
    if dtype is None:
        dtype = scales.dtype if mode == AQ_MODE_AFFINE else torch.bfloat16
    if out is None:
        out = torch.empty((N, K), dtype=dtype, device=w_q.device)
    check(lib().aq_dequantize(_ptr(w_q), _ptr(scales), _ptr(biases), _ptr(out), N, K, bits,
                              group_size, mode, _DT[dtype], _stream(w_q.device)), "aq_dequantize")
    return out


def _mm(fn_name, op, x, w_q, scales, biases, bits, group_size, out, workspace):
    M, K = x.shape
    N = w_q.shape[0]
    mode = _mode(scales)
    if out is None:
        out = torch.empty((M, N), dtype=x.dtype, device=x.device)
    ws_bytes = aq_workspace_size(op, M, N, K, bits, group_size, mode)
    ws = (workspace or _default_ws).get(x.device, ws_bytes)
    fn = getattr(lib(), fn_name)
    check(fn(_ptr(x), _ptr(w_q), _ptr(scales), _ptr(biases), _ptr(out), M, N, K, bits,
             group_size, mode, _dt(x), _ptr(ws), 0 if ws is None else ws.numel(),
             _stream(x.device)), fn_name)
    return out


def aq_qmv(x, w_q, scales, biases, bits=4, group_size=64, out=None, workspace=None):
    """y = x . dequant(w)^T for 1 <= M <= 16 rows of x."""
    return _mm("aq_qmv", AQ_OP_QMV, x, w_q, scales, biases, bits, group_size, out, workspace)


def aq_qmv_noalloc(x, w_q, scales, biases, bits=4, group_size=64, out=None):
    """aq_qmv on the library's fixed scratch (no workspace; the C call
    allocates nothing).  `out` is allocated here by torch if not given."""
    M, K = x.shape
    N = w_q.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=x.dtype, device=x.device)
    check(lib().aq_qmv_noalloc(_ptr(x), _ptr(w_q), _ptr(scales), _ptr(biases), _ptr(out), M, N,
                               K, bits, group_size, _mode(scales), _dt(x), _stream(x.device)),
          "aq_qmv_noalloc")
    return out


def aq_qmv_batched(xs, w_qs, scales, biases, bits=4, group_size=64, outs=None, workspace=None):
    """Independent problems y_i = x_i . dequant(w_i)^T (all x_i with the same
    M <= 16, one dtype, one format) in one call; biases is a list (or None for
    FP4).  Returns the list of outputs."""
    n = len(xs)
    if not (len(w_qs) == len(scales) == n) or (biases is not None and len(biases) != n):
        raise ValueError("one w_q, scales (and biases) per x")
    if n == 0:
        return []
    M = xs[0].shape[0]
    mode = _mode(scales[0])
    if outs is None:
        outs = [torch.empty((M, w.shape[0]), dtype=x.dtype, device=x.device) for x, w in zip(xs, w_qs)]
    arr = (_lib.QmvProblem * n)()
    for i in range(n):
        arr[i] = _lib.QmvProblem(_ptr(xs[i]), _ptr(w_qs[i]), _ptr(scales[i]),
                                 None if biases is None else _ptr(biases[i]), _ptr(outs[i]),
                                 w_qs[i].shape[0], xs[i].shape[1])
    L = lib()
    ws_bytes = L.aq_qmv_batched_workspace_size(arr, n, M, bits, group_size, mode)
    ws = (workspace or _default_ws).get(xs[0].device, ws_bytes)
    check(L.aq_qmv_batched(arr, n, M, bits, group_size, mode, _dt(xs[0]), _ptr(ws),
                           0 if ws is None else ws.numel(), _stream(xs[0].device)),
          "aq_qmv_batched")
    return outs


def aq_gather_qmm(x, w_q, scales, biases, lhs_indices=None, rhs_indices=None, bits=4,
                  group_size=64, out=None, workspace=None):
    """Pair i: y[i] = x[lhs[i]] . dequant(w[rhs[i]])^T, with x [Bx, M, K],
    w_q [E, N, K*bits/8], scales / biases [E, N, K/group_size]; the index
    lists are host sequences of int (None: 0, 1, ...).  Returns [P, M, N]."""
    import ctypes
    Bx, M, K = x.shape
    E, N = w_q.shape[0], w_q.shape[1]
    n = len(lhs_indices) if lhs_indices is not None else (
        len(rhs_indices) if rhs_indices is not None else min(Bx, E))
    mode = _mode(scales)

    def arr(ix):
        if ix is None:
            return None
        return (ctypes.c_int32 * n)(*[int(v) for v in ix])
    if out is None:
        out = torch.empty((n, M, N), dtype=x.dtype, device=x.device)
    L = lib()
    ws_bytes = L.aq_gather_qmm_workspace_size(n, M, N, K, bits, group_size, mode)
    ws = (workspace or _default_ws).get(x.device, ws_bytes)
    check(L.aq_gather_qmm(_ptr(x), _ptr(w_q), _ptr(scales), _ptr(biases), arr(lhs_indices),
                          arr(rhs_indices), _ptr(out), n, M, N, K, Bx, E, bits, group_size, mode,
                          _dt(x), _ptr(ws), 0 if ws is None else ws.numel(),
                          _stream(x.device)), "aq_gather_qmm")
    return out


def aq_qmm(x, w_q, scales, biases, bits=4, group_size=64, out=None, workspace=None):
    """y = x . dequant(w)^T for any M."""
    return _mm("aq_qmm", AQ_OP_QMM, x, w_q, scales, biases, bits, group_size, out, workspace)


def aq_qmm_nt(x, w_q, scales, biases, bits=4, group_size=64, out=None, workspace=None):
    """y [M, K] = x [M, N] . dequant(w) with the weight stored [N, K] as for
    aq_qmv / aq_qmm (the transpose = false product)."""
    M, N = x.shape
    K = w_q.shape[1] * 8 // bits
    mode = _mode(scales)
    if out is None:
        out = torch.empty((M, K), dtype=x.dtype, device=x.device)
    ws_bytes = aq_workspace_size(AQ_OP_QMM_NT, M, N, K, bits, group_size, mode)
    ws = (workspace or _default_ws).get(x.device, ws_bytes)
    check(lib().aq_qmm_nt(_ptr(x), _ptr(w_q), _ptr(scales), _ptr(biases), _ptr(out), M, N, K, bits,
                          group_size, mode, _dt(x), _ptr(ws), 0 if ws is None else ws.numel(),
                          _stream(x.device)), "aq_qmm_nt")
    return out


def conv_out_hw(H, W, kh, kw, stride, pad):
    return (H + 2 * pad[0] - kh) // stride[0] + 1, (W + 2 * pad[1] - kw) // stride[1] + 1


def aq_qconv2d_nhwc(x, w_q, scales, biases, Cout, kh, kw, stride=(1, 1), pad=(0, 0), groups=1,
                    bits=4, group_size=64, out=None, workspace=None):
    """x [B, H, W, Cin] T -> y [B, Ho, Wo, Cout] T (weights as aq_qconv2d_nhwc documents)."""
    B, H, W, Cin = x.shape
    Ho, Wo = conv_out_hw(H, W, kh, kw, stride, pad)
    if out is None:
        out = torch.empty((B, Ho, Wo, Cout), dtype=x.dtype, device=x.device)
    Cg = Cin // groups if groups > 0 else 0
    Kp = -(-kh * kw * Cg // group_size) * group_size if group_size > 0 else 0
    ws_bytes = aq_workspace_size(AQ_OP_QCONV2D, B * Ho * Wo, Cout // max(groups, 1), Kp, bits,
                                 group_size, AQ_MODE_AFFINE, groups)
    ws = (workspace or _default_ws).get(x.device, ws_bytes)
    check(lib().aq_qconv2d_nhwc(_ptr(x), _ptr(w_q), _ptr(scales), _ptr(biases), _ptr(out), B, H,
                                W, Cin, Cout, kh, kw, stride[0], stride[1], pad[0], pad[1],
                                groups, bits, group_size, _dt(x), _ptr(ws),
                                0 if ws is None else ws.numel(), _stream(x.device)),
          "aq_qconv2d_nhwc")
    return out
