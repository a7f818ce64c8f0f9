"""Test helpers: independent numpy routes for packing and T decoding, and the
matmul error bound.  None of this is the library or the oracle; the bit
packing here goes through numpy's packbits/unpackbits, a different route from
the oracle's shift-and-mask code, so that each checks the other.
"""
import numpy as np
import torch

F16, BF16 = 0, 1
AFFINE, FP4 = 0, 1
T_MAX = {F16: 65504.0, BF16: float(torch.finfo(torch.bfloat16).max)}
REL_TOL = 2e-3   # |y - y_ref| <= REL_TOL * sum_k |x_k w_hat_k| + 1 ulp_T(y_ref)


def u16_to_f64(u16, dt):
    """Decode raw fp16 / bf16 patterns with numpy / torch (library routes)."""
    u16 = np.ascontiguousarray(u16, dtype=np.uint16)
    if dt == F16:
        return u16.view(np.float16).astype(np.float64)
    t = torch.from_numpy(u16.view(np.int16).copy()).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def f64_to_u16(v, dt):
    """Round to T with torch (fp16 via numpy, which rounds fp64 -> fp16 once)."""
    v = np.asarray(v, dtype=np.float64)
    if dt == F16:
        return v.astype(np.float16).view(np.uint16)
    t = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def np_unpack(wq, N, K, bits):
    """Codes of a packed matrix, reading each row as a little-endian bit stream."""
    wq = np.ascontiguousarray(wq, dtype=np.uint8).reshape(N, K * bits // 8)
    b = np.unpackbits(wq, axis=1, bitorder="little").reshape(N, K, bits)
    weights = (1 << np.arange(bits)).astype(np.int64)
    return (b.astype(np.int64) * weights).sum(axis=2).astype(np.uint8)


def np_pack(codes, bits):
    """Inverse of np_unpack: [N, K] codes -> [N, K*bits/8] bytes."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    b = ((codes[..., None] >> np.arange(bits, dtype=np.uint8)) & 1).astype(np.uint8)
    return np.packbits(b.reshape(N, K * bits), axis=1, bitorder="little")


def ulp_t(v, dt):
    """Spacing of T at |round_T(v)| (the smallest subnormal spacing at 0)."""
    r = np.abs(u16_to_f64(f64_to_u16(v, dt), dt))
    frac = 10 if dt == F16 else 7
    emin = -14 if dt == F16 else -126
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(r > 0, r, 1.0)))
    e = np.maximum(e, emin)
    return np.ldexp(1.0, (e - frac).astype(np.int64))


def check_matmul(y_t_u16, y_ref, den, dt, rel=REL_TOL, what="y", overflow_any_nonfinite=False):
    """Assert the bound elementwise.  y_t_u16: T patterns from the device.
    Near T's overflow threshold either a finite value within the bound or the
    same-signed infinity is accepted; far above it only the infinity.  With
    overflow_any_nonfinite (weights whose scales reach 2^127, where fp32
    partial sums overflow and +inf meets -inf), any non-finite value is
    accepted where the exact result overflows T or where the sum of the
    terms' magnitudes reaches fp32's range."""
    y = u16_to_f64(y_t_u16, dt).reshape(y_ref.shape)
    tol = rel * den + ulp_t(y_ref, dt)
    tmax = T_MAX[dt]
    must_inf = np.abs(y_ref) - tol > tmax
    may_inf = np.abs(y_ref) + tol >= tmax
    fin = np.isfinite(y)
    ok_inf = (~fin) & np.isinf(y) & (np.sign(y) == np.sign(y_ref)) & may_inf
    if overflow_any_nonfinite:
        # fp32 accumulation can overflow on the way when the terms' magnitudes
        # sum past fp32's range, even if the exact result is finite.
        fp32_over = den >= 0.5 * float(np.finfo(np.float32).max)
        ok_inf = ok_inf | ((~fin) & (may_inf | fp32_over))
    ok_fin = fin & (np.abs(y - y_ref) <= tol) & ~must_inf
    ok = ok_inf | ok_fin
    if not ok.all():
        bad = np.argwhere(~ok)
        i = tuple(bad[0])
        raise AssertionError(
            "%s: %d of %d outside |y-y_ref| <= %g*den + ulp; first at %s: y=%r ref=%r den=%r"
            % (what, len(bad), ok.size, rel, i, y[i], y_ref[i], den[i]))
    err = np.abs(np.where(fin, y, 0) - y_ref) / np.maximum(tol, 1e-300)
    return float(np.max(np.where(fin, err, 0)))


def qmv_w_in_t(M, K, bits, gs, mode=0):
    """Which w_hat aq_qmv multiplies: every aq_qmv kernel keeps w_hat in fp32
    (scale and bias applied per group in fp32 to the exact integer-code
    products, as the qmv of "Add the 3bit packed qmm_t" does), so its
    reference is the exact product for every M and shape."""
    return False
