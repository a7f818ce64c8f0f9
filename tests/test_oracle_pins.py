"""Pins for the CPU oracle: each test checks the oracle against something other
than itself — values the pages print (tests/golden/), closed forms,
library routines (numpy / torch conversions, matmul, conv2d), brute force,
and invariants of the quantizer the pages describe.

Sources: "mlx 1.0.0, mlx/backend/cpu/quantized.cpp" (quantize, extract_bits,
FP4_LUT, dequantize_scale, fp_qmm_t); "Improvements in the quantizer and
dequantization kernel" (the scale/bias rule); "[Feature] Quantized
Convolution 2D - Possible PR?" (flatten, pad, im2col order, grouped conv).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests.util import (AFFINE, BF16, F16, FP4, f64_to_u16, np_pack, np_unpack,
                        u16_to_f64)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BITS = (2, 3, 4, 5, 6, 8)
GROUPS = (32, 64, 128)


def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ----------------------------------------------------------------- T decode

@pytest.mark.parametrize("dt", [F16, BF16])
def test_t_decode_all_patterns(dt):
    lib = oracle.lib()
    pats = np.arange(65536, dtype=np.uint16)
    ref = u16_to_f64(pats, dt)
    got = np.array([lib.orc_t_to_double(int(p), dt) for p in pats])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def test_round_to_f16_matches_numpy():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(20000) * s for s in (1e-7, 1e-5, 1e-2, 1, 1e3, 7e4)])
    # exact midpoints between neighbouring halves exercise ties-to-even
    h = np.arange(0, 0x7bff, 37, dtype=np.uint16)
    a = h.view(np.float16).astype(np.float64)
    b = (h + 1).view(np.float16).astype(np.float64)
    v = np.concatenate([v, (a + b) / 2, -(a + b) / 2, [0.0, -0.0, 65520.0, 65519.99, 1e-9]])
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    got = np.array([oracle.round_to_t(x, F16) for x in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_round_to_bf16_matches_torch():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32) * np.float32(s)
                        for s in (1e-38, 1e-20, 1e-3, 1, 1e20, 1e38)])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.round_to_t(float(x), BF16) for x in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------ FP4 and scales

def test_fp4_lut_matches_printed_table():
    rows = _golden_rows("fp4_e2m1_lut.txt")
    assert len(rows) == 16
    for code, val in rows:
        got = oracle.e2m1(int(code))
        assert got == float(val)
        assert np.signbit(got) == val.startswith("-")


def test_e8m0_matches_page_bit_rule():
    for s, bits in _golden_rows("e8m0_rule.txt"):
        assert (0x40 if int(s) == 0 else int(s) << 7) == int(bits, 16)
    for s in range(256):
        pat = np.array([0x40 if s == 0 else s << 7], dtype=np.uint16)
        ref = u16_to_f64(pat, BF16)[0]
        assert oracle.e8m0(s) == ref, s


def test_e4m3_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3(s) for s in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert oracle.e4m3(0x7E) == 448.0


# ------------------------------------------------------------------ packing

def _quantize_exact_grid(codes, bits, gs, dt, negative_scale=False):
    """Weights that sit exactly on a quantizer grid with known codes.

    Each group is bias + step*code with step = 2^-3 and bias = -q0*step (or
    mirrored for the negative-scale orientation) and contains both code 0 and
    code 2^bits - 1, so the quantizer must recover exactly `codes`."""
    nb = (1 << bits) - 1
    step = 0.125
    N, K = codes.shape
    c = codes.astype(np.float64)
    if not negative_scale:
        # |min| > |max|: bias at the minimum, positive scale, codes count up.
        lo = -(nb // 2 + 1) * step
        w = lo + step * c
    else:
        # |max| >= |min|: bias at the maximum, negative scale, codes count down.
        hi = (nb // 2 + 1) * step
        w = hi - step * c
    return f64_to_u16(w, dt)


def _grid_codes(N, K, bits, gs, seed):
    rng = np.random.default_rng(seed)
    nb = (1 << bits) - 1
    codes = rng.integers(0, nb + 1, size=(N, K)).astype(np.uint8)
    g = codes.reshape(N, K // gs, gs)
    g[:, :, 0] = 0
    g[:, :, 1] = nb
    return g.reshape(N, K)


@pytest.mark.parametrize("bits", BITS)
def test_unpack_matches_numpy_bitstream(bits):
    rng = np.random.default_rng(bits)
    N, K = 7, 384
    codes = rng.integers(0, 1 << bits, size=(N, K)).astype(np.uint8)
    wq = np_pack(codes, bits)
    assert np.array_equal(oracle.unpack(wq, N, K, bits), codes)


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("gs", GROUPS)
@pytest.mark.parametrize("dt", [F16, BF16])
@pytest.mark.parametrize("neg", [False, True])
def test_quantize_exact_grid(bits, gs, dt, neg):
    """Grid input: codes recovered exactly, packed bytes equal numpy's packing,
    scale/bias are the grid's, and w_hat reproduces w exactly."""
    N, K = 5, 2 * gs
    codes = _grid_codes(N, K, bits, gs, seed=bits * 1000 + gs)
    w = _quantize_exact_grid(codes, bits, gs, dt, negative_scale=neg)
    wq, s, b = oracle.quantize(w, bits, gs, dt)
    assert np.array_equal(wq, np_pack(codes, bits))
    nb = (1 << bits) - 1
    sv = u16_to_f64(s, dt)
    bv = u16_to_f64(b, dt)
    if not neg:
        assert np.all(sv == 0.125) and np.all(bv == -(nb // 2 + 1) * 0.125)
    else:
        assert np.all(sv == -0.125) and np.all(bv == (nb // 2 + 1) * 0.125)
    wh, wt = oracle.dequantize(wq, s, b, N, K, bits, gs, AFFINE, dt)
    assert np.array_equal(wh, u16_to_f64(w, dt))
    assert np.array_equal(wt, w)


@pytest.mark.parametrize("bits", [3, 5, 6])
def test_page_extraction_listing_random(bits):
    """The page's extract_bits masks and shifts, applied to packed bytes, give
    the oracle's codes (10^5 random packs with other codes random)."""
    terms = [r for r in _golden_rows("extract_bits_listing.txt") if int(r[0]) == bits]
    cpp = {3: 8, 5: 8, 6: 4}[bits]
    bpp = cpp * bits // 8
    rng = np.random.default_rng(bits)
    P = 100000
    codes = rng.integers(0, 1 << bits, size=(P, cpp)).astype(np.uint8)
    packed = np_pack(codes, bits)                              # [P, bpp]
    assert packed.shape[1] == bpp
    got = np.zeros((P, cpp), np.int64)
    for _, pos, order, byte, mask, r, l in terms:
        v = packed[:, int(byte)].astype(np.int64)
        mask, r, l = int(mask, 16), int(r), int(l)
        t = ((v & mask) >> r) if order == "M" else ((v >> r) & mask)
        got[:, int(pos)] += t << l
    assert np.array_equal(got, codes)
    assert np.array_equal(oracle.unpack(packed, P, cpp, bits), codes)


@pytest.mark.parametrize("bits", [3, 6])
@pytest.mark.slow
def test_page_extraction_listing_exhaustive_24bit(bits):
    """All 2^24 three-byte packs: the listing and the oracle's bit-stream read
    agree, and every pack decodes to a distinct code tuple (pack is a bijection)."""
    terms = [r for r in _golden_rows("extract_bits_listing.txt") if int(r[0]) == bits]
    cpp = 24 // bits
    allv = np.arange(1 << 24, dtype=np.int64)
    packed = np.stack([(allv >> (8 * i)) & 0xFF for i in range(3)], axis=1).astype(np.uint8)
    got = np.zeros((1 << 24, cpp), np.int64)
    for _, pos, order, byte, mask, r, l in terms:
        v = packed[:, int(byte)].astype(np.int64)
        mask, r, l = int(mask, 16), int(r), int(l)
        t = ((v & mask) >> r) if order == "M" else ((v >> r) & mask)
        got[:, int(pos)] += t << l
    recon = np.zeros(1 << 24, np.int64)
    for p in range(cpp):
        recon |= got[:, p] << (p * bits)
    assert np.array_equal(recon, allv)
    sub = packed[::4099]
    assert np.array_equal(oracle.unpack(sub, len(sub), cpp, bits).astype(np.int64), got[::4099])


def test_pack_factors_golden():
    for bits, cpp, bpp in _golden_rows("pack_factors.txt"):
        bits, cpp, bpp = int(bits), int(cpp), int(bpp)
        assert cpp * bits == 8 * bpp
        codes = (np.arange(cpp)[None, :] % (1 << bits)).astype(np.uint8)
        assert np_pack(codes, bits).shape[1] == bpp


# --------------------------------------------------------------- quantizer

@pytest.mark.parametrize("dt", [F16, BF16])
@pytest.mark.parametrize("bits", BITS)
def test_quantize_zero_and_constant_groups(dt, bits):
    gs = 32
    rows = [np.zeros(gs), np.full(gs, 0.75), np.full(gs, -3.0)]
    w = f64_to_u16(np.stack(rows), dt)
    wq, s, b = oracle.quantize(w, bits, gs, dt)
    codes = np_unpack(wq, 3, gs, bits)
    assert np.all(codes == 0)
    # all-zero group: range 0 -> scale = -1e-7 (|max| >= |min|), q0 = 0, bias 0
    assert u16_to_f64(s[0], dt)[0] == u16_to_f64(f64_to_u16(-np.float32(1e-7), dt), dt)[0]
    assert u16_to_f64(b[0], dt)[0] == 0.0
    # constant c: bias = c exactly, code 0 reproduces it
    assert u16_to_f64(b[1], dt)[0] == 0.75
    assert u16_to_f64(b[2], dt)[0] == -3.0
    wh, _ = oracle.dequantize(wq, s, b, 3, gs, bits, gs, AFFINE, dt)
    assert np.all(wh[1] == 0.75) and np.all(wh[2] == -3.0)


def _random_groups(dt, bits, n=400, gs=64, seed=0, zero_frac=0.2):
    rng = np.random.default_rng(seed + bits)
    sig = rng.choice([1e-3, 0.02, 1.0, 30.0], size=(n, 1))
    w = rng.standard_normal((n, gs)) * sig
    w[rng.random((n, gs)) < zero_frac / 4] = 0.0
    w[rng.random(n) < 0.2, 0] = 0.0
    return f64_to_u16(w, dt)


@pytest.mark.parametrize("dt", [F16, BF16])
@pytest.mark.parametrize("bits", BITS)
def test_quantize_invariants(dt, bits):
    """For random groups: (1) 0 maps to code -q0 (the zero-adjusted scale);
    (2) the refined error bound; (3) codes are monotone in w along the sign of
    the scale; (4) every code is the clamped nearest grid point."""
    gs = 64
    n = 400
    w = _random_groups(dt, bits, n=n, gs=gs)
    wq, s, b = oracle.quantize(w, bits, gs, dt)
    codes = np_unpack(wq, n, gs, bits).astype(np.int64)
    wv = u16_to_f64(w, dt)
    sT = u16_to_f64(s, dt)[:, 0]
    bT = u16_to_f64(b, dt)[:, 0]
    nb = (1 << bits) - 1
    w32 = wv.astype(np.float32)
    lo, hi = w32.min(1), w32.max(1)
    at_min = np.abs(lo) > np.abs(hi)
    for i in range(n):
        edge = lo[i] if at_min[i] else hi[i]
        # fp32 scale before T rounding, recomputed only to bound the error
        s0 = np.float32(max(np.float32(hi[i] - lo[i]) / np.float32(nb), np.float32(1e-7)))
        s0 = s0 if at_min[i] else -s0
        q0 = np.rint(np.float32(edge) / s0)
        s32 = np.float32(edge) / q0 if q0 != 0 else s0
        b32 = edge if q0 != 0 else 0.0
        # (1) zero lands on code -q0
        zeros = wv[i] == 0
        if zeros.any():
            assert np.all(codes[i][zeros] == (-q0 if q0 != 0 else 0))
        # (2) refined bound, with s the fp32 scale
        wh = sT[i] * codes[i] + bT[i]
        # T rounding of scale and bias, plus the fp32 rounding of (w - b)/s
        slack = (codes[i] * abs(sT[i] - float(s32)) + abs(bT[i] - float(b32))
                 + (nb + 1) * abs(float(s32)) * 2.0 ** -23)
        unclamped = np.abs(wh - wv[i]) <= (abs(float(s32)) / 2 + slack) * (1 + 1e-6)
        clamped_ok = np.abs(wh - wv[i]) <= (abs(float(s32)) + slack) * (1 + 1e-6)
        at_edge = (codes[i] == 0) | (codes[i] == nb)
        assert np.all(unclamped | (at_edge & clamped_ok)), i
        # (3) monotone
        order = np.argsort(wv[i], kind="stable")
        c_sorted = codes[i][order]
        d = np.diff(c_sorted)
        assert np.all(d >= 0) if sT[i] > 0 else np.all(d <= 0), i
        # (4) clamped nearest grid point in the fp32 grid
        t = (w32[i] - np.float32(b32)) / np.float32(s32)
        assert np.all(np.abs(codes[i] - np.clip(t, 0, nb)) <= 0.5 + 1e-6), i


def _tie_cases():
    cases, cur = [], None
    with open(os.path.join(GOLDEN, "quantize_ties.txt")) as f:
        for ln in f:
            if not ln.strip() or ln.startswith("#"):
                continue
            tok = ln.split()
            if tok[0] == "case":
                kv = dict(t.split("=") for t in tok[2:])
                cur = {"name": tok[1], "bits": int(kv["bits"]),
                       "dt": F16 if kv["dt"] == "f16" else BF16}
                cases.append(cur)
            else:
                vals = []
                for t in tok[1:]:
                    v, _, n = t.partition("*")
                    vals += [v] * (int(n) if n else 1)
                cur[tok[0]] = vals
    return cases


@pytest.mark.parametrize("case", _tie_cases(), ids=lambda c: "%s-%s" % (
    c["name"], "f16" if c["dt"] == F16 else "bf16"))
def test_quantize_golden_ties(case):
    """Hand-derived groups (tests/golden/quantize_ties.txt) whose codes,
    scale and bias are fixed by rint's ties-to-even and by the divisions
    (w - b)/s, edge/s0 and (hi - lo)/n_bins being done in fp32: an oracle
    that rounded half away from zero, or divided in fp64, fails here."""
    dt, bits = case["dt"], case["bits"]
    w = np.array([float(v) for v in case["w"]])
    assert len(w) == 32
    w16 = f64_to_u16(w, dt)
    assert np.array_equal(u16_to_f64(w16, dt), w), "inputs must be exact in T"
    wq, s, b = oracle.quantize(w16[None, :], bits, 32, dt)
    want = np.array([int(c) for c in case["codes"]], dtype=np.uint8)
    assert np.array_equal(np_unpack(wq, 1, 32, bits)[0], want)
    assert int(s[0, 0]) == int(case["scale"][0], 16)
    assert int(b[0, 0]) == int(case["bias"][0], 16)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantize_small_alphabet_smoke(bits):
    """Smoke check, not a pin: groups of 32 drawn from a 5-value alphabet,
    compared with the same steps restated in numpy float32.  The restatement
    repeats the oracle's own formula, so it only catches slips in the C++
    plumbing (packing, indexing); the rounding rule itself is pinned by
    test_quantize_golden_ties."""
    alphabet = np.array([-1.5, -0.25, 0.0, 0.5, 1.25])
    rng = np.random.default_rng(7)
    idx = rng.integers(0, 5, size=(3000, 32))
    w = f64_to_u16(alphabet[idx], F16)
    wq, s, b = oracle.quantize(w, bits, 32, F16)
    codes = np_unpack(wq, 3000, 32, bits)
    nb = (1 << bits) - 1
    wv = u16_to_f64(w, F16).astype(np.float32)
    for i in range(3000):
        lo, hi = wv[i].min(), wv[i].max()
        at_min = abs(lo) > abs(hi)
        st = np.float32(max(np.float32(hi - lo) / np.float32(nb), np.float32(1e-7)))
        st = st if at_min else -st
        edge = lo if at_min else hi
        q0 = np.rint(edge / st)
        if q0 != 0:
            st, bi = edge / q0, edge
        else:
            bi = np.float32(0)
        want = np.clip(np.rint((wv[i] - bi) / st), 0, nb)
        assert np.array_equal(codes[i], want.astype(np.uint8)), i


# --------------------------------------------------------------- matmuls

def _np_dequant(wq, s, b, N, K, bits, gs, dt):
    codes = np_unpack(wq, N, K, bits).astype(np.float64)
    sv = np.repeat(u16_to_f64(s, dt), gs, axis=1)
    bv = np.repeat(u16_to_f64(b, dt), gs, axis=1)
    return sv * codes + bv


@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("dt", [F16, BF16])
def test_qmm_matches_unfused_numpy(bits, dt):
    rng = np.random.default_rng(bits)
    M, N, K, gs = 5, 24, 256, 64
    w = f64_to_u16(rng.standard_normal((N, K)) * 0.05, dt)
    x = f64_to_u16(rng.standard_normal((M, K)), dt)
    wq, s, b = oracle.quantize(w, bits, gs, dt)
    y, den = oracle.qmm(x, wq, s, b, N, bits, gs, AFFINE, dt)
    W = _np_dequant(wq, s, b, N, K, bits, gs, dt)
    X = u16_to_f64(x, dt)
    assert np.allclose(y, X @ W.T, rtol=1e-12, atol=1e-12)
    assert np.allclose(den, np.abs(X) @ np.abs(W).T, rtol=1e-12, atol=1e-12)
    # the hoisted form used by weight-streaming kernels is the same sum
    codes = np_unpack(wq, N, K, bits).astype(np.float64)
    sv, bv = u16_to_f64(s, dt), u16_to_f64(b, dt)
    Xg = X.reshape(M, K // gs, gs)
    Cg = codes.reshape(N, K // gs, gs)
    hoisted = np.einsum("mgk,ngk,ng->mn", Xg, Cg, sv) + np.einsum("mgk,ng->mn", Xg, bv)
    assert np.allclose(y, hoisted, rtol=1e-12, atol=1e-10)
    ys, dens = oracle.qmm_sampled(x, wq, s, b, N, bits, gs, AFFINE, dt,
                                  [0, 4, 2], [0, 23, 11])
    assert np.array_equal(ys, y[[0, 4, 2], [0, 23, 11]])


@pytest.mark.parametrize("dt", [F16, BF16])
def test_qmm_w_in_t_uses_dequantize_output(dt):
    """The T-tile reference equals numpy's product with aq_dequantize's values
    (w_hat rounded once to T), and differs from the exact one by at most the
    T rounding of w_hat."""
    rng = np.random.default_rng(11 + dt)
    M, N, K, gs, bits = 3, 20, 192, 64, 3
    w = f64_to_u16(rng.standard_normal((N, K)) * 0.1, dt)
    x = f64_to_u16(rng.standard_normal((M, K)), dt)
    wq, s, b = oracle.quantize(w, bits, gs, dt)
    yt, dent = oracle.qmm(x, wq, s, b, N, bits, gs, AFFINE, dt, w_in_t=True)
    _, wt = oracle.dequantize(wq, s, b, N, K, bits, gs, AFFINE, dt)
    X = u16_to_f64(x, dt)
    WT = u16_to_f64(wt, dt)
    assert np.allclose(yt, X @ WT.T, rtol=1e-12, atol=1e-12)
    ye, den = oracle.qmm(x, wq, s, b, N, bits, gs, AFFINE, dt)
    u = 2.0 ** (-11 if dt == F16 else -8)
    assert np.all(np.abs(yt - ye) <= u * den * (1 + 1e-9))
    ys, _ = oracle.qmm_sampled(x, wq, s, b, N, bits, gs, AFFINE, dt, [1, 2], [3, 19], w_in_t=True)
    assert np.array_equal(ys, yt[[1, 2], [3, 19]])


def test_qmm_8bit_unit_scale_is_integer_gemm():
    """bits=8, scale 1, bias 0 reduces to an integer GEMM."""
    rng = np.random.default_rng(3)
    M, N, K, gs = 4, 16, 128, 32
    codes = rng.integers(0, 256, size=(N, K)).astype(np.uint8)
    wq = np_pack(codes, 8)
    s = f64_to_u16(np.ones((N, K // gs)), F16)
    b = f64_to_u16(np.zeros((N, K // gs)), F16)
    xi = rng.integers(-8, 9, size=(M, K))
    x = f64_to_u16(xi.astype(np.float64), F16)
    y, _ = oracle.qmm(x, wq, s, b, N, 8, gs, AFFINE, F16)
    assert np.array_equal(y, (xi @ codes.astype(np.int64).T).astype(np.float64))


@pytest.mark.parametrize("gs", [16, 32])
def test_fp4_qmm_matches_lut_times_scale(gs):
    rng = np.random.default_rng(gs)
    M, N, K = 3, 8, 128
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    wq = np_pack(codes, 4)
    if gs == 32:
        sc = rng.integers(117, 138, size=(N, K // gs)).astype(np.uint8)
        dec = np.ldexp(1.0, sc.astype(np.int64) - 127)
    else:
        sc = rng.integers(0, 0x7F, size=(N, K // gs)).astype(np.uint8)
        dec = torch.from_numpy(sc).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    lut = np.array([float(v) for _, v in _golden_rows("fp4_e2m1_lut.txt")])
    W = lut[codes] * np.repeat(dec, gs, axis=1)
    x = f64_to_u16(rng.standard_normal((M, K)), BF16)
    y, _ = oracle.qmm(x, wq, sc, None, N, 4, gs, FP4, BF16)
    assert np.allclose(y, u16_to_f64(x, BF16) @ W.T, rtol=1e-12, atol=1e-30)
    wh, wt = oracle.dequantize(wq, sc, None, N, K, 4, gs, FP4, BF16)
    assert np.array_equal(wh, W)


def test_fp4_fp16_scale_overflow_follows_t_cast():
    """E8M0 scales are cast to T before use: with fp16 activations 2^20
    overflows to inf and 2^-30 underflows to 0."""
    codes = np.full((1, 32), 2, np.uint8)              # LUT value 1.0
    wq = np_pack(codes, 4)
    for s, want in ((127 + 20, np.inf), (127 - 30, 0.0), (127, 1.0)):
        wh, _ = oracle.dequantize(wq, np.array([[s]], np.uint8), None, 1, 32, 4, 32, FP4, F16)
        assert np.all(wh == want), s


@pytest.mark.parametrize("groups,stride,pad", [(1, 1, 1), (2, 2, 0), (4, 1, 1), (1, 2, 1)])
def test_qconv_matches_torch_conv2d(groups, stride, pad):
    """Explicit im2col conv against torch's conv2d in fp64 on the same
    dequantized weights (flatten (kh, kw, Cg), pad to a group multiple)."""
    rng = np.random.default_rng(groups * 10 + stride)
    B, H, W, Cin, Cout, k, gs, bits, dt = 1, 5, 6, 8, 8, 3, 32, 4, BF16
    Cg = Cin // groups
    K = k * k * Cg
    Kp = (K + gs - 1) // gs * gs
    wt = rng.standard_normal((Cout, k, k, Cg)) * 0.2
    wflat = np.zeros((Cout, Kp))
    wflat[:, :K] = wt.reshape(Cout, K)
    wq, s, b = oracle.quantize(f64_to_u16(wflat, dt), bits, gs, dt)
    x = f64_to_u16(rng.standard_normal((B, H, W, Cin)), dt)
    y, den = oracle.qconv2d_nhwc(x, wq, s, b, Cout, k, k, (stride, stride), (pad, pad),
                                 groups, bits, gs, dt)
    What = _np_dequant(wq, s, b, Cout, Kp, bits, gs, dt)[:, :K].reshape(Cout, k, k, Cg)
    xt = torch.from_numpy(u16_to_f64(x, dt)).permute(0, 3, 1, 2)
    wt_t = torch.from_numpy(What).permute(0, 3, 1, 2)
    ref = torch.nn.functional.conv2d(xt, wt_t, stride=stride, padding=pad, groups=groups)
    ref = ref.permute(0, 2, 3, 1).numpy()
    assert y.shape == ref.shape
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    Ho, Wo = y.shape[1], y.shape[2]
    ms = [0, Ho * Wo - 1, (Ho * Wo) // 2]
    cs = [0, Cout - 1, 3]
    ys, _ = oracle.qconv2d_nhwc(x, wq, s, b, Cout, k, k, (stride, stride), (pad, pad), groups,
                                bits, gs, dt, ms=ms, cos=cs)
    assert np.array_equal(ys, y.reshape(-1, Cout)[ms, cs])


def test_oracle_rejects_bad_arguments():
    w = np.zeros((2, 64), np.uint16)
    with pytest.raises(ValueError):
        oracle.quantize(w, 7, 64, F16)
    with pytest.raises(ValueError):
        oracle.quantize(w, 4, 16, F16)
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros((2, 96), np.uint16), 4, 64, F16)


# ---------------------------------------------------------------- FP4 quantizer
# The steps of the FP4 quantize-dequantize in "mlx 1.0.0, .../quantized.cpp"
# (to_fp8_e8m0, to_fp4_e2m1, fp_quantize_dequantize): pinned against brute
# force over the FP4 value table, exact log2 arithmetic and torch's own
# float8_e4m3fn conversion.

def _fp4_magnitudes():
    return [oracle.e2m1(c) for c in range(8)]          # the table pinned above


def test_e2m1_encode_is_the_nearest_value_ties_to_even():
    """to_fp4_e2m1's thresholds: every |x| maps to the nearest table value;
    at a midpoint, to the one with an even mantissa bit (code bit 0 = 0)."""
    mags = _fp4_magnitudes()
    xs = np.concatenate([np.linspace(0.0, 7.0, 7001), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]])
    for x in xs:
        x = float(np.float32(x))
        d = [abs(x - v) for v in mags]
        best = min(d)
        cand = [c for c in range(8) if d[c] == best]
        want = cand[0] if len(cand) == 1 else [c for c in cand if c % 2 == 0][0]
        assert oracle.e2m1_encode(x) == want, x
        assert oracle.e2m1_encode(-x) == want | 8, -x
    assert oracle.e2m1_encode(float("nan")) == 7            # the page's NaN rule
    assert oracle.e2m1_encode(100.0) == 7                   # saturates at 6


def test_e8m0_encode_is_the_nearest_power_of_two_in_log_scale():
    rng = np.random.default_rng(0)
    xs = np.concatenate([2.0 ** np.arange(-126, 128, dtype=np.float64),
                         rng.uniform(0.5, 2.0, 4000) * 2.0 ** rng.integers(-120, 120, 4000)])
    for x in xs.astype(np.float32):
        x = float(x)
        # exact: log2(x) rounds up past k + 0.5 iff x >= 2^k * sqrt(2), i.e. x^2 >= 2^(2k+1)
        k = math.floor(math.log2(x))
        while 2.0 ** k > x:
            k -= 1
        while 2.0 ** (k + 1) <= x:
            k += 1
        n = k + 1 if x * x >= 2.0 ** (2 * k + 1) else k
        n = max(-127, min(127, n))
        assert oracle.e8m0_encode(x) == n + 127, x
    # around sqrt(2): the last float below rounds down, the first above rounds up
    lo = float(np.float32(1.4142135))
    hi = float(np.nextafter(np.float32(lo), np.float32(2.0)))
    assert lo * lo < 2.0 < hi * hi
    assert oracle.e8m0_encode(lo) == 127 and oracle.e8m0_encode(hi) == 128
    assert oracle.e8m0_encode(0.0) == 0                     # log2(0) = -inf, clamped
    assert oracle.e8m0_encode(float("inf")) == 255 and oracle.e8m0_encode(float("nan")) == 255
    assert oracle.e8m0_encode(3.0e38) == 254                # clamped to 127


def test_e4m3_encode_matches_torch_float8():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(1)
    xs = np.concatenate([np.linspace(0.0, 448.0, 20001),
                         rng.uniform(0.0, 1.0, 4000) * 2.0 ** rng.integers(-12, 9, 4000)])
    xs = xs[xs <= 448.0].astype(np.float32)
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in xs], np.uint8)
    assert np.array_equal(got, want)
    # the reading past the largest finite value: saturation (the scale is >= 0)
    assert oracle.e4m3_encode(449.0) == 0x7E and oracle.e4m3_encode(float("inf")) == 0x7E
    assert oracle.e4m3_encode(float("nan")) == 0x7F


@pytest.mark.parametrize("gs", [16, 32])
def test_quantize_fp4_recovers_table_multiples(gs):
    """A group whose largest magnitude is 6 * 2^k: the scale is 2^k (exact in
    both scale formats for the k used), and every element that is a table
    value times 2^k comes back as its own code."""
    rng = np.random.default_rng(gs)
    mags = _fp4_magnitudes()
    for dt in (0, 1):
        for k in (-3, 0, 2):
            codes = rng.integers(0, 16, gs)
            codes[0] = 7                                     # the group's max: 6 * 2^k
            vals = np.array([(-1.0 if c & 8 else 1.0) * mags[c & 7] * 2.0 ** k for c in codes])
            w16 = np.array([[oracle.round_to_t(v, dt) for v in vals]], np.uint16)
            q, s = oracle.quantize_fp4(w16, gs, dt)
            assert s[0, 0] == (oracle.e4m3_encode(2.0 ** k) if gs == 16 else 127 + k)
            got = np.stack([q[0] & 15, q[0] >> 4], axis=1).reshape(-1)
            # -0 (code 8) encodes as sign 8 | 0 only when the value is -0.0
            want = np.where((codes & 7) == 0, np.where(np.signbit(vals), 8, 0), codes)
            assert np.array_equal(got, want), (dt, k, got, want)


@pytest.mark.parametrize("gs", [16, 32])
def test_quantize_fp4_is_nearest_on_the_scaled_table(gs):
    """Random groups: the scale byte encodes absmax / 6, and each code is the
    table value nearest to w / s (ties to even), with s the decoded scale."""
    rng = np.random.default_rng(10 + gs)
    mags = np.array(_fp4_magnitudes())
    w = (rng.standard_normal((8, 4 * gs)) * 0.05).astype(np.float32)
    w16 = np.array([[oracle.round_to_t(float(v), 1) for v in row] for row in w], np.uint16)
    q, s = oracle.quantize_fp4(w16, gs, 1)
    for n in range(8):
        for g in range(4):
            wg = np.array([oracle.t_to_double(h, 1) for h in w16[n, g * gs:(g + 1) * gs]])
            amax = np.float32(np.max(np.abs(wg)))
            sc = np.float32(amax / np.float32(6.0))
            enc = oracle.e4m3_encode(float(sc)) if gs == 16 else oracle.e8m0_encode(float(sc))
            assert s[n, g] == enc
            sd = oracle.e4m3(enc) if gs == 16 else oracle.e8m0(enc)
            for j in range(gs):
                k = g * gs + j
                c = (q[n, k // 2] >> (4 * (k % 2))) & 15
                x = float(np.float32(wg[j]) / np.float32(sd))
                d = np.abs(abs(x) - mags)
                best = np.flatnonzero(d == d.min())
                want = best[0] if len(best) == 1 else best[best % 2 == 0][0]
                assert (c & 7) == want, (n, g, j, x)
                assert (c >> 3) == (1 if np.signbit(x) else 0)


def test_quantize_fp4_zero_group():
    q, s = oracle.quantize_fp4(np.zeros((2, 64), np.uint16), 32, 1)
    assert not q.any() and not s.any()


# ------------------------------------------- activation fake quantization (QQMatmul)

@pytest.mark.parametrize("dt", [0, 1])
@pytest.mark.parametrize("gs", [16, 32])
def test_fake_quant_fp4_is_the_dequantized_fp4_codes(dt, gs):
    """bits 4: fp_quantize_dequantize's output is the FP4 quantizer's codes
    times the decoded scale (both pinned above), cast once to T."""
    rng = np.random.default_rng(dt * 7 + gs)
    N, K = 6, 8 * gs
    w = rng.standard_normal((N, K)) * np.exp(rng.standard_normal((N, 1)))
    w16 = f64_to_u16(w, dt)
    xh = oracle.quantize_dequantize_fp(w16, 4, gs, dt)
    q, s = oracle.quantize_fp4(w16, gs, dt)
    _, wt = oracle.dequantize(q, s, None, N, K, 4, gs, FP4, dt)
    assert np.array_equal(xh, wt)


@pytest.mark.parametrize("gs", [16, 32])
def test_fake_quant_fp8_elements_match_torch_float8(gs):
    """bits 8: each element is s * E4M3(w / s).  Groups whose absmax is
    448 * 2^k have s = 2^k exactly in both scale formats, so w / s is exact
    and torch's float8_e4m3fn conversion (round to nearest even) gives the
    element."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(gs)
    rows = []
    for k in (-3, 0, 2):
        for _ in range(2):
            v = rng.uniform(-1.0, 1.0, gs) * 448.0
            v[rng.integers(0, gs)] = 448.0 * (1 if rng.integers(0, 2) else -1)
            rows.append(v * 2.0 ** k)
    w16 = f64_to_u16(np.array(rows), BF16)
    out = oracle.quantize_dequantize_fp(w16, 8, gs, BF16)
    w = u16_to_f64(w16, BF16)
    for i, k in enumerate([k for k in (-3, 0, 2) for _ in range(2)]):
        e = torch.from_numpy((w[i] / 2.0 ** k).astype(np.float32))
        v = e.to(torch.float8_e4m3fn).to(torch.float64).numpy() * 2.0 ** k
        assert np.array_equal(u16_to_f64(out[i], BF16), v), i


def test_fake_quant_special_groups():
    """A zero group stays zero; a NaN element is ignored by absmax and comes
    out as the code-7 value 6 s for E2M1 (the page's NaN rule) and NaN for
    E4M3."""
    z = oracle.quantize_dequantize_fp(np.zeros((1, 32), np.uint16), 4, 32, BF16)
    assert not z.any()
    w = np.ones((1, 32)) * 3.0
    w16 = f64_to_u16(w, BF16)
    w16[0, 5] = 0x7FC0                                     # bf16 NaN
    out4 = u16_to_f64(oracle.quantize_dequantize_fp(w16, 4, 32, BF16), BF16)[0]
    # absmax 3 -> scale 0.5 -> E8M0 2^-1; 3 / 0.5 = 6 -> 6 * 0.5 = 3
    assert out4[5] == 3.0 and np.all(np.delete(out4, 5) == 3.0)
    out8 = u16_to_f64(oracle.quantize_dequantize_fp(w16, 8, 32, BF16), BF16)[0]
    assert np.isnan(out8[5]) and np.all(np.delete(out8, 5) == 3.0)


def test_qqmm_is_qmm_over_fake_quantized_x():
    rng = np.random.default_rng(5)
    M, N, K, gs = 2, 8, 128, 32
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    wq = np_pack(codes, 4)
    sc = rng.integers(120, 134, size=(N, K // gs)).astype(np.uint8)
    x16 = f64_to_u16(rng.standard_normal((M, K)), BF16)
    y, _ = oracle.qqmm(x16, wq, sc, N, gs, BF16)
    xh = u16_to_f64(oracle.quantize_dequantize_fp(x16, 4, gs, BF16), BF16)
    lut = np.array([float(v) for _, v in _golden_rows("fp4_e2m1_lut.txt")])
    W = lut[codes] * np.repeat(np.ldexp(1.0, sc.astype(np.int64) - 127), gs, axis=1)
    assert np.allclose(y, xh @ W.T, rtol=1e-12, atol=0)


# ---------------------------------------------------------------- gather qmm

def test_gather_qmm_selects_x_batch_and_weight_by_index():
    """Pair i is x[lhs[i]] times the transpose of dequant(w[rhs[i]]), checked
    against numpy on weights dequantized per expert; x batches and experts
    differ in count and content, so swapped or ignored indices fail."""
    rng = np.random.default_rng(11)
    Bx, E, M, N, K, gs = 3, 4, 2, 8, 128, 64
    x16 = f64_to_u16(rng.standard_normal((Bx, M, K)), BF16)
    wq, sc, bi, W = [], [], [], []
    for e in range(E):
        w16 = f64_to_u16(rng.standard_normal((N, K)) * (e + 1), BF16)
        q, s, b = oracle.quantize(w16, 4, gs, BF16)
        wh, _ = oracle.dequantize(q, s, b, N, K, 4, gs, AFFINE, BF16)
        wq.append(q); sc.append(s); bi.append(b); W.append(wh)
    lhs = [2, 0, 1, 2, 0]
    rhs = [1, 3, 3, 0, 2]
    y, _ = oracle.gather_qmm(x16, np.stack(wq), np.stack(sc), np.stack(bi), lhs, rhs, N, 4, gs,
                             AFFINE, BF16)
    x = u16_to_f64(x16, BF16)
    for i, (l, r) in enumerate(zip(lhs, rhs)):
        assert np.allclose(y[i], x[l] @ W[r].T, rtol=1e-12, atol=1e-12), i


# ------------------------------------------------------- non-transposed qmm

@pytest.mark.parametrize("bits", [3, 4])
def test_qmm_nt_is_x_times_w_hat_by_brute_force(bits):
    """y[m, k] = sum_n x[m, n] (s[n, k/gs] q[n, k] + b[n, k/gs]), summed by
    plain loops over codes unpacked with the numpy packer (not the oracle's
    dequantize); a transposed operand or a group index along the wrong axis
    fails."""
    rng = np.random.default_rng(bits)
    M, N, K, gs = 2, 5, 64, 32
    codes = rng.integers(0, 2 ** bits, size=(N, K)).astype(np.uint8)
    wq = np_pack(codes, bits)
    s16 = f64_to_u16(rng.standard_normal((N, K // gs)) * 0.1, BF16)
    b16 = f64_to_u16(rng.standard_normal((N, K // gs)) * 0.1, BF16)
    x16 = f64_to_u16(rng.standard_normal((M, N)), BF16)
    y, den = oracle.qmm_nt(x16, wq, s16, b16, K, bits, gs, AFFINE, BF16)
    assert y.shape == (M, K)
    s, b, x = u16_to_f64(s16, BF16), u16_to_f64(b16, BF16), u16_to_f64(x16, BF16)
    q = np_unpack(wq, N, K, bits)
    for m in range(M):
        for k in range(K):
            want = sum(x[m, n] * (s[n, k // gs] * q[n, k] + b[n, k // gs]) for n in range(N))
            assert abs(y[m, k] - want) <= 1e-12 * (1 + abs(want)), (m, k)


# ------------------------------------------------------------------- MXFP8

def test_mxfp8_dequantize_is_e4m3_times_e8m0():
    """Every E4M3 byte under several E8M0 scales: the value torch's
    float8_e4m3fn decode gives, times 2^(s - 127) (the scale as bf16)."""
    N, K = 4, 256
    codes = np.tile(np.arange(256, dtype=np.uint8), (N, 1))
    sc = np.array([[127, 120, 131, 127, 100, 140, 127, 127]] * N, np.uint8)
    wh, _ = oracle.dequantize(codes, sc, None, N, K, 8, 32, oracle.MXFP8, BF16)
    dec = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    want = dec * np.repeat(np.ldexp(1.0, sc.astype(np.int64) - 127), 32, axis=1)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(wh), nan)
    assert np.array_equal(wh[~nan], want[~nan])


def test_mxfp8_quantize_codes_match_torch_float8():
    """Groups whose absmax is 448 * 2^k: the scale byte is 127 + k and every
    code is torch's float8_e4m3fn encoding (round to nearest even) of w / 2^k."""
    rng = np.random.default_rng(8)
    rows, ks = [], []
    for k in (-4, 0, 3):
        v = rng.uniform(-1.0, 1.0, 64) * 448.0
        v[0], v[40] = 448.0, -448.0
        rows.append(v * 2.0 ** k)
        ks.append(k)
    w16 = f64_to_u16(np.array(rows), BF16)
    codes, sc = oracle.quantize_mxfp8(w16, BF16)
    w = u16_to_f64(w16, BF16)
    for i, k in enumerate(ks):
        assert list(sc[i]) == [127 + k, 127 + k]
        want = torch.from_numpy((w[i] / 2.0 ** k).astype(np.float32)).to(
            torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(codes[i], want), i


def test_mxfp8_qmm_is_x_times_w_hat():
    rng = np.random.default_rng(9)
    M, N, K = 3, 6, 128
    codes = rng.integers(0, 0x7E, size=(N, K)).astype(np.uint8)   # finite E4M3 bytes
    sc = rng.integers(118, 136, size=(N, K // 32)).astype(np.uint8)
    x16 = f64_to_u16(rng.standard_normal((M, K)), BF16)
    y, _ = oracle.qmm(x16, codes, sc, None, N, 8, 32, oracle.MXFP8, BF16)
    dec = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    W = dec * np.repeat(np.ldexp(1.0, sc.astype(np.int64) - 127), 32, axis=1)
    assert np.allclose(y, u16_to_f64(x16, BF16) @ W.T, rtol=1e-12, atol=1e-12)


def test_mxfp8_mode_rules():
    with pytest.raises(Exception):
        oracle.dequantize(np.zeros((1, 64), np.uint8), np.zeros((1, 4), np.uint8), None, 1, 64, 8,
                          16, oracle.MXFP8, BF16)                  # group 32 only
