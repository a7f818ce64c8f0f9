// aq_oracle.cpp — the CPU oracle for group-wise affine quantized matmul.
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously-correct
// statement of what the library computes.  Only the test suite, the smoke
// check and the benchmark's CPU-baseline leg may load it.  It shares no code,
// header, table or helper with the CUDA library, and the CUDA library never
// calls it.
//
// Sources (web pages, cited by title and section):
//   [P1] "[Feature] Quantized Convolution 2D - Possible PR?" (ml-explore/mlx
//        issue 2714): quantize_weights (flatten, pad to a multiple of
//        group_size, quantize per conv group) and img2col (patch order
//        (kh, kw, C), zero padding), then quantized_matmul.
//   [P2] "Add the 3bit packed qmm_t" (packed-quants branch): the
//        quantized_matmul API, y = x @ dequant(w).T with w stored as rows of
//        output features.
//   [P3] "Improvements in the quantizer and dequantization kernel" (mlx PR
//        1061): bias at the edge with the larger magnitude, scale spanning
//        min..max, scale adjusted so that 0 lands on the grid.
//   [P4] "mlx 1.0.0, mlx/backend/cpu/quantized.cpp": the quantize routine
//        (fp32 arithmetic, packing), get_pack_factor / get_bytes_per_pack,
//        extract_bits, FP4_LUT, dequantize_scale (E8M0 / FP8 scales), fp_qmm_t,
//        and the FP4 quantizer's steps: to_fp8_e8m0, to_fp4_e2m1 and
//        fp_quantize_dequantize (scale = absmax / 6, or / 448 for 8-bit
//        elements), which QQMatmul applies to x before the FP4 matmul; the
//        8-bit branch of fp_qmm_t / fp_qmm_dispatch_typed (MXFP8 weights:
//        E4M3 elements, E8M0 scales at group 32).
//
// Precision.  The quantizer runs in fp32, in the order the quantize routine of
// [P4] takes its steps, because its codes, scales and biases are fixed by fp32
// rounding.  Dequantized weights are formed exactly in fp64, and every matmul
// accumulates in fp64.  Build flags: -O2 -ffp-contract=off -fno-fast-math.
//
// Storage of T (fp16 or bf16) is its raw 16-bit pattern (uint16_t).

#include <cmath>
#include <cstdint>
#include <cstring>
#include <cstdlib>
#include <limits>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

enum { DT_F16 = 0, DT_BF16 = 1 };
enum { MODE_AFFINE = 0, MODE_FP4 = 1, MODE_MXFP8 = 2 };

// ---------------------------------------------------------------- T <-> real
// IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits.
// bfloat16:      1 sign, 8 exponent (bias 127), 7 fraction bits.
struct TFormat {
  int frac_bits;   // stored fraction bits
  int exp_bits;
  int bias;
};
const TFormat kF16 = {10, 5, 15};
const TFormat kBF16 = {7, 8, 127};
inline const TFormat& fmt(int dt) { return dt == DT_F16 ? kF16 : kBF16; }

double t_to_double(uint16_t h, int dt) {
  const TFormat& f = fmt(dt);
  int sign = h >> 15;
  int e = (h >> f.frac_bits) & ((1 << f.exp_bits) - 1);
  int m = h & ((1 << f.frac_bits) - 1);
  double v;
  if (e == (1 << f.exp_bits) - 1) {
    v = m ? std::numeric_limits<double>::quiet_NaN()
          : std::numeric_limits<double>::infinity();
  } else if (e == 0) {
    v = std::ldexp((double)m, 1 - f.bias - f.frac_bits);          // subnormal
  } else {
    v = std::ldexp((double)(m | (1 << f.frac_bits)), e - f.bias - f.frac_bits);
  }
  return sign ? -v : v;
}

// Round a real number to the nearest T, ties to even (one rounding).
uint16_t round_to_t(double v, int dt) {
  const TFormat& f = fmt(dt);
  const uint16_t exp_all = (uint16_t)(((1 << f.exp_bits) - 1) << f.frac_bits);
  if (std::isnan(v)) return (uint16_t)(exp_all | (1 << (f.frac_bits - 1)));
  uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  double a = std::fabs(v);
  if (a == 0.0) return sign;
  const int p = f.frac_bits + 1;                 // significand precision
  const int emin = 1 - f.bias;                   // exponent of the smallest normal
  const int emax = f.bias;                       // exponent of the largest finite
  int e;
  std::frexp(a, &e);                             // a = fr * 2^e, fr in [0.5, 1)
  e -= 1;                                        // a in [2^e, 2^(e+1))
  int q = e < emin ? emin : e;                   // quantum exponent range
  double ulp = std::ldexp(1.0, q - p + 1);
  double r = std::nearbyint(a / ulp) * ulp;      // exact scaling, RNE rounding
  double max_finite = std::ldexp(2.0 - std::ldexp(1.0, 1 - p), emax);
  if (r > max_finite) return (uint16_t)(sign | exp_all);   // overflow -> inf
  if (r == 0.0) return sign;
  int re;
  std::frexp(r, &re);
  re -= 1;
  if (re < emin) {                               // subnormal encoding
    uint16_t m = (uint16_t)std::ldexp(r, f.bias - 1 + f.frac_bits);
    return (uint16_t)(sign | m);
  }
  uint16_t m = (uint16_t)(std::ldexp(r, f.frac_bits - re) - std::ldexp(1.0, f.frac_bits));
  uint16_t ebits = (uint16_t)((re + f.bias) << f.frac_bits);
  return (uint16_t)(sign | ebits | m);
}

inline float t_to_float(uint16_t h, int dt) { return (float)t_to_double(h, dt); }

// ------------------------------------------------------------------- packing
// [P4] get_pack_factor / get_bytes_per_pack: power-of-two widths put 32/bits
// codes into one uint32 word; 3- and 5-bit put 8 codes into 3 / 5 bytes and
// 6-bit puts 4 codes into 3 bytes.  In every case code k of a pack occupies
// bits [k*bits, (k+1)*bits) of the pack, stored little-endian.
struct PackShape {
  int codes_per_pack;
  int bytes_per_pack;
};
PackShape pack_shape(int bits) {
  switch (bits) {
    case 2: return {16, 4};
    case 4: return {8, 4};
    case 8: return {4, 4};
    case 3: return {8, 3};
    case 5: return {8, 5};
    case 6: return {4, 3};
    default: return {0, 0};
  }
}
bool valid_bits(int bits) { return pack_shape(bits).codes_per_pack != 0; }
bool valid_group(int gs) { return gs == 32 || gs == 64 || gs == 128; }

// Read code k of one packed row.  The row is a little-endian bit stream in
// which code k starts at bit k*bits (this holds for every width above, since
// packs are whole bytes and codes fill each pack from its low bit upward).
inline unsigned read_code(const uint8_t* row, int64_t k, int bits) {
  int64_t bit = k * bits;
  int64_t byte = bit >> 3;
  int sh = (int)(bit & 7);
  unsigned v = row[byte];
  if (sh + bits > 8) v |= (unsigned)row[byte + 1] << 8;
  return (v >> sh) & ((1u << bits) - 1u);
}

// ---------------------------------------------------------------- FP4 / FP8
// E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.
// E=0: 0.5*M (subnormal); otherwise 2^(E-1) * (1 + M/2).  [P4] FP4_LUT.
double e2m1_value(unsigned code) {
  unsigned s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double v = (e == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, (int)e - 1);
  return s ? -v : v;
}

// E8M0 group-32 scale: [P4] dequantize_scale writes the bf16 pattern
// (s == 0 ? 0x40 : s << 7), i.e. 2^(s-127) for s in 0..254 and +inf for 255.
double e8m0_value(unsigned s) {
  if (s == 255) return std::numeric_limits<double>::infinity();
  return std::ldexp(1.0, (int)s - 127);
}

// E4M3 group-16 scale: [P4] names detail::FromFP8 without its body.  Reading:
// OCP FP8 E4M3FN — bias 7, no infinities, S.1111.111 is NaN, max 448.
double e4m3_value(unsigned b) {
  unsigned s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
  double v;
  if (e == 15 && m == 7) v = std::numeric_limits<double>::quiet_NaN();
  else if (e == 0) v = std::ldexp((double)m / 8.0, -6);
  else v = std::ldexp(1.0 + (double)m / 8.0, (int)e - 7);
  return s ? -v : v;
}

// The scale in T, as [P4] dequantize_scale returns it (static_cast<T>).
double fp_scale_in_t(uint8_t s, int gs, int dt) {
  double v = gs == 16 ? e4m3_value(s) : e8m0_value(s);
  return t_to_double(round_to_t(v, dt), dt);
}

// ------------------------------------------------------- FP4 quantizer
// The steps of [P4] fp_quantize_dequantize for 4-bit codes, up to the codes
// and the scale byte (the library's FP4 weight format), with two readings:
//   * to_fp8_e8m0 takes n = round(log2(x)) in float.  Reading: the exact
//     nearest power of two on a log scale, i.e. x = m * 2^e (m in [1, 2))
//     rounds to 2^(e+1) exactly when m >= sqrt(2) (a float is never equal
//     to sqrt(2), so the tie rule never applies).  x = 0 has log2 = -inf,
//     which the clamp maps to -127.
//   * detail::ToFP8 (the E4M3 scale of group 16) has no body on the pages.
//     Reading: OCP E4M3FN, round to nearest with ties to even, finite values
//     and infinities saturated to +-448, NaN to 0x7F.
unsigned e8m0_encode(float x) {
  if (!std::isfinite(x)) return 0xFF;
  if (x < 0.0f) return 0x00;
  if (x == 0.0f) return 0x00;                    // n = -127
  int e;
  const double fr = std::frexp((double)x, &e);   // x = fr * 2^e, fr in [0.5, 1)
  const double m = 2.0 * fr;                     // x = m * 2^(e-1), m in [1, 2)
  int n = (m * m >= 2.0) ? e : e - 1;            // m >= sqrt(2); m*m is exact in double
  n = n < -127 ? -127 : (n > 127 ? 127 : n);
  return (unsigned)(n + 127);
}

unsigned e4m3_encode(float xf) {
  if (std::isnan(xf)) return 0x7F;
  const unsigned sign = std::signbit(xf) ? 0x80u : 0u;
  const double a = std::fabs((double)xf);
  if (a == 0.0) return sign;
  const double kMax = 448.0;
  if (a > kMax) return sign | 0x7E;              // saturate (infinities too)
  int e;
  std::frexp(a, &e);
  e -= 1;                                        // a in [2^e, 2^(e+1))
  const int q = e < -6 ? -6 : e;                 // below 2^-6: the subnormal quantum
  const double quantum = std::ldexp(1.0, q - 3); // 3 fraction bits
  double r = std::nearbyint(a / quantum) * quantum;   // ties to even (default mode)
  if (r > kMax) r = kMax;
  if (r == 0.0) return sign;
  int re;
  std::frexp(r, &re);
  re -= 1;
  if (re < -6) return sign | (unsigned)std::ldexp(r, 9);          // E = 0: m * 2^-9
  const unsigned m = (unsigned)(std::ldexp(r, 3 - re) - 8.0);
  return sign | ((unsigned)(re + 7) << 3) | m;
}

// [P4] to_fp4_e2m1: the threshold table (round to nearest, ties to even).
unsigned e2m1_encode(float x) {
  if (std::isnan(x)) return 0x7;
  const unsigned sign = std::signbit(x) ? 0x8u : 0u;
  const float a = std::fabs(x);
  unsigned bits;
  if (a > 5.0f) bits = 0x7;
  else if (a >= 3.5f) bits = 0x6;
  else if (a > 2.5f) bits = 0x5;
  else if (a >= 1.75f) bits = 0x4;
  else if (a > 1.25f) bits = 0x3;
  else if (a >= 0.75f) bits = 0x2;
  else if (a > 0.25f) bits = 0x1;
  else bits = 0x0;
  return bits | sign;
}

// ----------------------------------------------------------------- dequant
// One dequantized row: w_hat[k] exactly, in fp64.
//   affine [P4] _qmm_t:      scale * q + bias   (scale, bias are T values)
//   fp4    [P4] fp_qmm_t:    scale * FP4_LUT[q] (no bias)
void dequant_row(const uint8_t* wq, const void* scales, const uint16_t* biases,
                 int64_t n, int64_t K, int bits, int gs, int mode, int dt,
                 double* out) {
  const int64_t G = K / gs;
  if (mode == MODE_AFFINE) {
    const uint8_t* row = wq + n * (K * bits / 8);
    const uint16_t* s = (const uint16_t*)scales + n * G;
    const uint16_t* b = biases + n * G;
    for (int64_t g = 0; g < G; ++g) {
      double sc = t_to_double(s[g], dt), bi = t_to_double(b[g], dt);
      for (int64_t j = 0; j < gs; ++j) {
        int64_t k = g * gs + j;
        out[k] = sc * (double)read_code(row, k, bits) + bi;
      }
    }
  } else if (mode == MODE_FP4) {
    const uint8_t* row = wq + n * (K / 2);
    const uint8_t* s = (const uint8_t*)scales + n * G;
    for (int64_t g = 0; g < G; ++g) {
      double sc = fp_scale_in_t(s[g], gs, dt);
      for (int64_t j = 0; j < gs; ++j) {
        int64_t k = g * gs + j;
        out[k] = e2m1_value(read_code(row, k, 4)) * sc;
      }
    }
  } else {
    // MXFP8 ([P4] fp_qmm_t, bits 8): one E4M3 byte per element (FromFP8) times
    // the group's E8M0 scale as T.
    const uint8_t* row = wq + n * K;
    const uint8_t* s = (const uint8_t*)scales + n * G;
    for (int64_t g = 0; g < G; ++g) {
      double sc = fp_scale_in_t(s[g], gs, dt);
      for (int64_t j = 0; j < gs; ++j) {
        int64_t k = g * gs + j;
        out[k] = e4m3_value(row[k]) * sc;
      }
    }
  }
}

// w_hat rounded once to T: the dequantize operation's output ("Add the 3bit
// packed qmm_t", dequantize returns an array of the scales' type; the
// pages' Metal loader and CPU _qmm_t form scale * w + bias in T before the
// multiply).  Used for the products of kernels that dequantize into T tiles.
void round_row_to_t(double* row, int64_t K, int dt) {
  for (int64_t k = 0; k < K; ++k) row[k] = t_to_double(round_to_t(row[k], dt), dt);
}

int check_common(int64_t N, int64_t K, int bits, int gs, int mode, int dt) {
  if (dt != DT_F16 && dt != DT_BF16) return 1;
  if (N < 0 || K < 0) return 1;
  if (mode == MODE_AFFINE) {
    if (!valid_bits(bits) || !valid_group(gs)) return 1;
  } else if (mode == MODE_FP4) {
    if (bits != 4 || (gs != 16 && gs != 32)) return 1;
  } else if (mode == MODE_MXFP8) {
    if (bits != 8 || gs != 32) return 1;               // [P4] fp_qmm_dispatch_typed: bits 8 -> group 32
  } else {
    return 1;
  }
  if (gs && K % gs) return 1;
  return 0;
}

}  // namespace

extern "C" {

// Threads the oracle's parallel loops use (OpenMP); the timed CPU baseline
// also runs it on one thread.  Changes no result: every output element is
// computed by one thread in the same order either way.
void orc_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

double orc_t_to_double(uint16_t h, int dt) { return t_to_double(h, dt); }
uint16_t orc_round_to_t(double v, int dt) { return round_to_t(v, dt); }
double orc_e2m1(int code) { return e2m1_value((unsigned)code & 15); }
double orc_e8m0(int s) { return e8m0_value((unsigned)s & 255); }
double orc_e4m3(int s) { return e4m3_value((unsigned)s & 255); }
int orc_e8m0_encode(float x) { return (int)e8m0_encode(x); }
int orc_e4m3_encode(float x) { return (int)e4m3_encode(x); }
int orc_e2m1_encode(float x) { return (int)e2m1_encode(x); }

// FP4 quantizer ([P4] fp_quantize_dequantize, 4-bit, up to the codes).  w is
// [N, K] T; codes receives N rows of K/2 bytes (code k in the low nibble of
// byte k/2 when k is even, the high nibble when odd); scales is [N, K/gs]
// bytes: E8M0 for gs = 32, E4M3 for gs = 16.  Per group, in fp32:
//   absmax = max_j |w_j|  (starting from -inf, as std::max does: NaN ignored)
//   scale  = absmax / 6
//   byte   = gs == 16 ? ToFP8(scale) : to_fp8_e8m0(scale)
//   s      = the byte decoded to float (dequantize_scale<float>)
//   code_j = to_fp4_e2m1(s == 0 ? 0 : w_j / s)
int orc_quantize_fp4(const uint16_t* w, int64_t N, int64_t K, int gs, int dt, uint8_t* codes,
                     uint8_t* scales) {
  if (dt != DT_F16 && dt != DT_BF16) return 1;
  if ((gs != 16 && gs != 32) || N < 0 || K < 0 || K % gs) return 1;
  const int64_t G = K / gs;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < G; ++g) {
      const uint16_t* wg = w + n * K + g * gs;
      float amax = -std::numeric_limits<float>::infinity();
      for (int j = 0; j < gs; ++j) {
        const float a = std::fabs(t_to_float(wg[j], dt));
        amax = (amax < a) ? a : amax;            // std::max(amax, a)
      }
      const float scale = amax / 6.0f;
      const unsigned byte = gs == 16 ? e4m3_encode(scale) : e8m0_encode(scale);
      const float sdec = (float)(gs == 16 ? e4m3_value(byte) : e8m0_value(byte));
      scales[n * G + g] = (uint8_t)byte;
      for (int j = 0; j < gs; ++j) {
        const float el = sdec == 0.0f ? 0.0f : t_to_float(wg[j], dt) / sdec;
        const unsigned c = e2m1_encode(el);
        const int64_t k = g * gs + j;
        uint8_t& dst = codes[n * (K / 2) + k / 2];
        if (k % 2 == 0) dst = (uint8_t)((dst & 0xF0) | c);
        else dst = (uint8_t)((dst & 0x0F) | (c << 4));
      }
    }
  }
  return 0;
}

// MXFP8 quantizer: the steps of [P4] fp_quantize_dequantize for 8-bit
// elements up to the codes and the scale byte.  w is [N, K] T; codes is
// [N, K] E4M3 bytes; scales is [N, K/32] E8M0 bytes.  Per group of 32, fp32:
//   absmax (NaN ignored), scale = absmax / 448, byte = to_fp8_e8m0(scale),
//   s = the byte decoded, code_j = ToFP8(s == 0 ? 0 : w_j / s)
int orc_quantize_mxfp8(const uint16_t* w, int64_t N, int64_t K, int dt, uint8_t* codes,
                       uint8_t* scales) {
  if (dt != DT_F16 && dt != DT_BF16) return 1;
  if (N < 0 || K < 0 || K % 32) return 1;
  const int64_t G = K / 32;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < G; ++g) {
      const uint16_t* wg = w + n * K + g * 32;
      float amax = -std::numeric_limits<float>::infinity();
      for (int j = 0; j < 32; ++j) {
        const float a = std::fabs(t_to_float(wg[j], dt));
        amax = (amax < a) ? a : amax;
      }
      const float scale = amax / 448.0f;
      const unsigned byte = e8m0_encode(scale);
      const float sdec = (float)e8m0_value(byte);
      scales[n * G + g] = (uint8_t)byte;
      for (int j = 0; j < 32; ++j) {
        const float el = sdec == 0.0f ? 0.0f : t_to_float(wg[j], dt) / sdec;
        codes[n * K + g * 32 + j] = (uint8_t)e4m3_encode(el);
      }
    }
  }
  return 0;
}

// Fake quantization of activations, the other use of [P4]
// fp_quantize_dequantize (QQMatmul quantizes x with it before the FP4
// matmul).  w is [N, K] T; out is [N, K] T.  Per group, in fp32:
//   absmax = max_j |w_j|  (NaN ignored, as above)
//   scale  = absmax / (bits == 4 ? 6 : 448)
//   s      = the scale byte decoded to float (E4M3 for gs = 16, E8M0 for 32)
//   e_j    = s == 0 ? 0 : w_j / s
//   v_j    = bits == 4 ? the E2M1 table value of to_fp4_e2m1(e_j)
//                      : the E4M3 value of ToFP8(e_j)  (FromFP8 o ToFP8)
//   out_j  = T(s * v_j)   (one fp32 multiplication, then the cast to T)
int orc_quantize_dequantize_fp(const uint16_t* w, int64_t N, int64_t K, int bits, int gs, int dt,
                               uint16_t* out) {
  if (dt != DT_F16 && dt != DT_BF16) return 1;
  if ((bits != 4 && bits != 8) || (gs != 16 && gs != 32) || N < 0 || K < 0 || K % gs) return 1;
  const float div = bits == 4 ? 6.0f : 448.0f;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < K / gs; ++g) {
      const uint16_t* wg = w + n * K + g * gs;
      float amax = -std::numeric_limits<float>::infinity();
      for (int j = 0; j < gs; ++j) {
        const float a = std::fabs(t_to_float(wg[j], dt));
        amax = (amax < a) ? a : amax;
      }
      const float scale = amax / div;
      const float sdec = (float)(gs == 16 ? e4m3_value(e4m3_encode(scale))
                                          : e8m0_value(e8m0_encode(scale)));
      for (int j = 0; j < gs; ++j) {
        const float el = sdec == 0.0f ? 0.0f : t_to_float(wg[j], dt) / sdec;
        const float v = (float)(bits == 4 ? e2m1_value(e2m1_encode(el))
                                          : e4m3_value(e4m3_encode(el)));
        const float prod = sdec * v;
        out[n * K + g * gs + j] = round_to_t((double)prod, dt);
      }
    }
  }
  return 0;
}

// Affine quantizer, [P4] quantize and [P3] item 1.  w is [N, K] T row-major;
// w_q receives N rows of K*bits/8 bytes; scales/biases are [N, K/gs] T.
// Per group, in fp32:
//   lo, hi         = min, max of the group
//   at_min         = |lo| > |hi|
//   scale          = max((hi - lo) / (2^bits - 1), 1e-7), negated unless at_min
//   edge           = at_min ? lo : hi
//   q0             = rint(edge / scale)
//   if q0 != 0:      scale = edge / q0, bias = edge    (0 lands on code -q0)
//   else:            bias = 0
//   code           = clamp(rint((w - bias) / scale), 0, 2^bits - 1)
//   stored         = T(scale), T(bias)
int orc_quantize(const uint16_t* w, int64_t N, int64_t K, int bits, int gs, int dt,
                 uint8_t* w_q, uint16_t* scales, uint16_t* biases) {
  if (check_common(N, K, bits, gs, MODE_AFFINE, dt)) return 1;
  const PackShape ps = pack_shape(bits);
  const float n_bins = (float)((1 << bits) - 1);
  const float eps = 1e-7f;
  const int64_t G = K / gs;
  const int64_t row_bytes = K * bits / 8;
  std::vector<float> codes((size_t)gs);
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < G; ++g) {
      const uint16_t* grp = w + n * K + g * gs;
      float lo = std::numeric_limits<float>::infinity();
      float hi = -lo;
      for (int j = 0; j < gs; ++j) {
        float v = t_to_float(grp[j], dt);
        hi = std::max(hi, v);
        lo = std::min(lo, v);
      }
      const bool at_min = std::fabs(lo) > std::fabs(hi);
      float scale = std::max((hi - lo) / n_bins, eps);
      if (!at_min) scale = -scale;
      const float edge = at_min ? lo : hi;
      const float q0 = std::rint(edge / scale);
      float bias = 0.0f;
      if (q0 != 0.0f) {
        scale = edge / q0;
        bias = edge;
      }
      for (int j = 0; j < gs; ++j) {
        float c = std::rint((t_to_float(grp[j], dt) - bias) / scale);
        codes[(size_t)j] = std::min(std::max(c, 0.0f), n_bins);
      }
      // Pack: each pack gathers codes_per_pack codes at shifts k*bits, and is
      // written out as bytes_per_pack little-endian bytes.
      uint8_t* out = w_q + n * row_bytes + g * (int64_t)gs * bits / 8;
      const int packs = gs / ps.codes_per_pack;
      for (int p = 0; p < packs; ++p) {
        uint64_t acc = 0;
        for (int k = 0; k < ps.codes_per_pack; ++k)
          acc |= (uint64_t)codes[(size_t)(p * ps.codes_per_pack + k)] << (k * bits);
        for (int byte = 0; byte < ps.bytes_per_pack; ++byte)
          out[p * ps.bytes_per_pack + byte] = (uint8_t)(acc >> (8 * byte));
      }
      scales[n * G + g] = round_to_t((double)scale, dt);
      biases[n * G + g] = round_to_t((double)bias, dt);
    }
  }
  return 0;
}

// Integer codes of a packed matrix: codes[N*K] (one byte per code).
int orc_unpack(const uint8_t* w_q, int64_t N, int64_t K, int bits, uint8_t* codes) {
  if (!valid_bits(bits) || N < 0 || K < 0 || (K * bits) % 8) return 1;
  const int64_t row_bytes = K * bits / 8;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      codes[n * K + k] = (uint8_t)read_code(w_q + n * row_bytes, k, bits);
  return 0;
}

// Dequantize: w_hat (fp64, exact; may be NULL) and w_t = T(w_hat) rounded once
// (may be NULL).  mode 0 = affine (biases required), 1 = FP4 (u8 scales).
int orc_dequantize(const uint8_t* w_q, const void* scales, const uint16_t* biases,
                   int64_t N, int64_t K, int bits, int gs, int mode, int dt,
                   double* w_hat, uint16_t* w_t) {
  if (check_common(N, K, bits, gs, mode, dt)) return 1;
  std::vector<double> row((size_t)K);
  for (int64_t n = 0; n < N; ++n) {
    dequant_row(w_q, scales, biases, n, K, bits, gs, mode, dt, row.data());
    for (int64_t k = 0; k < K; ++k) {
      if (w_hat) w_hat[n * K + k] = row[(size_t)k];
      if (w_t) w_t[n * K + k] = round_to_t(row[(size_t)k], dt);
    }
  }
  return 0;
}

// y = x . w_hat^T in fp64 ([P2] quantized_matmul with transpose=true), and
// den = sum_k |x[m,k] * w_hat[n,k]| for the error bound.  With w_in_t the
// product uses w_hat rounded once to T (see round_row_to_t).  x is [M, K] T;
// y, den are [M, N] doubles.  The outer loop over n may run on several
// threads; each output is one sequential fp64 sum over k.
int orc_qmm(const uint16_t* x, const uint8_t* w_q, const void* scales,
            const uint16_t* biases, int64_t M, int64_t N, int64_t K, int bits,
            int gs, int mode, int dt, int w_in_t, double* y, double* den) {
  if (check_common(N, K, bits, gs, mode, dt) || M < 0) return 1;
  std::vector<double> xd((size_t)(M * K));
  for (int64_t i = 0; i < M * K; ++i) xd[(size_t)i] = t_to_double(x[i], dt);
#pragma omp parallel
  {
    std::vector<double> row((size_t)K);
#pragma omp for schedule(dynamic, 4)
    for (int64_t n = 0; n < N; ++n) {
      dequant_row(w_q, scales, biases, n, K, bits, gs, mode, dt, row.data());
      if (w_in_t) round_row_to_t(row.data(), K, dt);
      for (int64_t m = 0; m < M; ++m) {
        const double* xr = xd.data() + m * K;
        double acc = 0.0, mag = 0.0;
        for (int64_t k = 0; k < K; ++k) {
          double p = xr[k] * row[(size_t)k];
          acc += p;
          mag += std::fabs(p);
        }
        y[m * N + n] = acc;
        if (den) den[m * N + n] = mag;
      }
    }
  }
  return 0;
}

// The same products at `count` sampled (m, n) positions only.
int orc_qmm_sampled(const uint16_t* x, const uint8_t* w_q, const void* scales,
                    const uint16_t* biases, int64_t M, int64_t N, int64_t K, int bits,
                    int gs, int mode, int dt, int w_in_t, const int64_t* ms,
                    const int64_t* ns, int64_t count, double* y, double* den) {
  if (check_common(N, K, bits, gs, mode, dt) || M < 0) return 1;
  std::vector<double> row((size_t)K);
  for (int64_t i = 0; i < count; ++i) {
    if (ms[i] < 0 || ms[i] >= M || ns[i] < 0 || ns[i] >= N) return 1;
    dequant_row(w_q, scales, biases, ns[i], K, bits, gs, mode, dt, row.data());
    if (w_in_t) round_row_to_t(row.data(), K, dt);
    double acc = 0.0, mag = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      double p = t_to_double(x[ms[i] * K + k], dt) * row[(size_t)k];
      acc += p;
      mag += std::fabs(p);
    }
    y[i] = acc;
    if (den) den[i] = mag;
  }
  return 0;
}

// Quantized conv2d, NHWC, by explicit im2col ([P1] img2col + quantized_matmul).
//   x: [B, H, W, Cin] T.  Conv group g (of `groups`) reads input channels
//   [g*Cg, (g+1)*Cg) with Cg = Cin/groups and writes output channels
//   [g*Ng, (g+1)*Ng) with Ng = Cout/groups.
//   Weight row co is the flattened (kh, kw, Cg) filter, zero-padded to Kp (a
//   multiple of gs) before quantizing; w_q is [Cout, Kp*bits/8] bytes and
//   scales/biases are [Cout, Kp/gs].
//   im2col row for output (b, ho, wo): column (i*kw + j)*Cg + c holds
//   x[b, ho*sh - ph + i, wo*sw - pw + j, g*Cg + c], zero outside the image
//   and in the columns K..Kp-1.
//   y: [B, Ho, Wo, Cout] doubles (and den likewise).
// When ms/cos are non-NULL only the `count` sampled (m, co) outputs are
// computed into y[i], den[i] (m = (b*Ho + ho)*Wo + wo).
int orc_qconv2d_nhwc(const uint16_t* x, const uint8_t* w_q, const uint16_t* scales,
                     const uint16_t* biases, int B, int H, int W, int Cin, int Cout,
                     int kh, int kw, int sh, int sw, int ph, int pw, int groups,
                     int bits, int gs, int dt, int w_in_t, const int64_t* ms,
                     const int64_t* cos, int64_t count, double* y, double* den) {
  if (groups <= 0 || Cin % groups || Cout % groups || kh <= 0 || kw <= 0 ||
      sh <= 0 || sw <= 0 || ph < 0 || pw < 0 || B < 0 || H < 0 || W < 0)
    return 1;
  const int Cg = Cin / groups, Ng = Cout / groups;
  const int64_t K = (int64_t)kh * kw * Cg;
  const int64_t Kp = (K + gs - 1) / gs * gs;
  if (check_common(Cout, Kp, bits, gs, MODE_AFFINE, dt)) return 1;
  const int Ho = (H + 2 * ph - kh) / sh + 1, Wo = (W + 2 * pw - kw) / sw + 1;
  if (Ho <= 0 || Wo <= 0) return 1;
  const int64_t Mtot = (int64_t)B * Ho * Wo;

  auto im2col_row = [&](int64_t m, int g, double* a) {
    const int64_t b = m / ((int64_t)Ho * Wo);
    const int ho = (int)((m / Wo) % Ho), wo = (int)(m % Wo);
    for (int64_t k = 0; k < Kp; ++k) a[k] = 0.0;
    for (int i = 0; i < kh; ++i)
      for (int j = 0; j < kw; ++j) {
        const int hi = ho * sh - ph + i, wi = wo * sw - pw + j;
        if (hi < 0 || hi >= H || wi < 0 || wi >= W) continue;
        for (int c = 0; c < Cg; ++c)
          a[((int64_t)i * kw + j) * Cg + c] =
              t_to_double(x[(((int64_t)b * H + hi) * W + wi) * Cin + (int64_t)g * Cg + c], dt);
      }
  };

  if (ms) {
    std::vector<double> a((size_t)Kp), wrow((size_t)Kp);
    for (int64_t i = 0; i < count; ++i) {
      if (ms[i] < 0 || ms[i] >= Mtot || cos[i] < 0 || cos[i] >= Cout) return 1;
      const int g = (int)(cos[i] / Ng);
      im2col_row(ms[i], g, a.data());
      dequant_row(w_q, scales, biases, cos[i], Kp, bits, gs, MODE_AFFINE, dt, wrow.data());
      if (w_in_t) round_row_to_t(wrow.data(), Kp, dt);
      double acc = 0.0, mag = 0.0;
      for (int64_t k = 0; k < Kp; ++k) {
        double p = a[(size_t)k] * wrow[(size_t)k];
        acc += p;
        mag += std::fabs(p);
      }
      y[i] = acc;
      if (den) den[i] = mag;
    }
    return 0;
  }

  // Full output: materialise the im2col matrix per conv group, then the
  // matmul of each output channel of that group against it.
  std::vector<double> A((size_t)(Mtot * Kp));
  std::vector<double> wrow((size_t)Kp);
  for (int g = 0; g < groups; ++g) {
    for (int64_t m = 0; m < Mtot; ++m) im2col_row(m, g, A.data() + m * Kp);
    for (int n = 0; n < Ng; ++n) {
      const int co = g * Ng + n;
      dequant_row(w_q, scales, biases, co, Kp, bits, gs, MODE_AFFINE, dt, wrow.data());
      if (w_in_t) round_row_to_t(wrow.data(), Kp, dt);
      for (int64_t m = 0; m < Mtot; ++m) {
        const double* a = A.data() + m * Kp;
        double acc = 0.0, mag = 0.0;
        for (int64_t k = 0; k < Kp; ++k) {
          double p = a[k] * wrow[(size_t)k];
          acc += p;
          mag += std::fabs(p);
        }
        y[m * Cout + co] = acc;
        if (den) den[m * Cout + co] = mag;
      }
    }
  }
  return 0;
}

}  // extern "C"
