// common.cuh — shared device helpers of the CUDA library (not of the oracle).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/aq.h"

namespace aq {

// ----------------------------------------------------------------- T traits
template <typename T> struct TT;
template <> struct TT<__half> {
  static __device__ __forceinline__ float to_f(__half v) { return __half2float(v); }
  static __device__ __forceinline__ __half from_f(float v) { return __float2half_rn(v); }
  static __device__ __forceinline__ __half from_u(unsigned v) { return __uint2half_rn(v); }
};
template <> struct TT<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_u(unsigned v) { return __uint2bfloat16_rn(v); }
};

// ----------------------------------------------------------- FP4 and scales
// E2M1 value of a 4-bit code: sign bit 3, exponent bits 2..1 (bias 1),
// mantissa bit 0; exponent 0 is the subnormal 0.5 * m.
__device__ __forceinline__ float e2m1_to_float(unsigned c) {
  const unsigned e = (c >> 1) & 3u, m = c & 1u;
  unsigned bits = e ? (((e + 126u) << 23) | (m << 22)) : (m ? 0x3F000000u : 0u);
  bits |= (c & 8u) << 28;
  return __uint_as_float(bits);
}

// E8M0 group-32 scale: 2^(s - 127); 255 is +inf (bf16 pattern s << 7).
__device__ __forceinline__ float e8m0_to_float(unsigned s) {
  if (s == 0) return __uint_as_float(0x00400000u);          // 2^-127, fp32 subnormal
  return __uint_as_float(s << 23);                          // s = 255 -> +inf
}

// OCP FP8 E4M3FN: bias 7, S.1111.111 is NaN, no infinities.
__device__ __forceinline__ float e4m3_to_float(unsigned b) {
  const unsigned s = (b >> 7) & 1u, e = (b >> 3) & 15u, m = b & 7u;
  float v;
  if (e == 15u && m == 7u) v = __uint_as_float(0x7FC00000u);
  else if (e == 0u) v = (float)m * 0.001953125f;            // m * 2^-9, exact
  else v = __uint_as_float(((e + 120u) << 23) | (m << 20));
  return s ? -v : v;
}

// The FP4 group scale as T (the value the matmul multiplies by).
template <typename T>
__device__ __forceinline__ float fp4_scale_t(unsigned s, int gs) {
  const float v = gs == 16 ? e4m3_to_float(s) : e8m0_to_float(s);
  return TT<T>::to_f(TT<T>::from_f(v));
}

// Code `c` (compile-time index) out of a register array of 32-bit words that
// holds consecutive codes of BITS bits as a little-endian bit stream.
template <int BITS, int C, int NW>
__device__ __forceinline__ unsigned code_at(const uint32_t (&w)[NW]) {
  constexpr int bit = C * BITS;
  constexpr int word = bit >> 5;
  constexpr int sh = bit & 31;
  constexpr unsigned mask = (1u << BITS) - 1u;
  if constexpr (sh + BITS <= 32) {
    return (w[word] >> sh) & mask;
  } else {
    return __funnelshift_r(w[word], w[word + 1], sh) & mask;
  }
}

// Exact small-integer to float: OR the code into the mantissa of 2^23 and
// subtract 2^23 (valid for codes below 2^23).
__device__ __forceinline__ float u_to_f_exact(unsigned q) {
  return __uint_as_float(0x4B000000u | q) - 8388608.0f;
}

}  // namespace aq

// Sizes the kernels and their host planning share.
namespace aq {
constexpr int64_t kMaxRowsDec = (int64_t)1 << 24;      // N and K limit of the decode kernel
constexpr int64_t kDecUnitBytes = 128 * 1024;          // packed bytes per unit, batched launches
// aq_qmv_noalloc's fixed scratch (a file-scope device array in qmv_mma.cu).
constexpr size_t kQmvNoallocScratchBytes = (size_t)4 << 20;
struct QmvProblemDesc {
  const void* x;
  const void* w_q;
  const void* scales;
  const void* biases;
  void* y;
  int64_t N, K;
};
}  // namespace aq

// Host-side launchers and plans (declarations only).
#include "launch.h"
