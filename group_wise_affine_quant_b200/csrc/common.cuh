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

// Launchers implemented in the .cu files; all return cudaSuccess or the
// launch error.
namespace aq {
cudaError_t launch_quantize(const void* w, void* w_q, void* scales, void* biases, int64_t N,
                            int64_t K, int bits, int gs, int dtype, cudaStream_t st);
cudaError_t launch_quantize_fp4(const void* w, void* codes, void* scales, int64_t N, int64_t K,
                                int gs, int dtype, cudaStream_t st);
size_t qmm_nt_workspace(int64_t M, int64_t N, int64_t K);
cudaError_t launch_qmm_nt(const void* x, const void* w_q, const void* scales, const void* biases,
                          void* y, int64_t M, int64_t N, int64_t K, int bits, int gs, int mode,
                          int dtype, void* workspace, cudaStream_t st);
cudaError_t launch_quantize_dequantize_fp(const void* w, void* out, int64_t N, int64_t K, int bits,
                                          int gs, int dtype, cudaStream_t st);
cudaError_t launch_dequantize(const void* w_q, const void* scales, const void* biases,
                              void* w_out, int64_t N, int64_t K, int bits, int gs, int mode,
                              int dtype, cudaStream_t st);

struct QmvPlan {
  int mt;          // compile-time row count the kernel is built for (>= M)
  int64_t ks;      // K-slice per CTA (multiple of 32)
  int splits;      // number of K-slices
  int lpr;         // lanes per weight row
  int rows_cta;    // weight rows per CTA
  int64_t row_blocks;
  int ri;          // row groups per CTA
  int chunk_units; // 32-code units of x staged at a time
  size_t smem;     // dynamic shared memory
  size_t ws_bytes; // workspace bytes (0: the cluster reduction needs none)
};
QmvPlan plan_qmv(int64_t M, int64_t N, int64_t K, int bits, int gs, int mode);
cudaError_t launch_qmv(const QmvPlan& p, const void* x, const void* w_q, const void* scales,
                       const void* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
                       int gs, int mode, int dtype, void* ws, cudaStream_t st);

struct QmmPlan {
  int bt;          // x rows per tile (MMA N)
  int64_t n_tiles; // weight row tiles of 128
  int64_t m_tiles; // x row tiles of bt
  int k_tiles;     // K / 64 rounded up
  int k_tiles_split;
  int splits;      // K-slices, one cluster per output tile
  int64_t tiles_main;     // tiles launched with `splits` slices (the rest: tail)
  int tail_splits;        // K-slices of each remaining tile
  int tail_k_tiles_split;
};
QmmPlan plan_qmm(int64_t M, int64_t N, int64_t K, int bits, int gs, int mode);
cudaError_t launch_qmm(const QmmPlan& p, const void* x, const void* w_q, const void* scales,
                       const void* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
                       int gs, int mode, int dtype, cudaStream_t st);
cudaError_t launch_qconv(const void* x, const void* w_q, const void* scales, const void* biases,
                         void* y, int Bn, int H, int W, int Cin, int Cout, int kh, int kw,
                         int sh, int sw, int ph, int pw, int groups, int bits, int gs, int dtype,
                         cudaStream_t st);
cudaError_t read_device_error_qmm(unsigned* out);
// Tensor-core decode path for 1 <= M <= 16 (qmv_tc.cu): applies when the
// packed rows and the scale rows are 16-byte multiples (TMA chunks) and the
// scales / biases are 16-byte aligned.
constexpr int64_t kMaxRowsDec = (int64_t)1 << 24;      // N and K limit of the decode kernel
constexpr int64_t kDecUnitBytes = 128 * 1024;          // packed bytes per unit, batched launches
struct QmvProblemDesc {
  const void* x;
  const void* w_q;
  const void* scales;
  const void* biases;
  void* y;
  int64_t N, K;
};
bool qmv_tc_shape_ok(int64_t N, int64_t K, int bits, int gs, int mode);
bool qmv_tc_applies(int64_t M, int64_t N, int64_t K, int bits, int gs, int mode,
                    const void* scales, const void* biases);
size_t qmv_tc_workspace(int64_t M, int64_t N, int64_t K, int bits, int gs);
size_t qmv_tc_batched_workspace(const QmvProblemDesc* probs, int count, int64_t M, int bits,
                                int gs);
cudaError_t launch_qmv_tc(const void* x, const void* w_q, const void* scales, const void* biases,
                          void* y, int64_t M, int64_t N, int64_t K, int bits, int gs, int mode,
                          int dtype, void* ws, cudaStream_t st);
cudaError_t launch_qmv_tc_batched(const QmvProblemDesc* probs, int count, int64_t M, int bits,
                                  int gs, int mode, int dtype, void* ws, cudaStream_t st);
cudaError_t read_device_error_qmv_tc(unsigned* out);
// Warp-MMA decode path for 4-bit affine weights (qmv_mma.cu): applies when K
// is a multiple of the sub-slice (512 columns; 1024 for group size 128) and
// the scales / biases are 16-byte aligned.
bool qmv_mma_shape_ok(int64_t N, int64_t K, int bits, int gs, int mode);
bool qmv_mma_applies(int64_t M, int64_t N, int64_t K, int bits, int gs, int mode,
                     const void* scales, const void* biases);
size_t qmv_mma_workspace(int64_t M, int64_t N, int64_t K, int gs);
size_t qmv_mma_batched_workspace(const QmvProblemDesc* probs, int count, int64_t M, int gs);
cudaError_t launch_qmv_mma(const void* x, const void* w_q, const void* scales,
                           const void* biases, void* y, int64_t M, int64_t N, int64_t K, int gs,
                           int dtype, void* ws, cudaStream_t st);
cudaError_t launch_qmv_mma_batched(const QmvProblemDesc* probs, int count, int64_t M, int gs,
                                   int dtype, void* ws, cudaStream_t st);
cudaError_t read_device_error_qmv_mma(unsigned* out);
// Test hooks of the warp-MMA decode kernel (aq_testing.h).
void testing_set_mv_wait_ns(uint64_t ns);
void testing_set_mv_delay_ns(uint64_t ns);
cudaError_t testing_clear_device_error_qmv_mma();
// aq_qmv_noalloc's fixed scratch (a file-scope device array in qmv_mma.cu).
constexpr size_t kQmvNoallocScratchBytes = (size_t)4 << 20;
// Launches the warp-MMA decode kernel on that scratch.  Sets *need to the
// scratch bytes the shape needs; returns cudaErrorMemoryAllocation (nothing
// launched, nothing allocated) when that exceeds kQmvNoallocScratchBytes.
cudaError_t launch_qmv_noalloc(const void* x, const void* w_q, const void* scales,
                               const void* biases, void* y, int64_t M, int64_t N, int64_t K,
                               int gs, int dtype, cudaStream_t st, size_t* need);
// aq_set_weight_prefetch's process-wide setting (0 or 1).
int weight_prefetch_enabled();
// aq_set_input_prefetch's process-wide setting (0 or 1).
int input_prefetch_enabled();
cudaError_t read_device_error_conv(unsigned* out);
}  // namespace aq
