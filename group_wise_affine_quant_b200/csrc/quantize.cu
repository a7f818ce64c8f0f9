// quantize.cu — the affine group quantizer and the dequantizer.
//
// Quantizer ("mlx 1.0.0, mlx/backend/cpu/quantized.cpp", quantize;
// "Improvements in the quantizer and dequantization kernel", item 1): one
// warp per group.  The arithmetic is fp32 with IEEE division (__fdiv_rn),
// explicit round-to-nearest subtraction and rintf (ties to even), so codes,
// scales and biases are bit-exact with the definition.  Codes are packed as
// the little-endian bit stream of the row: each lane ORs its run of codes into
// a per-warp shared-memory copy of the group's words, which the warp then
// stores with 32-bit writes (a group's packed size, gs*bits/8 bytes, is a
// multiple of 4 for every supported width).
//
// FP4 quantizer (the steps of fp_quantize_dequantize, to_fp8_e8m0 and
// to_fp4_e2m1 in "mlx 1.0.0, mlx/backend/cpu/quantized.cpp", up to the codes
// and the scale byte): one element per lane, a warp per 32 elements (one
// group of 32, or two groups of 16).  Per group, in fp32: absmax (NaN
// ignored), scale = absmax / 6 (IEEE division), the scale byte (E8M0 for
// group 32: the nearest power of two on a log scale; E4M3 for group 16: ties
// to even, saturating), the byte decoded back to float, and each code from
// the E2M1 threshold table applied to w / decoded scale.
//
// Fake quantization of activations (the same page's fp_quantize_dequantize,
// which QQMatmul applies to x): the FP4 quantizer's group steps with the
// scale divided by 6 (E2M1 elements) or 448 (E4M3 elements), each element
// replaced by T(s * v) with v the element's E2M1 / E4M3 value and s the
// decoded scale (one fp32 multiplication, one rounding to T).
//
// Dequantizer: one thread per 8 consecutive elements (8 codes = `bits`
// bytes), w_hat = fma(s, q, b) in T (a single rounding of the exact value;
// q is exact in fp16 and bf16 for q <= 256), or LUT[q] * s_T in fp32 (exact)
// rounded once to T in FP4 mode.
#include <cuda_fp8.h>

#include "common.cuh"

namespace aq {
namespace {

constexpr int kQWarps = 8;

template <typename T, int BITS>
__global__ void __launch_bounds__(kQWarps * 32)
quantize_kernel(const T* __restrict__ w, uint8_t* __restrict__ wq, T* __restrict__ scales,
                T* __restrict__ biases, int64_t N, int64_t K, int gs) {
  __shared__ uint32_t words[kQWarps][32];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int64_t G = K / gs;
  const int64_t total = N * G;
  const int E = gs >> 5;                     // elements per lane: 1, 2 or 4
  const int nwords = gs * BITS / 32;         // packed words per group (<= 32)
  const float n_bins = (float)((1 << BITS) - 1);
  const int64_t row_bytes = K * BITS / 8;

  for (int64_t grp = (int64_t)blockIdx.x * kQWarps + wid; grp < total;
       grp += (int64_t)gridDim.x * kQWarps) {
    const int64_t n = grp / G, g = grp - n * G;
    const T* src = w + n * K + g * gs + lane * E;
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = e < E ? TT<T>::to_f(src[e]) : 0.0f;
    float lo = v[0], hi = v[0];
#pragma unroll
    for (int e = 1; e < 4; ++e)
      if (e < E) { lo = fminf(lo, v[e]); hi = fmaxf(hi, v[e]); }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const bool at_min = fabsf(lo) > fabsf(hi);
    float scale = fmaxf(__fdiv_rn(__fsub_rn(hi, lo), n_bins), 1e-7f);
    if (!at_min) scale = -scale;
    const float edge = at_min ? lo : hi;
    const float q0 = rintf(__fdiv_rn(edge, scale));
    float bias = 0.0f;
    if (q0 != 0.0f) {
      scale = __fdiv_rn(edge, q0);
      bias = edge;
    }
    uint64_t run = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (e < E) {
        float c = rintf(__fdiv_rn(__fsub_rn(v[e], bias), scale));
        c = fminf(fmaxf(c, 0.0f), n_bins);
        run |= (uint64_t)(uint32_t)c << (e * BITS);
      }
    }
    if (lane < nwords) words[wid][lane] = 0u;
    __syncwarp();
    const int bitpos = lane * E * BITS;
    const int wi = bitpos >> 5, sh = bitpos & 31;
    atomicOr(&words[wid][wi], (uint32_t)(run << sh));
    if (sh + E * BITS > 32) atomicOr(&words[wid][wi + 1], (uint32_t)(run >> (32 - sh)));
    __syncwarp();
    uint32_t* dst = reinterpret_cast<uint32_t*>(wq + n * row_bytes + g * (int64_t)(gs * BITS / 8));
    if (lane < nwords) dst[lane] = words[wid][lane];
    if (lane == 0) {
      scales[grp] = TT<T>::from_f(scale);
      biases[grp] = TT<T>::from_f(bias);
    }
    __syncwarp();
  }
}

// E8M0 byte of a float: 0xFF for NaN / inf, 0 for x <= 0; otherwise
// round(log2(x)) taken exactly (x = m * 2^e with m in [1, 2) rounds up to
// 2^(e+1) when m >= sqrt(2), i.e. m * m >= 2, exact in double), clamped to
// [-127, 127], plus 127.
__device__ __forceinline__ unsigned e8m0_byte(float x) {
  if (!isfinite(x)) return 0xFFu;
  if (!(x > 0.0f)) return 0u;
  int e;
  const double m = 2.0 * frexp((double)x, &e);     // x = m * 2^(e-1)
  int n = (m * m >= 2.0) ? e : e - 1;
  n = n < -127 ? -127 : (n > 127 ? 127 : n);
  return (unsigned)(n + 127);
}

// E2M1 code of a float (the threshold table: round to nearest, ties to even,
// saturating at 6; NaN gives 0x7).
__device__ __forceinline__ unsigned e2m1_code(float x) {
  if (isnan(x)) return 0x7u;
  const unsigned sign = signbit(x) ? 0x8u : 0u;
  const float a = fabsf(x);
  unsigned b = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
               (a >= 3.5f) + (a > 5.0f);
  return b | sign;
}

template <typename T, int GS>
__global__ void __launch_bounds__(256)
quantize_fp4_kernel(const T* __restrict__ w, uint8_t* __restrict__ codes,
                    uint8_t* __restrict__ scales, int64_t N, int64_t K) {
  const int lane = threadIdx.x & 31;
  const int64_t chunks = N * (K / 32);                  // 32-element runs of a row
  const int64_t G = K / GS;
  for (int64_t ch = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; ch < chunks;
       ch += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int64_t n = ch / (K / 32), k0 = (ch - n * (K / 32)) * 32;
    const float v = TT<T>::to_f(w[n * K + k0 + lane]);
    float amax = isnan(v) ? -INFINITY : fabsf(v);
#pragma unroll
    for (int o = GS / 2; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float scale = __fdiv_rn(amax, 6.0f);
    unsigned byte;
    float sdec;
    if (GS == 32) {
      byte = e8m0_byte(scale);
      sdec = e8m0_to_float(byte);
    } else {
      byte = (unsigned)__nv_cvt_float_to_fp8(scale, __NV_SATFINITE, __NV_E4M3);
      sdec = e4m3_to_float(byte);
    }
    const float el = sdec == 0.0f ? 0.0f : __fdiv_rn(v, sdec);
    const unsigned c = e2m1_code(el);
    const unsigned hi = __shfl_down_sync(0xffffffffu, c, 1);
    if ((lane & 1) == 0) codes[n * (K / 2) + (k0 + lane) / 2] = (uint8_t)(c | (hi << 4));
    if ((lane & (GS - 1)) == 0) scales[n * G + (k0 + lane) / GS] = (uint8_t)byte;
  }
}

template <typename T, int GS, int BITS>
__global__ void __launch_bounds__(256)
quantize_dequantize_fp_kernel(const T* __restrict__ w, T* __restrict__ out, int64_t N, int64_t K) {
  const int lane = threadIdx.x & 31;
  const int64_t chunks = N * (K / 32);
  for (int64_t ch = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; ch < chunks;
       ch += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int64_t e = ch * 32 + lane;                   // rows are whole 32-element runs
    const float v = TT<T>::to_f(w[e]);
    float amax = isnan(v) ? -INFINITY : fabsf(v);
#pragma unroll
    for (int o = GS / 2; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float scale = __fdiv_rn(amax, BITS == 4 ? 6.0f : 448.0f);
    const float sdec =
        GS == 32 ? e8m0_to_float(e8m0_byte(scale))
                 : e4m3_to_float((unsigned)__nv_cvt_float_to_fp8(scale, __NV_SATFINITE, __NV_E4M3));
    const float el = sdec == 0.0f ? 0.0f : __fdiv_rn(v, sdec);
    const float q = BITS == 4
                        ? e2m1_to_float(e2m1_code(el))
                        : e4m3_to_float((unsigned)__nv_cvt_float_to_fp8(el, __NV_SATFINITE, __NV_E4M3));
    out[e] = TT<T>::from_f(__fmul_rn(sdec, q));
  }
}

template <typename T, int BITS>
__global__ void __launch_bounds__(256)
dequantize_affine_kernel(const uint8_t* __restrict__ wq, const T* __restrict__ scales,
                         const T* __restrict__ biases, T* __restrict__ out, int64_t N, int64_t K,
                         int gs) {
  const int64_t per_row = K >> 3;
  const int64_t total = N * per_row;
  const int64_t G = K / gs;
  const int64_t row_bytes = K * BITS / 8;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < total;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = it / per_row, e8 = it - n * per_row;
    const uint8_t* p = wq + n * row_bytes + e8 * BITS;
    uint32_t wd[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < BITS; ++i) wd[i >> 2] |= (uint32_t)__ldg(p + i) << ((i & 3) * 8);
    const int64_t gi = n * G + (e8 * 8) / gs;
    const T s = scales[gi], b = biases[gi];
    alignas(16) T o[8];
    o[0] = __hfma(s, TT<T>::from_u(code_at<BITS, 0>(wd)), b);
    o[1] = __hfma(s, TT<T>::from_u(code_at<BITS, 1>(wd)), b);
    o[2] = __hfma(s, TT<T>::from_u(code_at<BITS, 2>(wd)), b);
    o[3] = __hfma(s, TT<T>::from_u(code_at<BITS, 3>(wd)), b);
    o[4] = __hfma(s, TT<T>::from_u(code_at<BITS, 4>(wd)), b);
    o[5] = __hfma(s, TT<T>::from_u(code_at<BITS, 5>(wd)), b);
    o[6] = __hfma(s, TT<T>::from_u(code_at<BITS, 6>(wd)), b);
    o[7] = __hfma(s, TT<T>::from_u(code_at<BITS, 7>(wd)), b);
    *reinterpret_cast<uint4*>(out + n * K + e8 * 8) = *reinterpret_cast<const uint4*>(o);
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
dequantize_fp4_kernel(const uint8_t* __restrict__ wq, const uint8_t* __restrict__ scales,
                      T* __restrict__ out, int64_t N, int64_t K, int gs) {
  const int64_t per_row = K >> 3;
  const int64_t total = N * per_row;
  const int64_t G = K / gs;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < total;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = it / per_row, e8 = it - n * per_row;
    const uint32_t wd = __ldg(reinterpret_cast<const uint32_t*>(wq + n * (K / 2)) + e8);
    const float s = fp4_scale_t<T>(__ldg(scales + n * G + (e8 * 8) / gs), gs);
    alignas(16) T o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = TT<T>::from_f(e2m1_to_float((wd >> (4 * i)) & 15u) * s);
    *reinterpret_cast<uint4*>(out + n * K + e8 * 8) = *reinterpret_cast<const uint4*>(o);
  }
}

int grid_for(int64_t items, int per_block) {
  int64_t b = (items + per_block - 1) / per_block;
  if (b < 1) b = 1;
  if (b > 148 * 64) b = 148 * 64;
  return (int)b;
}

template <typename T>
cudaError_t quantize_t(const void* w, void* w_q, void* scales, void* biases, int64_t N,
                       int64_t K, int bits, int gs, cudaStream_t st) {
  const int64_t groups = N * (K / gs);
  if (groups == 0) return cudaSuccess;
  dim3 grid(grid_for(groups, kQWarps)), block(kQWarps * 32);
  auto args = [&](auto kern) {
    kern<<<grid, block, 0, st>>>((const T*)w, (uint8_t*)w_q, (T*)scales, (T*)biases, N, K, gs);
  };
  switch (bits) {
    case 2: args(quantize_kernel<T, 2>); break;
    case 3: args(quantize_kernel<T, 3>); break;
    case 4: args(quantize_kernel<T, 4>); break;
    case 5: args(quantize_kernel<T, 5>); break;
    case 6: args(quantize_kernel<T, 6>); break;
    case 8: args(quantize_kernel<T, 8>); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t dequantize_t(const void* w_q, const void* scales, const void* biases, void* out,
                         int64_t N, int64_t K, int bits, int gs, int mode, cudaStream_t st) {
  const int64_t items = N * (K / 8);
  if (items == 0) return cudaSuccess;
  dim3 grid(grid_for(items, 256)), block(256);
  if (mode == AQ_MODE_FP4) {
    dequantize_fp4_kernel<T><<<grid, block, 0, st>>>((const uint8_t*)w_q, (const uint8_t*)scales,
                                                     (T*)out, N, K, gs);
    return cudaGetLastError();
  }
  auto args = [&](auto kern) {
    kern<<<grid, block, 0, st>>>((const uint8_t*)w_q, (const T*)scales, (const T*)biases, (T*)out,
                                 N, K, gs);
  };
  switch (bits) {
    case 2: args(dequantize_affine_kernel<T, 2>); break;
    case 3: args(dequantize_affine_kernel<T, 3>); break;
    case 4: args(dequantize_affine_kernel<T, 4>); break;
    case 5: args(dequantize_affine_kernel<T, 5>); break;
    case 6: args(dequantize_affine_kernel<T, 6>); break;
    case 8: args(dequantize_affine_kernel<T, 8>); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t quantize_fp4_t(const void* w, void* codes, void* scales, int64_t N, int64_t K,
                           int gs, cudaStream_t st) {
  const int64_t chunks = N * (K / 32);
  if (chunks == 0) return cudaSuccess;
  dim3 grid(grid_for(chunks, 8)), block(256);
  if (gs == 32)
    quantize_fp4_kernel<T, 32><<<grid, block, 0, st>>>((const T*)w, (uint8_t*)codes,
                                                       (uint8_t*)scales, N, K);
  else
    quantize_fp4_kernel<T, 16><<<grid, block, 0, st>>>((const T*)w, (uint8_t*)codes,
                                                       (uint8_t*)scales, N, K);
  return cudaGetLastError();
}

template <typename T, int BITS>
cudaError_t qdq_fp_t(const void* w, void* out, int64_t N, int64_t K, int gs, cudaStream_t st) {
  const int64_t chunks = N * (K / 32);
  if (chunks == 0) return cudaSuccess;
  dim3 grid(grid_for(chunks, 8)), block(256);
  if (gs == 32)
    quantize_dequantize_fp_kernel<T, 32, BITS><<<grid, block, 0, st>>>((const T*)w, (T*)out, N, K);
  else
    quantize_dequantize_fp_kernel<T, 16, BITS><<<grid, block, 0, st>>>((const T*)w, (T*)out, N, K);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_dequantize_fp(const void* w, void* out, int64_t N, int64_t K, int bits,
                                          int gs, int dtype, cudaStream_t st) {
  if (dtype == AQ_F16)
    return bits == 4 ? qdq_fp_t<__half, 4>(w, out, N, K, gs, st)
                     : qdq_fp_t<__half, 8>(w, out, N, K, gs, st);
  return bits == 4 ? qdq_fp_t<__nv_bfloat16, 4>(w, out, N, K, gs, st)
                   : qdq_fp_t<__nv_bfloat16, 8>(w, out, N, K, gs, st);
}

cudaError_t launch_quantize_fp4(const void* w, void* codes, void* scales, int64_t N, int64_t K,
                                int gs, int dtype, cudaStream_t st) {
  return dtype == AQ_F16 ? quantize_fp4_t<__half>(w, codes, scales, N, K, gs, st)
                         : quantize_fp4_t<__nv_bfloat16>(w, codes, scales, N, K, gs, st);
}

cudaError_t launch_quantize(const void* w, void* w_q, void* scales, void* biases, int64_t N,
                            int64_t K, int bits, int gs, int dtype, cudaStream_t st) {
  return dtype == AQ_F16 ? quantize_t<__half>(w, w_q, scales, biases, N, K, bits, gs, st)
                         : quantize_t<__nv_bfloat16>(w, w_q, scales, biases, N, K, bits, gs, st);
}

cudaError_t launch_dequantize(const void* w_q, const void* scales, const void* biases,
                              void* w_out, int64_t N, int64_t K, int bits, int gs, int mode,
                              int dtype, cudaStream_t st) {
  return dtype == AQ_F16
             ? dequantize_t<__half>(w_q, scales, biases, w_out, N, K, bits, gs, mode, st)
             : dequantize_t<__nv_bfloat16>(w_q, scales, biases, w_out, N, K, bits, gs, mode, st);
}

}  // namespace aq
