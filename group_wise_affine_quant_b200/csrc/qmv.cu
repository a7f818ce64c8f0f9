// qmv.cu — weight-streaming GEMV for few rows of x (M <= 16).
//
// Prior art: affine_packed_qmv_fast in "Add the 3bit packed qmm_t" (one
// simdgroup streams a few weight rows, fp32 accumulation, simd_sum).  The
// B200 design:
//   * The weight is read exactly once from HBM.  A lane's unit is 32
//     consecutive codes of one row (4*bits bytes, loaded with the widest
//     aligned vector: 16 B for 4/8-bit, 8 B for 2/6-bit, 4 B for 3/5-bit), and
//     the lanes that share a row read consecutive units, so each warp load is
//     one contiguous span.
//   * x for the CTA's K-slice is staged once in shared memory as fp32, padded
//     by 16 bytes every 32 values so that lanes reading neighbouring units hit
//     distinct banks; the per-unit sums of x are staged beside it.
//   * Scale and bias are hoisted out of the 32-code dot product:
//       y += s * sum_k x_k q_k + b * sum_k x_k
//     (the form used by the qmv kernel of "Add the 3bit packed qmm_t"), so the
//     inner loop is one exact int->float conversion and one FMA per code per
//     row of x.  A 32-code unit never straddles an affine group (group_size
//     >= 32); FP4 at group 16 applies one scale per 16-code half.
//   * Lanes of a row combine by warp shuffles.  With more than one K-slice
//     (split-K), each CTA writes fp32 partial sums to the workspace and the
//     last CTA of a row block to finish (an atomic ticket) adds the slices in
//     slice order and writes y; it then resets its ticket, so the workspace is
//     ready for the next call.  No CTA waits for another.
#include <utility>

#include "common.cuh"

namespace aq {
namespace {

constexpr int kThreads = 256;
constexpr int kUnit = 32;          // codes per lane unit
constexpr int kUnitStride = 36;    // floats per unit in shared memory (16 B pad)

template <int BITS, int NW, int... C>
__device__ __forceinline__ void unpack_affine(const uint32_t (&w)[NW], float (&q)[kUnit],
                                              std::integer_sequence<int, C...>) {
  ((q[C] = u_to_f_exact(code_at<BITS, C>(w))), ...);
}
template <int NW, int... C>
__device__ __forceinline__ void unpack_fp4(const uint32_t (&w)[NW], float (&q)[kUnit],
                                           std::integer_sequence<int, C...>) {
  ((q[C] = e2m1_to_float(code_at<4, C>(w))), ...);
}

// 32 codes = 4*BITS bytes at p (aligned to the load width chosen here).
template <int BITS>
__device__ __forceinline__ void load_unit(const uint8_t* p, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4 || BITS == 8) {
#pragma unroll
    for (int i = 0; i < BITS / 4; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + i);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (BITS == 2 || BITS == 6) {
#pragma unroll
    for (int i = 0; i < BITS / 2; ++i) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p) + i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t*>(p) + i);
  }
}

template <typename T, int BITS, int MT, bool FP4>
__global__ void __launch_bounds__(kThreads)
qmv_kernel(const T* __restrict__ x, const uint8_t* __restrict__ wq,
           const void* __restrict__ scales_v, const T* __restrict__ biases, T* __restrict__ y,
           float* __restrict__ partials, unsigned* __restrict__ counters, int M, int64_t N,
           int64_t K, int gs, int64_t Ks, int S, int lpr_log2) {
  extern __shared__ float4 smem4[];
  float* smem = reinterpret_cast<float*>(smem4);
  const int split = blockIdx.y;
  const int64_t k0 = (int64_t)split * Ks;
  const int64_t klen = (K - k0 < Ks) ? (K - k0) : Ks;        // multiple of 32
  const int nunits = (int)(klen / kUnit);
  const int units_max = (int)(Ks / kUnit);
  const int xs_stride = units_max * kUnitStride;
  float* xs = smem;                                         // [MT][xs_stride]
  float* bs = smem + MT * xs_stride;                        // [MT][units_max]
  const int lpr = 1 << lpr_log2;
  const int rpw = 32 >> lpr_log2;
  const int rows_cta = (kThreads / 32) * rpw;
  const int64_t row0 = (int64_t)blockIdx.x * rows_cta;

  // Stage x[:, k0:k0+klen) as fp32 (rows m >= M read as zero).
  {
    const int per_row = (int)(klen / 8);
    for (int i = threadIdx.x; i < MT * per_row; i += kThreads) {
      const int m = i / per_row, c8 = i - m * per_row;
      float f[8];
      if (m < M) {
        const uint4 raw = *reinterpret_cast<const uint4*>(x + (int64_t)m * K + k0 + c8 * 8);
        const T* t = reinterpret_cast<const T*>(&raw);
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = TT<T>::to_f(t[j]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = 0.0f;
      }
      const int k = c8 * 8;
      float* dst = xs + m * xs_stride + (k / kUnit) * kUnitStride + (k % kUnit);
      reinterpret_cast<float4*>(dst)[0] = make_float4(f[0], f[1], f[2], f[3]);
      reinterpret_cast<float4*>(dst)[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
    __syncthreads();
    if (!FP4) {
      for (int i = threadIdx.x; i < MT * nunits; i += kThreads) {
        const int m = i / nunits, u = i - m * nunits;
        const float* src = xs + m * xs_stride + u * kUnitStride;
        float s = 0.0f;
#pragma unroll
        for (int j = 0; j < kUnit; ++j) s += src[j];
        bs[m * units_max + u] = s;
      }
    }
    __syncthreads();
  }

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = lane >> lpr_log2, ul = lane & (lpr - 1);
  const int64_t row = row0 + warp * rpw + seg;
  const int64_t G = K / gs;
  float acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.0f;

  if (row < N) {
    const uint8_t* wrow = wq + row * (K * BITS / 8) + k0 * BITS / 8;
    uint32_t wd[BITS];
    if (ul < nunits) load_unit<BITS>(wrow + (int64_t)ul * (4 * BITS), wd);
    for (int u = ul; u < nunits; u += lpr) {
      uint32_t cur[BITS];
#pragma unroll
      for (int i = 0; i < BITS; ++i) cur[i] = wd[i];
      if (u + lpr < nunits) load_unit<BITS>(wrow + (int64_t)(u + lpr) * (4 * BITS), wd);
      const int64_t g = (k0 + (int64_t)u * kUnit) / gs;
      // FP4 at group 16 has two scales per 32-code unit (halves lo / hi).
      float s_lo, s_hi, b = 0.0f;
      if constexpr (FP4) {
        const uint8_t* sp = reinterpret_cast<const uint8_t*>(scales_v) + row * G;
        s_lo = fp4_scale_t<T>(__ldg(sp + g), gs);
        s_hi = gs == 16 ? fp4_scale_t<T>(__ldg(sp + g + 1), gs) : s_lo;
      } else {
        s_lo = s_hi = TT<T>::to_f(reinterpret_cast<const T*>(scales_v)[row * G + g]);
        b = TT<T>::to_f(biases[row * G + g]);
      }
      float q[kUnit];
      if constexpr (FP4) unpack_fp4(cur, q, std::make_integer_sequence<int, kUnit>{});
      else unpack_affine<BITS>(cur, q, std::make_integer_sequence<int, kUnit>{});
      const float* xu = xs + u * kUnitStride;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float4* xv = reinterpret_cast<const float4*>(xu + m * xs_stride);
        float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // [half][parity]
#pragma unroll
        for (int j = 0; j < kUnit / 4; ++j) {
          const float4 a = xv[j];
          const int h = (j >= kUnit / 8) ? 2 : 0;
          d[h] = fmaf(a.x, q[4 * j + 0], d[h]);
          d[h + 1] = fmaf(a.y, q[4 * j + 1], d[h + 1]);
          d[h] = fmaf(a.z, q[4 * j + 2], d[h]);
          d[h + 1] = fmaf(a.w, q[4 * j + 3], d[h + 1]);
        }
        if constexpr (FP4) {
          acc[m] = fmaf(s_lo, d[0] + d[1], acc[m]);
          acc[m] = fmaf(s_hi, d[2] + d[3], acc[m]);
        } else {
          acc[m] = fmaf(s_lo, (d[0] + d[1]) + (d[2] + d[3]), acc[m]);
          acc[m] = fmaf(b, bs[m * units_max + u], acc[m]);
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m)
    for (int o = lpr >> 1; o; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);

  if (S == 1) {
    if (ul == 0 && row < N) {
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < M) y[(int64_t)m * N + row] = TT<T>::from_f(acc[m]);
    }
    return;
  }
  if (ul == 0 && row < N) {
#pragma unroll
    for (int m = 0; m < MT; ++m)
      if (m < M) partials[((int64_t)split * M + m) * N + row] = acc[m];
  }
  __threadfence();
  __syncthreads();
  __shared__ unsigned ticket;
  if (threadIdx.x == 0) ticket = atomicAdd(counters + blockIdx.x, 1u);
  __syncthreads();
  if (ticket != (unsigned)(S - 1)) return;
  __threadfence();
  for (int i = threadIdx.x; i < rows_cta * M; i += kThreads) {
    const int m = i / rows_cta;
    const int64_t r = row0 + (i - m * rows_cta);
    if (r >= N) continue;
    float sum = 0.0f;
    for (int s = 0; s < S; ++s) sum += __ldcg(partials + ((int64_t)s * M + m) * N + r);
    y[(int64_t)m * N + r] = TT<T>::from_f(sum);
  }
  if (threadIdx.x == 0) counters[blockIdx.x] = 0u;
}

int ilog2_floor(int64_t v) {
  int r = 0;
  while ((int64_t(1) << (r + 1)) <= v) ++r;
  return r;
}

template <typename T, int BITS, int MT, bool FP4>
cudaError_t launch_one(const QmvPlan& p, const void* x, const void* w_q, const void* scales,
                       const void* biases, void* y, int64_t M, int64_t N, int64_t K, int gs,
                       void* ws, cudaStream_t st) {
  auto kern = qmv_kernel<T, BITS, MT, FP4>;
  if (p.smem > 48 * 1024) {
    static bool attr_done[64] = {};   // per instantiation and device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !attr_done[dev]) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      if (e != cudaSuccess) return e;
      if (dev < 64) attr_done[dev] = true;
    }
  }
  float* partials = nullptr;
  unsigned* counters = nullptr;
  if (p.splits > 1) {
    partials = reinterpret_cast<float*>(ws);
    size_t off = ((size_t)p.splits * M * N * sizeof(float) + 255) & ~size_t(255);
    counters = reinterpret_cast<unsigned*>(reinterpret_cast<char*>(ws) + off);
  }
  dim3 grid((unsigned)p.row_blocks, (unsigned)p.splits);
  kern<<<grid, kThreads, p.smem, st>>>((const T*)x, (const uint8_t*)w_q, scales,
                                       (const T*)biases, (T*)y, partials, counters, (int)M, N, K,
                                       gs, p.ks, p.splits, ilog2_floor(p.lpr));
  return cudaGetLastError();
}

template <typename T, int BITS, bool FP4>
cudaError_t by_mt(const QmvPlan& p, const void* x, const void* w_q, const void* scales,
                  const void* biases, void* y, int64_t M, int64_t N, int64_t K, int gs, void* ws,
                  cudaStream_t st) {
  switch (p.mt) {
    case 1: return launch_one<T, BITS, 1, FP4>(p, x, w_q, scales, biases, y, M, N, K, gs, ws, st);
    case 2: return launch_one<T, BITS, 2, FP4>(p, x, w_q, scales, biases, y, M, N, K, gs, ws, st);
    case 4: return launch_one<T, BITS, 4, FP4>(p, x, w_q, scales, biases, y, M, N, K, gs, ws, st);
    case 8: return launch_one<T, BITS, 8, FP4>(p, x, w_q, scales, biases, y, M, N, K, gs, ws, st);
    default: return launch_one<T, BITS, 16, FP4>(p, x, w_q, scales, biases, y, M, N, K, gs, ws, st);
  }
}

template <typename T>
cudaError_t by_bits(const QmvPlan& p, const void* x, const void* w_q, const void* scales,
                    const void* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
                    int gs, int mode, void* ws, cudaStream_t st) {
  if (mode == AQ_MODE_FP4) return by_mt<T, 4, true>(p, x, w_q, scales, biases, y, M, N, K, gs, ws, st);
  switch (bits) {
    case 2: return by_mt<T, 2, false>(p, x, w_q, scales, biases, y, M, N, K, gs, ws, st);
    case 3: return by_mt<T, 3, false>(p, x, w_q, scales, biases, y, M, N, K, gs, ws, st);
    case 4: return by_mt<T, 4, false>(p, x, w_q, scales, biases, y, M, N, K, gs, ws, st);
    case 5: return by_mt<T, 5, false>(p, x, w_q, scales, biases, y, M, N, K, gs, ws, st);
    case 6: return by_mt<T, 6, false>(p, x, w_q, scales, biases, y, M, N, K, gs, ws, st);
    case 8: return by_mt<T, 8, false>(p, x, w_q, scales, biases, y, M, N, K, gs, ws, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

QmvPlan plan_qmv(int64_t M, int64_t N, int64_t K, int bits, int gs, int mode) {
  (void)bits; (void)gs; (void)mode;
  QmvPlan p{};
  p.mt = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16;
  const int64_t units = K / kUnit;
  const int64_t max_units = (16384 / p.mt) / kUnit;        // shared-memory bound on Ks
  const int64_t target_ctas = 2 * 148;
  int64_t S = (units + max_units - 1) / max_units;
  if (S < 1) S = 1;
  for (;;) {
    const int64_t us = (units + S - 1) / S;                // units per slice
    p.ks = us * kUnit;
    p.splits = (int)((units + us - 1) / us);
    int64_t l = 1;
    while (l * 2 <= us && l * 2 <= 32) l *= 2;
    p.lpr = (int)l;
    p.rows_cta = (kThreads / 32) * (32 / p.lpr);
    p.row_blocks = (N + p.rows_cta - 1) / p.rows_cta;
    if (p.row_blocks * p.splits >= target_ctas || us <= 8) break;
    ++S;
  }
  if (p.row_blocks < 1) p.row_blocks = 1;
  const int64_t umax = p.ks / kUnit;
  p.smem = (size_t)p.mt * (umax * kUnitStride + umax) * sizeof(float);
  p.ws_bytes = 0;
  if (p.splits > 1) {
    size_t part = ((size_t)p.splits * M * N * sizeof(float) + 255) & ~size_t(255);
    p.ws_bytes = part + (((size_t)p.row_blocks * sizeof(unsigned) + 255) & ~size_t(255));
  }
  return p;
}

cudaError_t launch_qmv(const QmvPlan& p, const void* x, const void* w_q, const void* scales,
                       const void* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
                       int gs, int mode, int dtype, void* ws, cudaStream_t st) {
  return dtype == AQ_F16
             ? by_bits<__half>(p, x, w_q, scales, biases, y, M, N, K, bits, gs, mode, ws, st)
             : by_bits<__nv_bfloat16>(p, x, w_q, scales, biases, y, M, N, K, bits, gs, mode, ws,
                                      st);
}

}  // namespace aq
