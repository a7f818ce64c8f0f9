// qmv_nt.cu — the non-transposed product of a quantized weight,
//   y [M, K] = x [M, N] . w_hat [N, K],
// with the weight stored as aq_qmv takes it (N rows of K codes, quantized
// along K).  It is the transpose = false form of quantized_matmul in "Add
// the 3bit packed qmm_t" (the product its VJP forms for x), here for
// decode-sized M (1..16 rows of x per launch; larger M runs in chunks).
//
// Design (fp32 CUDA cores; the weight is streamed once per launch):
//   * A thread owns 8 consecutive codes of every weight row in its CTA's row
//     range: one run of BITS bytes, and the 128 threads of a CTA read
//     consecutive runs, so each row's loads are one contiguous span.  A run
//     lies inside one group (group_size >= 16), so it takes one scale and one
//     bias per row.
//   * Per row n and row m of x: acc[m][c] += (x[m,n] s) q_c and
//     accb[m] += x[m,n] b (the bias term is common to the run), all fp32 with
//     the exact w_hat = s q + b kept as its two factors.
//   * x is staged as fp32 in shared memory, 128 weight rows at a time.
//   * Rows are split over blockIdx.y so that the grid fills the GPU; with more
//     than one split each split writes fp32 partial sums to the workspace
//     (after its first 64 KB, the counter area other calls keep zero) and a
//     second kernel adds the splits in split order and rounds to T once.
#include <algorithm>

#include "common.cuh"

namespace aq {
namespace {

int log2_of(int v) {
  int l = 0;
  while ((1 << l) < v) ++l;
  return l;
}

constexpr int kNtThreads = 128;           // threads per CTA = 8-code runs per CTA
constexpr int kNtRows = 128;              // weight rows per shared-memory stage of x
constexpr size_t kNtCounterArea = 65536;  // workspace bytes left untouched

// The BITS bytes of the 8-code run at byte offset off of a row (little-endian
// bit stream of the codes).
template <int BITS>
__device__ __forceinline__ uint64_t load_run(const uint8_t* p) {
  if constexpr (BITS == 8) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    return ((uint64_t)v.y << 32) | v.x;
  } else if constexpr (BITS == 4) {
    return __ldg(reinterpret_cast<const uint32_t*>(p));
  } else if constexpr (BITS == 2) {
    return __ldg(reinterpret_cast<const uint16_t*>(p));
  } else {
    uint64_t v = 0;
#pragma unroll
    for (int i = 0; i < BITS; ++i) v |= (uint64_t)__ldg(p + i) << (8 * i);
    return v;
  }
}

template <typename T, int BITS, int MT, bool FP4>
__global__ void __launch_bounds__(kNtThreads)
qmv_nt_kernel(const T* __restrict__ x, const uint8_t* __restrict__ wq,
              const void* __restrict__ scales, const T* __restrict__ biases,
              float* __restrict__ part, T* __restrict__ y, int M, int N, int K, int gs_log2,
              int rows_per_split) {
  __shared__ float xs[MT][kNtRows];
  const int run = blockIdx.x * kNtThreads + threadIdx.x;
  const int k0 = run * 8;
  const bool active = k0 < K;
  const int n_lo = blockIdx.y * rows_per_split;
  const int n_hi = min(N, n_lo + rows_per_split);
  const int64_t rb = (int64_t)K * BITS / 8;               // bytes per weight row
  const int G = K >> gs_log2;
  const int g = k0 >> gs_log2;
  float acc[MT][8], accb[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    accb[m] = 0.0f;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[m][c] = 0.0f;
  }
  for (int n0 = n_lo; n0 < n_hi; n0 += kNtRows) {
    const int rows = min(kNtRows, n_hi - n0);
    __syncthreads();                                       // the previous stage is consumed
    for (int i = threadIdx.x; i < MT * kNtRows; i += kNtThreads) {
      const int m = i / kNtRows, r = i % kNtRows;
      xs[m][r] = (m < M && r < rows) ? TT<T>::to_f(x[(int64_t)m * N + n0 + r]) : 0.0f;
    }
    __syncthreads();
    if (!active) continue;
    const uint8_t* wp = wq + (int64_t)n0 * rb + (int64_t)k0 * BITS / 8;
#pragma unroll 4
    for (int r = 0; r < rows; ++r) {
      const uint64_t v = load_run<BITS>(wp + r * rb);
      const int64_t sg = (int64_t)(n0 + r) * G + g;
      float s, b = 0.0f;
      if constexpr (FP4) {
        s = fp4_scale_t<T>(__ldg(reinterpret_cast<const uint8_t*>(scales) + sg), 1 << gs_log2);
      } else {
        s = TT<T>::to_f(reinterpret_cast<const T*>(scales)[sg]);
        b = TT<T>::to_f(biases[sg]);
      }
      float q[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const unsigned code = (unsigned)(v >> (c * BITS)) & ((1u << BITS) - 1u);
        q[c] = FP4 ? e2m1_to_float(code) : u_to_f_exact(code);
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float xv = xs[m][r];
        const float xsv = xv * s;
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[m][c] = fmaf(xsv, q[c], acc[m][c]);
        if constexpr (!FP4) accb[m] = fmaf(xv, b, accb[m]);
      }
    }
  }
  if (!active) return;
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if (m >= M) break;
    if (part) {
      float* dst = part + ((int64_t)blockIdx.y * M + m) * K + k0;
      const float4 lo = make_float4(acc[m][0] + accb[m], acc[m][1] + accb[m], acc[m][2] + accb[m],
                                    acc[m][3] + accb[m]);
      const float4 hi = make_float4(acc[m][4] + accb[m], acc[m][5] + accb[m], acc[m][6] + accb[m],
                                    acc[m][7] + accb[m]);
      reinterpret_cast<float4*>(dst)[0] = lo;
      reinterpret_cast<float4*>(dst)[1] = hi;
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) y[(int64_t)m * K + k0 + c] = TT<T>::from_f(acc[m][c] + accb[m]);
    }
  }
}

// y[m, k] = T(sum over splits, in split order, of the partial sums).
template <typename T>
__global__ void __launch_bounds__(256)
qmv_nt_reduce_kernel(const float* __restrict__ part, T* __restrict__ y, int M, int K, int splits) {
  const int64_t total = (int64_t)M * K;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int j = 0; j < splits; ++j) s += part[(int64_t)j * total + i];
    y[i] = TT<T>::from_f(s);
  }
}

struct NtPlan {
  int kblocks, splits, rows_per_split;
};

NtPlan plan_nt(int64_t N, int64_t K) {
  NtPlan p;
  p.kblocks = (int)((K / 8 + kNtThreads - 1) / kNtThreads);
  // about two CTAs per SM, each with at least 64 weight rows
  int splits = (2 * 148 + p.kblocks - 1) / p.kblocks;
  splits = std::max(1, std::min(splits, (int)((N + 63) / 64)));
  p.rows_per_split = (int)((N + splits - 1) / splits);
  p.splits = (int)((N + p.rows_per_split - 1) / p.rows_per_split);
  return p;
}

template <typename T, int BITS, bool FP4>
cudaError_t nt_by_m(const void* x, const void* w_q, const void* scales, const void* biases,
                    void* y, int M, int N, int K, int gs_log2, float* part, const NtPlan& p,
                    cudaStream_t st) {
  dim3 grid(p.kblocks, p.splits), block(kNtThreads);
  const T* xt = (const T*)x;
  const uint8_t* w = (const uint8_t*)w_q;
  const T* b = (const T*)biases;
  T* yt = (T*)y;
  if (M == 1)
    qmv_nt_kernel<T, BITS, 1, FP4><<<grid, block, 0, st>>>(xt, w, scales, b, part, yt, M, N, K, gs_log2, p.rows_per_split);
  else if (M == 2)
    qmv_nt_kernel<T, BITS, 2, FP4><<<grid, block, 0, st>>>(xt, w, scales, b, part, yt, M, N, K, gs_log2, p.rows_per_split);
  else if (M <= 4)
    qmv_nt_kernel<T, BITS, 4, FP4><<<grid, block, 0, st>>>(xt, w, scales, b, part, yt, M, N, K, gs_log2, p.rows_per_split);
  else if (M <= 8)
    qmv_nt_kernel<T, BITS, 8, FP4><<<grid, block, 0, st>>>(xt, w, scales, b, part, yt, M, N, K, gs_log2, p.rows_per_split);
  else
    qmv_nt_kernel<T, BITS, 16, FP4><<<grid, block, 0, st>>>(xt, w, scales, b, part, yt, M, N, K, gs_log2, p.rows_per_split);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !part) return e;
  const int64_t total = (int64_t)M * K;
  qmv_nt_reduce_kernel<T><<<(int)std::min<int64_t>((total + 255) / 256, 4 * 148), 256, 0, st>>>(
      part, yt, M, K, p.splits);
  return cudaGetLastError();
}

template <typename T>
cudaError_t nt_by_bits(const void* x, const void* w_q, const void* scales, const void* biases,
                       void* y, int M, int N, int K, int bits, int gs_log2, bool fp4, float* part,
                       const NtPlan& p, cudaStream_t st) {
  if (fp4) return nt_by_m<T, 4, true>(x, w_q, scales, biases, y, M, N, K, gs_log2, part, p, st);
  switch (bits) {
    case 2: return nt_by_m<T, 2, false>(x, w_q, scales, biases, y, M, N, K, gs_log2, part, p, st);
    case 3: return nt_by_m<T, 3, false>(x, w_q, scales, biases, y, M, N, K, gs_log2, part, p, st);
    case 4: return nt_by_m<T, 4, false>(x, w_q, scales, biases, y, M, N, K, gs_log2, part, p, st);
    case 5: return nt_by_m<T, 5, false>(x, w_q, scales, biases, y, M, N, K, gs_log2, part, p, st);
    case 6: return nt_by_m<T, 6, false>(x, w_q, scales, biases, y, M, N, K, gs_log2, part, p, st);
    default: return nt_by_m<T, 8, false>(x, w_q, scales, biases, y, M, N, K, gs_log2, part, p, st);
  }
}

}  // namespace

size_t qmm_nt_workspace(int64_t M, int64_t N, int64_t K, int bits) {
  (void)bits;
  const NtPlan p = plan_nt(N, K);
  if (p.splits <= 1) return 0;
  return kNtCounterArea + (size_t)p.splits * (size_t)std::min<int64_t>(M, 16) * (size_t)K * 4;
}

cudaError_t launch_qmm_nt(const void* x, const void* w_q, const void* scales, const void* biases,
                          void* y, int64_t M, int64_t N, int64_t K, int bits, int gs, int mode,
                          int dtype, void* workspace, cudaStream_t st) {
  const NtPlan p = plan_nt(N, K);
  float* part = p.splits > 1
                    ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kNtCounterArea)
                    : nullptr;
  const int gl = log2_of(gs);
  const bool fp4 = mode == AQ_MODE_FP4;
  // 16 rows of x per launch; the chunks run in stream order and reuse the
  // partial-sum area.
  for (int64_t m0 = 0; m0 < M; m0 += 16) {
    const int mc = (int)std::min<int64_t>(16, M - m0);
    const uint8_t* xc = static_cast<const uint8_t*>(x) + m0 * N * 2;
    uint8_t* yc = static_cast<uint8_t*>(y) + m0 * K * 2;
    const cudaError_t e =
        dtype == AQ_F16
            ? nt_by_bits<__half>(xc, w_q, scales, biases, yc, mc, (int)N, (int)K, bits, gl, fp4,
                                 part, p, st)
            : nt_by_bits<__nv_bfloat16>(xc, w_q, scales, biases, yc, mc, (int)N, (int)K, bits, gl,
                                        fp4, part, p, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace aq
