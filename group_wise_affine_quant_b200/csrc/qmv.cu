// qmv.cu — fp32 CUDA-core weight-streaming GEMV for 1 <= M <= 16 rows of x:
// aq_qmv's fallback for the shapes that neither decode kernel takes (packed
// rows or scale rows that are not 16-byte multiples, or scales / biases that
// are not 16-byte aligned; see qmv_mma.cu and qmv_tc.cu).
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
//     (split-K, up to 8 slices), the slices of a row block form one thread
//     block cluster; each CTA keeps its fp32 row sums in shared memory and,
//     after a cluster barrier, adds the slices' sums in slice order through
//     distributed shared memory.  No workspace and no global atomics.
//   * A CTA stages x once and then walks RI groups of rows, and each lane
//     issues the load of its first weight unit before staging x.
#include <atomic>
#include <cooperative_groups.h>

#include <utility>

#include "common.cuh"

namespace cg = cooperative_groups;

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
           int M, int64_t N, int64_t K, int gs_log2, int64_t Ks, int S, int lpr_log2, int RI,
           int chunk_units, int weights_early, int x_early) {
  const int gs = 1 << gs_log2;
  extern __shared__ float4 smem4[];
  float* smem = reinterpret_cast<float*>(smem4);
  const int rank = blockIdx.y;                              // cluster spans all of y
  const int64_t k0 = (int64_t)rank * Ks;
  const int64_t klen = (K - k0 < Ks) ? (K - k0) : Ks;       // multiple of 32, > 0
  const int nunits = (int)(klen / kUnit);
  const int lpr = 1 << lpr_log2;
  const int rpw = 32 >> lpr_log2;
  const int rows_cta = (kThreads / 32) * rpw;
  const int rows_blk = rows_cta * RI;
  const int64_t row_base = (int64_t)blockIdx.x * rows_blk;
  const int xs_stride = chunk_units * kUnitStride;
  float* xs = smem;                                         // [MT][xs_stride]
  float* bs = xs + MT * xs_stride;                          // [MT][chunk_units]
  float* red = bs + ((MT * chunk_units + 3) & ~3);          // [MT][rows_blk], 16-byte aligned

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int seg = lane >> lpr_log2, ul = lane & (lpr - 1);
  const int64_t G = K >> gs_log2;
  const int64_t row_bytes = K * BITS / 8;

  // Programmatic dependent launch: let the next kernel start its prologue.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // Prefetch this lane's first weight unit before staging x, so the HBM
  // latency overlaps the staging (and, when the caller allows it, the end
  // of the previous kernel: weights are then read before the dependency
  // wait, x only after it).
  if (!weights_early) asm volatile("griddepcontrol.wait;" ::: "memory");
  uint32_t wd[BITS];
  {
    const int64_t row = row_base + warp * rpw + seg;
    if (row < N && ul < nunits && ul < chunk_units)
      load_unit<BITS>(wq + row * row_bytes + k0 * BITS / 8 + (int64_t)ul * (4 * BITS), wd);
  }
  if (!x_early) asm volatile("griddepcontrol.wait;" ::: "memory");

  for (int c0 = 0; c0 < nunits; c0 += chunk_units) {
    const int cu = (nunits - c0 < chunk_units) ? (nunits - c0) : chunk_units;
    if (c0) __syncthreads();                                // previous chunk fully consumed
    // Stage x[:, k0 + 32 c0 : + 32 cu) as fp32 (rows m >= M are zero).
    const int per_row = cu * (kUnit / 8);
    for (int i = threadIdx.x; i < MT * per_row; i += kThreads) {
      const int m = i / per_row, c8 = i - m * per_row;
      float f[8];
      if (m < M) {
        const uint4 raw =
            *reinterpret_cast<const uint4*>(x + (int64_t)m * K + k0 + (int64_t)c0 * kUnit + c8 * 8);
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
      for (int i = threadIdx.x; i < MT * cu; i += kThreads) {
        const int m = i / cu, u = i - m * cu;
        const float* src = xs + m * xs_stride + u * kUnitStride;
        float sum = 0.0f;
#pragma unroll
        for (int j = 0; j < kUnit; ++j) sum += src[j];
        bs[m * chunk_units + u] = sum;
      }
      __syncthreads();
    }

    for (int ri = 0; ri < RI; ++ri) {
      const int rloc = ri * rows_cta + warp * rpw + seg;
      const int64_t row = row_base + rloc;
      float acc[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
      if (row < N) {
        const uint8_t* wrow = wq + row * row_bytes + (k0 + (int64_t)c0 * kUnit) * BITS / 8;
        // the first unit of this row was prefetched (ri == 0, c0 == 0) or is loaded now
        if (ri > 0 || c0 > 0) {
          if (ul < cu) load_unit<BITS>(wrow + (int64_t)ul * (4 * BITS), wd);
        }
        for (int u = ul; u < cu; u += lpr) {
          uint32_t cur[BITS];
#pragma unroll
          for (int i = 0; i < BITS; ++i) cur[i] = wd[i];
          if (u + lpr < cu) load_unit<BITS>(wrow + (int64_t)(u + lpr) * (4 * BITS), wd);
          const int g = (int)(((int)k0 + (c0 + u) * kUnit) >> gs_log2);
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
              acc[m] = fmaf(b, bs[m * chunk_units + u], acc[m]);
            }
          }
        }
      }
#pragma unroll
      for (int m = 0; m < MT; ++m)
        for (int o = lpr >> 1; o; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
      if (ul == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m) red[m * rows_blk + rloc] = (c0 ? red[m * rows_blk + rloc] : 0.0f) + acc[m];
      }
    }
  }

  // Combine the K-slices: slice `rank` of the cluster finishes rows i with
  // i % S == rank, adding the slices' sums in slice order through
  // distributed shared memory.  Two cluster barriers: one before the reads,
  // one so that no CTA exits while another still reads its shared memory.
  cg::cluster_group cluster = cg::this_cluster();
  if (S > 1) cluster.sync(); else __syncthreads();
  asm volatile("griddepcontrol.wait;" ::: "memory");     // before y is written
  {
    // Rank `rank` finishes a contiguous slice of the [MT][rows_blk] sums with
    // 16-byte loads of every slice's partials (rows_blk is a multiple of 8),
    // added in slice order.
    const float4* red4 = reinterpret_cast<const float4*>(red);
    const int e4 = MT * rows_blk / 4;
    const int per = (e4 + S - 1) / S;
    const int f0 = rank * per, f1 = min(e4, f0 + per);
    for (int f = f0 + (int)threadIdx.x; f < f1; f += kThreads) {
      float4 acc = (S > 1 ? cluster.map_shared_rank(red4, 0) : red4)[f];
      for (int q = 1; q < S; ++q) {
        const float4 v = cluster.map_shared_rank(red4, q)[f];
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      const int e = 4 * f;
      const int m = e / rows_blk, rloc = e - m * rows_blk;
      if (m >= M) continue;
      const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int64_t row = row_base + rloc + t;
        if (row < N) y[(int64_t)m * N + row] = TT<T>::from_f(vals[t]);
      }
    }
  }
  if (S > 1) cluster.sync();
}

int ilog2_floor(int64_t v) {
  int r = 0;
  while ((int64_t(1) << (r + 1)) <= v) ++r;
  return r;
}

template <typename T, int BITS, int MT, bool FP4>
cudaError_t launch_one(const QmvPlan& p, const void* x, const void* w_q, const void* scales,
                       const void* biases, void* y, int64_t M, int64_t N, int64_t K, int gs,
                       cudaStream_t st) {
  auto kern = qmv_kernel<T, BITS, MT, FP4>;
  if (p.smem > 48 * 1024) {
    static std::atomic<bool> attr_done[64];   // per instantiation and device
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !attr_done[dev].load(std::memory_order_acquire)) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      if (e != cudaSuccess) return e;
      if (dev < 64) attr_done[dev].store(true, std::memory_order_release);
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.row_blocks, (unsigned)p.splits, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = (unsigned)p.splits;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, (const T*)x, (const uint8_t*)w_q, scales,
                            (const T*)biases, (T*)y, (int)M, N, K, ilog2_floor(gs), p.ks, p.splits,
                            ilog2_floor(p.lpr), p.ri, p.chunk_units, weight_prefetch_enabled(),
                            input_prefetch_enabled());
}

template <typename T, int BITS, bool FP4>
cudaError_t by_mt(const QmvPlan& p, const void* x, const void* w_q, const void* scales,
                  const void* biases, void* y, int64_t M, int64_t N, int64_t K, int gs,
                  cudaStream_t st) {
  switch (p.mt) {
    case 1: return launch_one<T, BITS, 1, FP4>(p, x, w_q, scales, biases, y, M, N, K, gs, st);
    case 2: return launch_one<T, BITS, 2, FP4>(p, x, w_q, scales, biases, y, M, N, K, gs, st);
    case 4: return launch_one<T, BITS, 4, FP4>(p, x, w_q, scales, biases, y, M, N, K, gs, st);
    case 8: return launch_one<T, BITS, 8, FP4>(p, x, w_q, scales, biases, y, M, N, K, gs, st);
    default: return launch_one<T, BITS, 16, FP4>(p, x, w_q, scales, biases, y, M, N, K, gs, st);
  }
}

template <typename T>
cudaError_t by_bits(const QmvPlan& p, const void* x, const void* w_q, const void* scales,
                    const void* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
                    int gs, int mode, cudaStream_t st) {
  if (mode == AQ_MODE_FP4) return by_mt<T, 4, true>(p, x, w_q, scales, biases, y, M, N, K, gs, st);
  switch (bits) {
    case 2: return by_mt<T, 2, false>(p, x, w_q, scales, biases, y, M, N, K, gs, st);
    case 3: return by_mt<T, 3, false>(p, x, w_q, scales, biases, y, M, N, K, gs, st);
    case 4: return by_mt<T, 4, false>(p, x, w_q, scales, biases, y, M, N, K, gs, st);
    case 5: return by_mt<T, 5, false>(p, x, w_q, scales, biases, y, M, N, K, gs, st);
    case 6: return by_mt<T, 6, false>(p, x, w_q, scales, biases, y, M, N, K, gs, st);
    case 8: return by_mt<T, 8, false>(p, x, w_q, scales, biases, y, M, N, K, gs, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

QmvPlan plan_qmv(int64_t M, int64_t N, int64_t K, int bits, int gs, int mode) {
  (void)bits; (void)gs; (void)mode;
  QmvPlan p{};
  p.mt = M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16;
  const int64_t units = K / kUnit;
  // Shared memory per staged unit and row of x: 36 floats + 1 sum.
  const int64_t smem_cap = 160 * 1024;
  const int64_t cap_units = smem_cap / ((int64_t)p.mt * (kUnitStride + 1) * 4);
  const int64_t target_ctas = 2 * 148;
  // Split K over up to 8 CTAs of a cluster until there are enough CTAs.
  int64_t S = 1, us = units;
  for (;;) {
    us = (units + S - 1) / S;
    int64_t l = 1;
    while (l * 2 <= us && l * 2 <= 32) l *= 2;
    const int64_t rows_cta = (kThreads / 32) * (32 / l);
    const int64_t rb = (N + rows_cta - 1) / rows_cta;
    const bool fits = us <= cap_units;
    if ((rb * S >= target_ctas && fits) || S == 8 || us <= 8) break;
    ++S;
  }
  p.ks = us * kUnit;
  p.splits = (int)((units + us - 1) / us);
  int64_t l = 1;
  while (l * 2 <= us && l * 2 <= 32) l *= 2;
  p.lpr = (int)l;
  p.rows_cta = (kThreads / 32) * (32 / p.lpr);
  p.chunk_units = (int)(us < cap_units ? us : cap_units);
  // Several row groups per CTA (x staged once) when the slice fits in one
  // chunk and there are CTAs to spare.
  const int64_t rb1 = (N + p.rows_cta - 1) / p.rows_cta;
  p.ri = 1;
  if (p.chunk_units >= us) {
    while (p.ri < 8 && (rb1 + 2 * p.ri - 1) / (2 * p.ri) * p.splits >= target_ctas) p.ri *= 2;
  }
  p.row_blocks = (N + (int64_t)p.rows_cta * p.ri - 1) / ((int64_t)p.rows_cta * p.ri);
  if (p.row_blocks < 1) p.row_blocks = 1;
  p.smem = ((size_t)p.mt * p.chunk_units * kUnitStride + (((size_t)p.mt * p.chunk_units + 3) & ~(size_t)3) +
            (size_t)p.mt * p.rows_cta * p.ri) * sizeof(float);
  p.ws_bytes = 0;
  return p;
}

cudaError_t launch_qmv(const QmvPlan& p, const void* x, const void* w_q, const void* scales,
                       const void* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
                       int gs, int mode, int dtype, void* ws, cudaStream_t st) {
  (void)ws;
  return dtype == AQ_F16
             ? by_bits<__half>(p, x, w_q, scales, biases, y, M, N, K, bits, gs, mode, st)
             : by_bits<__nv_bfloat16>(p, x, w_q, scales, biases, y, M, N, K, bits, gs, mode, st);
}

}  // namespace aq
