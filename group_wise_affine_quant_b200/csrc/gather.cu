// gather.cu — row gather and scatter for aq_gather_qmm's expert grouping:
// the pairs of a gather that share a weight matrix become one decode problem
// whose x rows are copied together (and whose y rows are copied back), so
// that each weight matrix is streamed once per call instead of once per pair.
// Plain copies of whole rows, 16 bytes per thread per step.  The row maps
// travel as kernel parameters (no host-to-device copy, so the call can be
// captured in a CUDA graph), kGatherMapRows rows per launch.
#include <algorithm>

#include "common.cuh"

namespace aq {
namespace {

struct RowMap {
  int32_t r[kGatherMapRows];
};

// dst row r = src row map[r] (map[r] < 0: a zero row); rows of `bytes` bytes,
// a multiple of 16.
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                   const __grid_constant__ RowMap map, int rows, int64_t bytes) {
  const int64_t vec = bytes / 16;
  const int64_t total = (int64_t)rows * vec;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / vec, c = i - r * vec;
    const int32_t s = map.r[r];
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (s >= 0) v = reinterpret_cast<const uint4*>(src + (int64_t)s * bytes)[c];
    reinterpret_cast<uint4*>(dst + r * bytes)[c] = v;
  }
}

// dst row map[r] = src row r where map[r] >= 0 (other rows are padding).
__global__ void __launch_bounds__(256)
scatter_rows_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                    const __grid_constant__ RowMap map, int rows, int64_t bytes) {
  const int64_t vec = bytes / 16;
  const int64_t total = (int64_t)rows * vec;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / vec, c = i - r * vec;
    const int32_t d = map.r[r];
    if (d >= 0)
      reinterpret_cast<uint4*>(dst + (int64_t)d * bytes)[c] =
          reinterpret_cast<const uint4*>(src + r * bytes)[c];
  }
}

int copy_grid(int64_t total) {
  return (int)std::min<int64_t>((total + 255) / 256, 8 * 148);
}

}  // namespace

// Gather (scatter = false): dst row i = src row map[i] (zero for -1), for
// i < rows.  Scatter: dst row map[i] = src row i (skipped for -1).  Rows of
// `bytes` bytes (a multiple of 16; both bases 16-byte aligned).
cudaError_t launch_row_copy(const void* src, void* dst, const int32_t* map, int rows,
                            int64_t bytes, bool scatter, cudaStream_t st) {
  for (int r0 = 0; r0 < rows; r0 += kGatherMapRows) {
    const int n = std::min(kGatherMapRows, rows - r0);
    RowMap m;
    for (int i = 0; i < kGatherMapRows; ++i) m.r[i] = i < n ? map[r0 + i] : -1;
    const int64_t total = (int64_t)n * (bytes / 16);
    if (total == 0) continue;
    if (scatter)
      scatter_rows_kernel<<<copy_grid(total), 256, 0, st>>>(
          (const uint8_t*)src + (int64_t)r0 * bytes, (uint8_t*)dst, m, n, bytes);
    else
      gather_rows_kernel<<<copy_grid(total), 256, 0, st>>>(
          (const uint8_t*)src, (uint8_t*)dst + (int64_t)r0 * bytes, m, n, bytes);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace aq
