// qmm.cu — dense entry of the tensor-core quantized matmul: plan and launch
// of y = x . dequant(W)^T with x [M, K] read by 2-D TMA (kernel template in
// qmm_kernel.cuh).
#include "qmm_kernel.cuh"

namespace aq {

QmmPlan plan_qmm(int64_t M, int64_t N, int64_t K, int bits, int gs, int mode) {
  (void)gs; (void)mode;
  QmmPlan p{};
  const int64_t n_tiles = (N + kRowsW - 1) / kRowsW;
  const int64_t k_tiles = (K + kBK - 1) / kBK;
  const int sms = 148;
  // Token tile: the smallest that covers M up to 128 (one wave of weight
  // tiles), else 256.  The widest tile dequantizes each weight stage once for
  // the most rows of x; when its tiles underfill the GPU, K is split over a
  // cluster instead of narrowing the tile (measured on B200: 1024x1024x4096
  // runs at 417 TFLOP/s as 32 tiles of 256 split four ways, 257 as 128
  // tiles of 64; 1024x4096x1024 at 565 as 128 tiles of 256, 343 as 256
  // tiles of 128).
  int bt;
  if (M <= 16) bt = 16;
  else if (M <= 32) bt = 32;
  else if (M <= 64) bt = 64;
  else if (M <= 128) bt = 128;
  else bt = 256;
  p.bt = bt;
  p.n_tiles = n_tiles;
  p.m_tiles = (M + bt - 1) / bt;
  p.k_tiles = (int)k_tiles;
  // Light CTAs (bt <= 32) fit two per SM.
  plan_splits(p, bits, bt <= 32 ? 2 * sms : sms);
  return p;
}

cudaError_t launch_qmm(const QmmPlan& p, const void* x, const void* w_q, const void* scales,
                       const void* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
                       int gs, int mode, int dtype, cudaStream_t st) {
  QmmMaps maps;
  memset(&maps, 0, sizeof(maps));
  const CUtensorMapDataType tt =
      dtype == AQ_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cudaError_t e = make_map(&maps.x, x, tt, 2, M, K, kBK, p.bt, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  QmmArgs a;
  memset(&a, 0, sizeof(a));
  a.wq = (const uint8_t*)w_q;
  a.scales = scales;
  a.biases = biases;
  a.y = y;
  a.x = x;
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.gs_log2 = ilog2i(gs);
  a.weights_early = weight_prefetch_enabled();
  a.x_early = input_prefetch_enabled();
  a.k_tiles = p.k_tiles;
  a.k_tiles_split = p.k_tiles_split;
  a.splits = p.splits;
  a.ldy = (int)N;
  a.n_limit = (int)N;
  a.ntg = (int)p.n_tiles;
  bool fast = false;
  e = weight_maps(maps, a, w_q, scales, biases, N, K, bits, gs, mode, &fast);
  if (e != cudaSuccess) return e;
  if (fast)
    return dtype == AQ_F16 ? by_bits_tc<__half, true, 0>(p, maps, a, bits, mode, st)
                           : by_bits_tc<__nv_bfloat16, true, 0>(p, maps, a, bits, mode, st);
  return dtype == AQ_F16 ? by_bits_tc<__half, false, 0>(p, maps, a, bits, mode, st)
                         : by_bits_tc<__nv_bfloat16, false, 0>(p, maps, a, bits, mode, st);
}

cudaError_t read_device_error_qmm(unsigned* out) { return read_tu_error(out); }

}  // namespace aq
