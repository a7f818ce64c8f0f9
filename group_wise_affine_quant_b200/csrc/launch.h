// launch.h — host-side launchers and plans of the kernels (declarations
// only; the definitions are in the .cu files).  Included at the end of
// common.cuh, after the constants and the problem descriptor they use.
#pragma once

// Launchers implemented in the .cu files; all return cudaSuccess or the
// launch error.
namespace aq {
cudaError_t launch_quantize(const void* w, void* w_q, void* scales, void* biases, int64_t N,
                            int64_t K, int bits, int gs, int dtype, cudaStream_t st);
cudaError_t launch_quantize_fp4(const void* w, void* codes, void* scales, int64_t N, int64_t K,
                                int gs, int dtype, cudaStream_t st);
size_t qmm_nt_workspace(int64_t M, int64_t N, int64_t K, int bits);
cudaError_t launch_qmm_nt(const void* x, const void* w_q, const void* scales, const void* biases,
                          void* y, int64_t M, int64_t N, int64_t K, int bits, int gs, int mode,
                          int dtype, void* workspace, cudaStream_t st);
// Row gather / scatter of aq_gather_qmm's expert grouping (gather.cu): row
// maps of up to kGatherMapRows rows travel as kernel parameters.
constexpr int kGatherMapRows = 960;
cudaError_t launch_row_copy(const void* src, void* dst, const int32_t* map, int rows,
                            int64_t bytes, bool scatter, cudaStream_t st);
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
// Launches the warp-MMA decode kernel on that scratch.  Sets *need to the
// scratch bytes the shape needs; returns cudaErrorMemoryAllocation (nothing
// launched, nothing allocated) when that exceeds kQmvNoallocScratchBytes.
cudaError_t launch_qmv_noalloc(const void* x, const void* w_q, const void* scales,
                               const void* biases, void* y, int64_t M, int64_t N, int64_t K,
                               int gs, int dtype, cudaStream_t st, size_t* need);
// aq_set_weight_prefetch's setting of the calling thread (0 or 1).
int weight_prefetch_enabled();
// aq_set_input_prefetch's setting of the calling thread (0 or 1).
int input_prefetch_enabled();
cudaError_t read_device_error_conv(unsigned* out);
}  // namespace aq
