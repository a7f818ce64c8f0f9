// api.cu — the exported C ABI: argument validation, planning and dispatch.
// Every entry point validates on the host before it enqueues anything and
// reports failures through its return value and a thread-local message.
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include <algorithm>
#include <atomic>
#include <vector>

#include "common.cuh"
#include "../../include/aq_testing.h"

namespace {

thread_local char g_err[512] = "";

aq_status fail(aq_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

aq_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return AQ_OK;
  return fail(AQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

const int64_t kMaxDim = (int64_t(1) << 31) - 1;

// Format checks shared by every entry point.
aq_status check_format(int bits, int gs, aq_mode mode, aq_dtype dt) {
  if (dt != AQ_F16 && dt != AQ_BF16) return fail(AQ_ERR_UNSUPPORTED, "dtype %d is not fp16 (0) or bf16 (1)", (int)dt);
  if (mode == AQ_MODE_AFFINE) {
    if (!(bits == 2 || bits == 3 || bits == 4 || bits == 5 || bits == 6 || bits == 8))
      return fail(AQ_ERR_UNSUPPORTED, "bits %d: affine mode supports 2, 3, 4, 5, 6 or 8", bits);
    if (!(gs == 32 || gs == 64 || gs == 128))
      return fail(AQ_ERR_UNSUPPORTED, "group_size %d: affine mode supports 32, 64 or 128", gs);
  } else if (mode == AQ_MODE_FP4) {
    if (bits != 4) return fail(AQ_ERR_UNSUPPORTED, "bits %d: FP4 mode has 4-bit codes", bits);
    if (gs != 16 && gs != 32)
      return fail(AQ_ERR_UNSUPPORTED, "group_size %d: FP4 mode supports 32 (E8M0) or 16 (E4M3)", gs);
  } else {
    return fail(AQ_ERR_UNSUPPORTED, "mode %d is not affine (0) or fp4 (1)", (int)mode);
  }
  return AQ_OK;
}

aq_status check_weight(const void* w_q, const void* scales, const void* biases, int64_t N,
                       int64_t K, int bits, int gs, aq_mode mode, aq_dtype dt) {
  aq_status st = check_format(bits, gs, mode, dt);
  if (st != AQ_OK) return st;
  if (N < 0 || K < 0 || N > kMaxDim || K > kMaxDim)
    return fail(AQ_ERR_INVALID_ARG, "N=%lld K=%lld out of range", (long long)N, (long long)K);
  if (K % gs) return fail(AQ_ERR_INVALID_ARG, "K=%lld is not a multiple of group_size %d", (long long)K, gs);
  if (N > 0 && K > 0) {
    if (!w_q || !scales) return fail(AQ_ERR_INVALID_ARG, "w_q and scales must not be NULL");
    if (!aligned(w_q, 16)) return fail(AQ_ERR_MISALIGNED, "w_q must be 16-byte aligned");
    if (mode == AQ_MODE_AFFINE) {
      if (!biases) return fail(AQ_ERR_INVALID_ARG, "affine mode needs biases");
      if (!aligned(scales, 2) || !aligned(biases, 2))
        return fail(AQ_ERR_MISALIGNED, "scales and biases must be 2-byte aligned");
    } else if (biases) {
      return fail(AQ_ERR_INVALID_ARG, "FP4 mode takes no biases (pass NULL)");
    }
  }
  return AQ_OK;
}

}  // namespace

namespace {
// Per calling thread: one component's setting never reaches another's calls.
thread_local int g_weight_prefetch = 0;
thread_local int g_input_prefetch = 0;
}

int aq::weight_prefetch_enabled() { return g_weight_prefetch; }
int aq::input_prefetch_enabled() { return g_input_prefetch; }

extern "C" {

const char* aq_last_error(void) { return g_err; }

void aq_set_weight_prefetch(int enable) { g_weight_prefetch = enable ? 1 : 0; }

int aq_get_weight_prefetch(void) { return aq::weight_prefetch_enabled(); }

void aq_set_input_prefetch(int enable) { g_input_prefetch = enable ? 1 : 0; }

int aq_get_input_prefetch(void) { return aq::input_prefetch_enabled(); }

int aq_version(void) { return 100; }

aq_status aq_quantize(const void* w, void* w_q, void* scales, void* biases, int64_t N,
                      int64_t K, int bits, int group_size, aq_dtype dtype, aq_stream_t stream) {
  g_err[0] = 0;
  aq_status st = check_weight(w_q, scales, biases, N, K, bits, group_size, AQ_MODE_AFFINE, dtype);
  if (st != AQ_OK) return st;
  if (N == 0 || K == 0) return AQ_OK;
  if (!w) return fail(AQ_ERR_INVALID_ARG, "w must not be NULL");
  if (!aligned(w, 16)) return fail(AQ_ERR_MISALIGNED, "w must be 16-byte aligned");
  return cuda_status(aq::launch_quantize(w, w_q, scales, biases, N, K, bits, group_size, dtype,
                                         (cudaStream_t)stream),
                     "aq_quantize launch");
}

aq_status aq_quantize_fp4(const void* w, void* codes, void* scales, int64_t N, int64_t K,
                          int group_size, aq_dtype dtype, aq_stream_t stream) {
  g_err[0] = 0;
  if (dtype != AQ_F16 && dtype != AQ_BF16)
    return fail(AQ_ERR_UNSUPPORTED, "dtype %d is not fp16 (0) or bf16 (1)", (int)dtype);
  if (group_size != 16 && group_size != 32)
    return fail(AQ_ERR_UNSUPPORTED, "group_size %d: FP4 scales are E8M0 (32) or E4M3 (16)", group_size);
  if (N < 0 || K < 0 || N > kMaxDim || K > kMaxDim)
    return fail(AQ_ERR_INVALID_ARG, "N=%lld K=%lld out of range", (long long)N, (long long)K);
  if (K % 32)
    return fail(AQ_ERR_INVALID_ARG, "K=%lld is not a multiple of 32", (long long)K);
  if (N == 0 || K == 0) return AQ_OK;
  if (!w || !codes || !scales) return fail(AQ_ERR_INVALID_ARG, "w, codes and scales must not be NULL");
  if (!aligned(w, 2)) return fail(AQ_ERR_MISALIGNED, "w must be 2-byte aligned");
  return cuda_status(aq::launch_quantize_fp4(w, codes, scales, N, K, group_size, dtype,
                                             (cudaStream_t)stream),
                     "aq_quantize_fp4 launch");
}

aq_status aq_dequantize(const void* w_q, const void* scales, const void* biases, void* w_out,
                        int64_t N, int64_t K, int bits, int group_size, aq_mode mode,
                        aq_dtype dtype, aq_stream_t stream) {
  g_err[0] = 0;
  aq_status st = check_weight(w_q, scales, biases, N, K, bits, group_size, mode, dtype);
  if (st != AQ_OK) return st;
  if (N == 0 || K == 0) return AQ_OK;
  if (!w_out) return fail(AQ_ERR_INVALID_ARG, "w_out must not be NULL");
  if (!aligned(w_out, 16)) return fail(AQ_ERR_MISALIGNED, "w_out must be 16-byte aligned");
  return cuda_status(aq::launch_dequantize(w_q, scales, biases, w_out, N, K, bits, group_size,
                                           mode, dtype, (cudaStream_t)stream),
                     "aq_dequantize launch");
}

static aq_status check_mm(const void* x, const void* y, int64_t M, int64_t N, int64_t K) {
  if (M < 0 || M > kMaxDim) return fail(AQ_ERR_INVALID_ARG, "M=%lld out of range", (long long)M);
  if (M > 0 && N > 0) {
    if (!y) return fail(AQ_ERR_INVALID_ARG, "y must not be NULL");
    if (!aligned(y, 16)) return fail(AQ_ERR_MISALIGNED, "y must be 16-byte aligned");
    if (K > 0) {
      if (!x) return fail(AQ_ERR_INVALID_ARG, "x must not be NULL");
      if (!aligned(x, 16)) return fail(AQ_ERR_MISALIGNED, "x must be 16-byte aligned");
    }
  }
  return AQ_OK;
}

static aq_status check_workspace(const void* ws, size_t bytes, size_t need) {
  if (need == 0) return AQ_OK;
  if (!ws || bytes < need)
    return fail(AQ_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu%s)", need, bytes,
                ws ? "" : ", NULL");
  if (!aligned(ws, 256)) return fail(AQ_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  return AQ_OK;
}

static aq_status zero_output(void* y, int64_t M, int64_t N, aq_stream_t stream) {
  // K == 0: the empty sum is +0 in every output.
  return cuda_status(cudaMemsetAsync(y, 0, (size_t)(M * N) * 2, (cudaStream_t)stream),
                     "zero-fill of y");
}

// Kernel choice of aq_qmv forced by a test (0: automatic).
static std::atomic<int> g_qmv_kernel{0};

aq_status aq_qmv(const void* x, const void* w_q, const void* scales, const void* biases,
                 void* y, int64_t M, int64_t N, int64_t K, int bits, int group_size,
                 aq_mode mode, aq_dtype dtype, void* workspace, size_t workspace_bytes,
                 aq_stream_t stream) {
  g_err[0] = 0;
  aq_status st = check_weight(w_q, scales, biases, N, K, bits, group_size, mode, dtype);
  if (st != AQ_OK) return st;
  if (M < 1 || M > 16) return fail(AQ_ERR_INVALID_ARG, "aq_qmv takes 1 <= M <= 16 (got %lld)", (long long)M);
  if ((st = check_mm(x, y, M, N, K)) != AQ_OK) return st;
  if (N == 0) return AQ_OK;
  if (K == 0) return zero_output(y, M, N, stream);
  // 4-bit affine weights with K a multiple of the sub-slice run the
  // warp-MMA streaming kernel; other shapes whose packed rows and scale rows
  // are 16-byte multiples (TMA) run the tcgen05 decode kernel; the rest run
  // the fp32 CUDA-core kernel.  All keep w_hat in fp32 (scale and bias per
  // group).
  // A single small problem (M = 1 up to 2^24 weights, M <= 2 up to 2^22,
  // M <= 4 up to 2^20) runs the fp32 kernel: it has fewer serial phases per
  // call than the warp-MMA kernel's TMA / prep / MMA pipeline, and a lone call
  // of that size is bound by those phases, not by the weight stream.  Measured
  // on B200 in chains of dependent calls: at M = 1, 4.1 against 7.5 us for
  // 512 x 2048 and 10.8 against 14.1 us for 2048 x 8192; at M = 2, 8.3
  // against 9.3 us for 2048 x 2048; from 8192 x 8192 (M = 1), 8192 x 2048
  // (M = 2) and 2048 x 2048 (M = 4) on the warp-MMA kernel is faster.
  const int force = g_qmv_kernel.load(std::memory_order_relaxed);
  const int64_t nk = N * K;
  const bool lone_small = (M == 1 && nk <= ((int64_t)1 << 24)) ||
                          (M <= 2 && nk <= ((int64_t)1 << 22)) ||
                          (M <= 4 && nk <= ((int64_t)1 << 20));
  if (force != 2 && force != 3 && (force == 1 || !lone_small) &&
      aq::qmv_mma_applies(M, N, K, bits, group_size, mode, scales, biases)) {
    const size_t need = aq::qmv_mma_workspace(M, N, K, group_size);
    if ((st = check_workspace(workspace, workspace_bytes, need)) != AQ_OK) return st;
    return cuda_status(aq::launch_qmv_mma(x, w_q, scales, biases, y, M, N, K, group_size, dtype,
                                          workspace, (cudaStream_t)stream),
                       "aq_qmv launch");
  }
  if (force != 3 && !(force == 0 && lone_small && mode == AQ_MODE_AFFINE && bits == 4) &&
      aq::qmv_tc_applies(M, N, K, bits, group_size, mode, scales, biases)) {
    const size_t need = aq::qmv_tc_workspace(M, N, K, bits, group_size);
    if ((st = check_workspace(workspace, workspace_bytes, need)) != AQ_OK) return st;
    return cuda_status(aq::launch_qmv_tc(x, w_q, scales, biases, y, M, N, K, bits, group_size,
                                         mode, dtype, workspace, (cudaStream_t)stream),
                       "aq_qmv launch");
  }
  const aq::QmvPlan p = aq::plan_qmv(M, N, K, bits, group_size, mode);
  return cuda_status(aq::launch_qmv(p, x, w_q, scales, biases, y, M, N, K, bits, group_size,
                                    mode, dtype, workspace, (cudaStream_t)stream),
                     "aq_qmv launch");
}

// Whether every problem of a batch takes the warp-MMA decode kernel (the
// batch then runs on it; otherwise on the tcgen05 decode kernel).
static bool all_mma(const aq_qmv_problem* problems, int count, int64_t M, int bits,
                    int group_size, aq_mode mode) {
  for (int i = 0; i < count; ++i)
    if (!aq::qmv_mma_applies(M, problems[i].N, problems[i].K, bits, group_size, mode,
                             problems[i].scales, problems[i].biases))
      return false;
  return true;
}

aq_status aq_qmv_noalloc(const void* x, const void* w_q, const void* scales,
                         const void* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
                         int group_size, aq_mode mode, aq_dtype dtype, aq_stream_t stream) {
  g_err[0] = 0;
  aq_status st = check_weight(w_q, scales, biases, N, K, bits, group_size, mode, dtype);
  if (st != AQ_OK) return st;
  if (M < 1 || M > 16)
    return fail(AQ_ERR_INVALID_ARG, "aq_qmv_noalloc takes 1 <= M <= 16 (got %lld)", (long long)M);
  if ((st = check_mm(x, y, M, N, K)) != AQ_OK) return st;
  if (N == 0 || K == 0)
    return fail(AQ_ERR_INVALID_ARG, "aq_qmv_noalloc needs N, K > 0");
  if (!aq::qmv_mma_applies(M, N, K, bits, group_size, mode, scales, biases))
    return fail(AQ_ERR_UNSUPPORTED,
                "aq_qmv_noalloc takes 4-bit affine weights with K a multiple of 512 (1024 for "
                "group_size 128) and 16-byte aligned scales / biases; use aq_qmv");
  size_t need = 0;
  const cudaError_t e = aq::launch_qmv_noalloc(x, w_q, scales, biases, y, M, N, K, group_size,
                                               dtype, (cudaStream_t)stream, &need);
  if (e == cudaErrorMemoryAllocation)
    return fail(AQ_ERR_UNSUPPORTED,
                "aq_qmv_noalloc: this shape needs %zu bytes of scratch, more than the %zu "
                "bytes it holds; use aq_qmv with a workspace",
                need, aq::kQmvNoallocScratchBytes);
  return cuda_status(e, "aq_qmv_noalloc launch");
}

static aq_status check_batch(const aq_qmv_problem* problems, int count, int64_t M, int bits,
                             int group_size, aq_mode mode, aq_dtype dtype) {
  aq_status st = check_format(bits, group_size, mode, dtype);
  if (st != AQ_OK) return st;
  if (count < 0) return fail(AQ_ERR_INVALID_ARG, "count=%d is negative", count);
  if (count > 0 && !problems) return fail(AQ_ERR_INVALID_ARG, "problems must not be NULL");
  if (M < 1 || M > 16) return fail(AQ_ERR_INVALID_ARG, "aq_qmv_batched takes 1 <= M <= 16 (got %lld)", (long long)M);
  for (int i = 0; i < count; ++i) {
    const aq_qmv_problem& q = problems[i];
    st = check_weight(q.w_q, q.scales, q.biases, q.N, q.K, bits, group_size, mode, dtype);
    if (st == AQ_OK) st = check_mm(q.x, q.y, M, q.N, q.K);
    if (st != AQ_OK) {
      char msg[640];
      snprintf(msg, sizeof(msg), "problem %d: %s", i, g_err);
      return fail(st, "%s", msg);
    }
    if (q.N == 0 || q.K == 0)
      return fail(AQ_ERR_INVALID_ARG, "problem %d: N and K must be positive", i);
    if (!aq::qmv_tc_applies(M, q.N, q.K, bits, group_size, mode, q.scales, q.biases))
      return fail(AQ_ERR_UNSUPPORTED,
                  "problem %d: packed rows and scale rows must be 16-byte multiples and scales / "
                  "biases 16-byte aligned (use aq_qmv for this shape)", i);
  }
  return AQ_OK;
}

aq_status aq_qmv_batched(const aq_qmv_problem* problems, int count, int64_t M, int bits,
                         int group_size, aq_mode mode, aq_dtype dtype, void* workspace,
                         size_t workspace_bytes, aq_stream_t stream) {
  g_err[0] = 0;
  aq_status st = check_batch(problems, count, M, bits, group_size, mode, dtype);
  if (st != AQ_OK) return st;
  if (count == 0) return AQ_OK;
  std::vector<aq::QmvProblemDesc> d((size_t)count);
  for (int i = 0; i < count; ++i)
    d[(size_t)i] = {problems[i].x, problems[i].w_q, problems[i].scales, problems[i].biases,
                    problems[i].y, problems[i].N, problems[i].K};
  if (all_mma(problems, count, M, bits, group_size, mode)) {
    const size_t need = aq::qmv_mma_batched_workspace(d.data(), count, M, group_size);
    if ((st = check_workspace(workspace, workspace_bytes, need)) != AQ_OK) return st;
    return cuda_status(aq::launch_qmv_mma_batched(d.data(), count, M, group_size, dtype,
                                                  workspace, (cudaStream_t)stream),
                       "aq_qmv_batched launch");
  }
  const size_t need = aq::qmv_tc_batched_workspace(d.data(), count, M, bits, group_size);
  if ((st = check_workspace(workspace, workspace_bytes, need)) != AQ_OK) return st;
  return cuda_status(aq::launch_qmv_tc_batched(d.data(), count, M, bits, group_size, mode, dtype,
                                               workspace, (cudaStream_t)stream),
                     "aq_qmv_batched launch");
}

size_t aq_qmv_batched_workspace_size(const aq_qmv_problem* problems, int count, int64_t M,
                                     int bits, int group_size, aq_mode mode) {
  if (!problems || count <= 0 || M < 1 || M > 16 || group_size <= 0) return 0;
  std::vector<aq::QmvProblemDesc> d;
  for (int i = 0; i < count; ++i)
    if (problems[i].N <= 0 || problems[i].K <= 0 || problems[i].K % group_size) return 0;
  if (all_mma(problems, count, M, bits, group_size, mode)) {
    for (int i = 0; i < count; ++i)
      d.push_back({problems[i].x, problems[i].w_q, problems[i].scales, problems[i].biases,
                   problems[i].y, problems[i].N, problems[i].K});
    return aq::qmv_mma_batched_workspace(d.data(), count, M, group_size);
  }
  for (int i = 0; i < count; ++i) {
    if (!aq::qmv_tc_shape_ok(problems[i].N, problems[i].K, bits, group_size, mode)) continue;
    d.push_back({problems[i].x, problems[i].w_q, problems[i].scales, problems[i].biases,
                 problems[i].y, problems[i].N, problems[i].K});
  }
  return d.empty() ? 0 : aq::qmv_tc_batched_workspace(d.data(), (int)d.size(), M, bits, group_size);
}

aq_status aq_qmm(const void* x, const void* w_q, const void* scales, const void* biases,
                 void* y, int64_t M, int64_t N, int64_t K, int bits, int group_size,
                 aq_mode mode, aq_dtype dtype, void* workspace, size_t workspace_bytes,
                 aq_stream_t stream) {
  g_err[0] = 0;
  (void)workspace; (void)workspace_bytes;
  aq_status st = check_weight(w_q, scales, biases, N, K, bits, group_size, mode, dtype);
  if (st != AQ_OK) return st;
  if ((st = check_mm(x, y, M, N, K)) != AQ_OK) return st;
  if (M == 0 || N == 0) return AQ_OK;
  if (K == 0) return zero_output(y, M, N, stream);
  const aq::QmmPlan p = aq::plan_qmm(M, N, K, bits, group_size, mode);
  return cuda_status(aq::launch_qmm(p, x, w_q, scales, biases, y, M, N, K, bits, group_size,
                                    mode, dtype, (cudaStream_t)stream),
                     "aq_qmm launch");
}

// Pointers of gather pair i (byte offsets of the batch strides).
static aq_qmv_problem gather_pair(const void* x, const void* w_q, const void* scales,
                                  const void* biases, void* y, int64_t l, int64_t r, int64_t i,
                                  int64_t M, int64_t N, int64_t K, int bits, int group_size,
                                  aq_mode mode) {
  const int64_t G = K / group_size;
  const int64_t sb = mode == AQ_MODE_FP4 ? 1 : 2;            // bytes per scale / bias
  aq_qmv_problem q;
  q.x = static_cast<const uint8_t*>(x) + l * M * K * 2;
  q.w_q = static_cast<const uint8_t*>(w_q) + r * N * (K * bits / 8);
  q.scales = static_cast<const uint8_t*>(scales) + r * N * G * sb;
  q.biases = biases ? static_cast<const uint8_t*>(biases) + r * N * G * sb : nullptr;
  q.y = static_cast<uint8_t*>(y) + i * M * N * 2;
  q.N = N;
  q.K = K;
  return q;
}

static aq_status check_gather(const int32_t* lhs, const int32_t* rhs, int64_t n_pairs,
                              int64_t x_batch, int64_t w_batch) {
  if (n_pairs < 0 || n_pairs > INT32_MAX)
    return fail(AQ_ERR_INVALID_ARG, "n_pairs=%lld out of range", (long long)n_pairs);
  if (x_batch < 1 || w_batch < 1)
    return fail(AQ_ERR_INVALID_ARG, "x_batch and w_batch must be positive");
  for (int64_t i = 0; i < n_pairs; ++i) {
    const int64_t l = lhs ? lhs[i] : i, r = rhs ? rhs[i] : i;
    if (l < 0 || l >= x_batch || r < 0 || r >= w_batch)
      return fail(AQ_ERR_INVALID_ARG, "pair %lld: indices (%lld, %lld) outside x_batch %lld / w_batch %lld",
                  (long long)i, (long long)l, (long long)r, (long long)x_batch, (long long)w_batch);
  }
  return AQ_OK;
}

// Expert grouping of a gather: the pairs that share weight matrix e, up to
// 16 / M of them per problem, become one problem of Mb rows (the largest
// group's rows; smaller groups are padded with zero rows).  Row maps index x
// as [x_batch * M, K] and y as [n_pairs * M, N].
struct GatherGroups {
  bool use = false;
  int G = 0, Mb = 0;
  std::vector<int64_t> expert;          // weight matrix of each group
  std::vector<int32_t> xmap, ymap;      // G * Mb rows each
};

static GatherGroups group_pairs(const int32_t* lhs, const int32_t* rhs, int64_t n_pairs,
                                int64_t M, int64_t N, int64_t K, int64_t x_batch) {
  GatherGroups gg;
  const int64_t per = 16 / M;                              // pairs per problem
  if (per < 2 || (K * 2) % 16 || (N * 2) % 16 || n_pairs > 65536 || x_batch * M > INT32_MAX)
    return gg;
  // pairs ordered by weight matrix (stable: pair order within a matrix)
  std::vector<int64_t> order((size_t)n_pairs);
  for (int64_t i = 0; i < n_pairs; ++i) order[(size_t)i] = i;
  auto mat = [&](int64_t i) { return rhs ? (int64_t)rhs[i] : i; };
  std::stable_sort(order.begin(), order.end(),
                   [&](int64_t a, int64_t b) { return mat(a) < mat(b); });
  std::vector<std::vector<int64_t>> groups;
  for (size_t q = 0; q < order.size();) {
    const int64_t e = mat(order[q]);
    std::vector<int64_t> g;
    while (q < order.size() && mat(order[q]) == e && (int64_t)g.size() < per) g.push_back(order[q++]);
    gg.expert.push_back(e);
    groups.push_back(std::move(g));
  }
  gg.G = (int)groups.size();
  if (gg.G >= n_pairs) return gg;                          // nothing shared: no gain
  for (auto& g : groups) gg.Mb = std::max(gg.Mb, (int)(g.size() * M));
  gg.xmap.assign((size_t)gg.G * gg.Mb, -1);
  gg.ymap.assign((size_t)gg.G * gg.Mb, -1);
  for (int gi = 0; gi < gg.G; ++gi)
    for (size_t q = 0; q < groups[(size_t)gi].size(); ++q) {
      const int64_t i = groups[(size_t)gi][q];
      const int64_t l = lhs ? lhs[i] : i;
      for (int64_t m = 0; m < M; ++m) {
        const size_t row = (size_t)gi * gg.Mb + q * M + m;
        gg.xmap[row] = (int32_t)(l * M + m);
        gg.ymap[row] = (int32_t)(i * M + m);
      }
    }
  gg.use = true;
  return gg;
}

static size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

// Workspace of the grouped path: the batch's own workspace first (counters in
// the first 64 KB), then the gathered x and the grouped y.
static aq_status run_grouped(const GatherGroups& gg, const void* x, const void* w_q,
                             const void* scales, const void* biases, void* y, int64_t M,
                             int64_t N, int64_t K, int bits, int group_size, aq_mode mode,
                             aq_dtype dtype, void* workspace, size_t workspace_bytes,
                             aq_stream_t stream) {
  const int64_t G = gg.G, Mb = gg.Mb;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  std::vector<aq_qmv_problem> Q((size_t)G);
  for (int64_t g = 0; g < G; ++g) {
    Q[(size_t)g] = gather_pair(x, w_q, scales, biases, y, 0, gg.expert[(size_t)g], 0, Mb, N, K,
                               bits, group_size, mode);
  }
  const size_t need_b = aq_qmv_batched_workspace_size(Q.data(), (int)G, Mb, bits, group_size, mode);
  const size_t off_x = align256(std::max<size_t>(65536, need_b));
  const size_t off_y = off_x + align256((size_t)(G * Mb * K) * 2);
  const size_t need = off_y + align256((size_t)(G * Mb * N) * 2);
  if (!workspace || workspace_bytes < need) return AQ_ERR_WORKSPACE;
  for (int64_t g = 0; g < G; ++g) {
    Q[(size_t)g].x = ws + off_x + (size_t)(g * Mb * K) * 2;
    Q[(size_t)g].y = ws + off_y + (size_t)(g * Mb * N) * 2;
  }
  aq_status st = cuda_status(aq::launch_row_copy(x, ws + off_x, gg.xmap.data(), (int)(G * Mb),
                                                 K * 2, false, (cudaStream_t)stream),
                             "aq_gather_qmm row gather");
  if (st != AQ_OK) return st;
  // The batch reads the gathered x that the launch above writes: no input
  // prefetch for this thread's inner call.
  const int input_prefetch = g_input_prefetch;
  g_input_prefetch = 0;
  st = aq_qmv_batched(Q.data(), (int)G, Mb, bits, group_size, mode, dtype, workspace, off_x,
                      stream);
  g_input_prefetch = input_prefetch;
  if (st != AQ_OK) return st;
  return cuda_status(aq::launch_row_copy(ws + off_y, y, gg.ymap.data(), (int)(G * Mb), N * 2,
                                         true, (cudaStream_t)stream),
                     "aq_gather_qmm row scatter");
}

aq_status aq_gather_qmm(const void* x, const void* w_q, const void* scales, const void* biases,
                        const int32_t* lhs_indices, const int32_t* rhs_indices, void* y,
                        int64_t n_pairs, int64_t M, int64_t N, int64_t K, int64_t x_batch,
                        int64_t w_batch, int bits, int group_size, aq_mode mode, aq_dtype dtype,
                        void* workspace, size_t workspace_bytes, aq_stream_t stream) {
  g_err[0] = 0;
  aq_status st = check_gather(lhs_indices, rhs_indices, n_pairs, x_batch, w_batch);
  if (st != AQ_OK) return st;
  if ((st = check_weight(w_q, scales, biases, N, K, bits, group_size, mode, dtype)) != AQ_OK)
    return st;
  if ((st = check_mm(x, y, M, N, K)) != AQ_OK) return st;
  if (n_pairs == 0 || M == 0 || N == 0) return AQ_OK;
  if (K == 0) return zero_output(y, n_pairs * M, N, stream);
  std::vector<aq_qmv_problem> P((size_t)n_pairs);
  for (int64_t i = 0; i < n_pairs; ++i)
    P[(size_t)i] = gather_pair(x, w_q, scales, biases, y,
                               lhs_indices ? lhs_indices[i] : i, rhs_indices ? rhs_indices[i] : i,
                               i, M, N, K, bits, group_size, mode);
  // Decode-sized pairs whose matrices the batched decode kernels take run as
  // one batch (the unit scheduler walks every pair's row tiles and K-slices);
  // pairs that share a weight matrix are grouped into one problem first when
  // that saves weight reads.  The others, and M > 16, run one call per pair.
  if (M <= 16 && check_batch(P.data(), (int)n_pairs, M, bits, group_size, mode, dtype) == AQ_OK) {
    GatherGroups gg = group_pairs(lhs_indices, rhs_indices, n_pairs, M, N, K, x_batch);
    if (gg.use) {
      st = run_grouped(gg, x, w_q, scales, biases, y, M, N, K, bits, group_size, mode, dtype,
                       workspace, workspace_bytes, stream);
      if (st != AQ_ERR_WORKSPACE) return st;
      g_err[0] = 0;                                        // too small for grouping: per pair
    }
    return aq_qmv_batched(P.data(), (int)n_pairs, M, bits, group_size, mode, dtype, workspace,
                          workspace_bytes, stream);
  }
  g_err[0] = 0;
  for (int64_t i = 0; i < n_pairs; ++i) {
    const aq_qmv_problem& q = P[(size_t)i];
    st = M <= 16 ? aq_qmv(q.x, q.w_q, q.scales, q.biases, q.y, M, N, K, bits, group_size, mode,
                          dtype, workspace, workspace_bytes, stream)
                 : aq_qmm(q.x, q.w_q, q.scales, q.biases, q.y, M, N, K, bits, group_size, mode,
                          dtype, nullptr, 0, stream);
    if (st != AQ_OK) {
      char msg[640];
      snprintf(msg, sizeof(msg), "pair %lld: %s", (long long)i, g_err);
      return fail(st, "%s", msg);
    }
  }
  return AQ_OK;
}

size_t aq_gather_qmm_workspace_size(int64_t n_pairs, int64_t M, int64_t N, int64_t K, int bits,
                                    int group_size, aq_mode mode) {
  if (n_pairs <= 0 || n_pairs > INT32_MAX || M < 1 || M > 16 || N <= 0 || K <= 0 ||
      group_size <= 0 || K % group_size)
    return 0;
  // Sized for either path: the batch (aligned stand-in pointers; the size
  // depends on the shapes only) and one call per pair.
  const void* a = reinterpret_cast<const void*>((uintptr_t)1 << 20);
  std::vector<aq_qmv_problem> P((size_t)n_pairs, aq_qmv_problem{a, a, a, a, const_cast<void*>(a), N, K});
  size_t need = std::max(aq_qmv_batched_workspace_size(P.data(), (int)n_pairs, M, bits, group_size, mode),
                         aq_workspace_size(AQ_OP_QMV, M, N, K, bits, group_size, mode, 1));
  // the expert-grouped path: at most n_pairs problems of at most 16 rows
  if (16 / M >= 2) {
    const size_t b16 = aq_qmv_batched_workspace_size(P.data(), (int)n_pairs, 16, bits, group_size, mode);
    need = std::max(need, align256(std::max<size_t>(65536, b16)) +
                              align256((size_t)(n_pairs * 16 * K) * 2) +
                              align256((size_t)(n_pairs * 16 * N) * 2));
  }
  return need;
}

aq_status aq_qmm_nt(const void* x, const void* w_q, const void* scales, const void* biases,
                    void* y, int64_t M, int64_t N, int64_t K, int bits, int group_size,
                    aq_mode mode, aq_dtype dtype, void* workspace, size_t workspace_bytes,
                    aq_stream_t stream) {
  g_err[0] = 0;
  aq_status st = check_weight(w_q, scales, biases, N, K, bits, group_size, mode, dtype);
  if (st != AQ_OK) return st;
  if (M < 0 || M > kMaxDim) return fail(AQ_ERR_INVALID_ARG, "M=%lld out of range", (long long)M);
  if (M == 0 || K == 0) return AQ_OK;
  if (!y) return fail(AQ_ERR_INVALID_ARG, "y must not be NULL");
  if (!aligned(y, 16)) return fail(AQ_ERR_MISALIGNED, "y must be 16-byte aligned");
  if (N == 0) return zero_output(y, M, K, stream);
  if (!x) return fail(AQ_ERR_INVALID_ARG, "x must not be NULL");
  if (!aligned(x, 2)) return fail(AQ_ERR_MISALIGNED, "x must be 2-byte aligned");
  const size_t need = aq::qmm_nt_workspace(M, N, K, bits);
  if ((st = check_workspace(workspace, workspace_bytes, need)) != AQ_OK) return st;
  return cuda_status(aq::launch_qmm_nt(x, w_q, scales, biases, y, M, N, K, bits, group_size, mode,
                                       dtype, workspace, (cudaStream_t)stream),
                     "aq_qmm_nt launch");
}

aq_status aq_quantize_dequantize_fp(const void* x, void* out, int64_t N, int64_t K, int bits,
                                    int group_size, aq_dtype dtype, aq_stream_t stream) {
  g_err[0] = 0;
  if (dtype != AQ_F16 && dtype != AQ_BF16)
    return fail(AQ_ERR_UNSUPPORTED, "dtype %d is not fp16 (0) or bf16 (1)", (int)dtype);
  if (bits != 4 && bits != 8)
    return fail(AQ_ERR_UNSUPPORTED, "bits %d: elements are E2M1 (4) or E4M3 (8)", bits);
  if (group_size != 16 && group_size != 32)
    return fail(AQ_ERR_UNSUPPORTED, "group_size %d: scales are E8M0 (32) or E4M3 (16)", group_size);
  if (N < 0 || K < 0 || N > kMaxDim || K > kMaxDim)
    return fail(AQ_ERR_INVALID_ARG, "N=%lld K=%lld out of range", (long long)N, (long long)K);
  if (K % 32) return fail(AQ_ERR_INVALID_ARG, "K=%lld is not a multiple of 32", (long long)K);
  if (N == 0 || K == 0) return AQ_OK;
  if (!x || !out) return fail(AQ_ERR_INVALID_ARG, "x and out must not be NULL");
  if (!aligned(x, 2) || !aligned(out, 2)) return fail(AQ_ERR_MISALIGNED, "x and out must be 2-byte aligned");
  return cuda_status(aq::launch_quantize_dequantize_fp(x, out, N, K, bits, group_size, dtype,
                                                       (cudaStream_t)stream),
                     "aq_quantize_dequantize_fp launch");
}

// Workspace of aq_qqmm: the matmul's own first, then the fake-quantized x,
// never inside the first 64 KB (the counters that every call leaves zero, so
// that the buffer still serves the other calls).
static size_t qqmm_mm_bytes(int64_t M, int64_t N, int64_t K, int group_size) {
  const size_t b = M <= 16 ? aq_workspace_size(AQ_OP_QMV, M, N, K, 4, group_size, AQ_MODE_FP4, 1) : 0;
  return std::max((size_t)65536, (b + 255) & ~(size_t)255);
}

aq_status aq_qqmm(const void* x, const void* w_q, const void* scales, void* y, int64_t M,
                  int64_t N, int64_t K, int group_size, aq_dtype dtype, void* workspace,
                  size_t workspace_bytes, aq_stream_t stream) {
  g_err[0] = 0;
  aq_status st = check_weight(w_q, scales, nullptr, N, K, 4, group_size, AQ_MODE_FP4, dtype);
  if (st != AQ_OK) return st;
  if ((st = check_mm(x, y, M, N, K)) != AQ_OK) return st;
  if (M == 0 || N == 0) return AQ_OK;
  if (K == 0) return zero_output(y, M, N, stream);
  if (K % 32) return fail(AQ_ERR_INVALID_ARG, "K=%lld is not a multiple of 32", (long long)K);
  const size_t need = aq_workspace_size(AQ_OP_QQMM, M, N, K, 4, group_size, AQ_MODE_FP4, 1);
  if ((st = check_workspace(workspace, workspace_bytes, need)) != AQ_OK) return st;
  const size_t mb = qqmm_mm_bytes(M, N, K, group_size);
  void* xq = static_cast<uint8_t*>(workspace) + mb;
  if ((st = aq_quantize_dequantize_fp(x, xq, M, K, 4, group_size, dtype, stream)) != AQ_OK)
    return st;
  // The matmul reads the fake-quantized x that the launch above writes, so
  // it must not read x before its dependency wait: input prefetch is off for
  // this thread's inner call.
  const int input_prefetch = g_input_prefetch;
  g_input_prefetch = 0;
  if (M <= 16)
    st = aq_qmv(xq, w_q, scales, nullptr, y, M, N, K, 4, group_size, AQ_MODE_FP4, dtype,
                workspace, mb, stream);
  else
    st = aq_qmm(xq, w_q, scales, nullptr, y, M, N, K, 4, group_size, AQ_MODE_FP4, dtype,
                nullptr, 0, stream);
  g_input_prefetch = input_prefetch;
  return st;
}

int aq_testing_gather_groups(const int32_t* lhs_indices, const int32_t* rhs_indices,
                             int64_t n_pairs, int64_t M, int64_t N, int64_t K, int64_t x_batch,
                             int32_t* xmap, int32_t* ymap, int64_t map_rows, int* rows_per_group) {
  const GatherGroups gg = group_pairs(lhs_indices, rhs_indices, n_pairs, M, N, K, x_batch);
  if (!gg.use) return 0;
  if (rows_per_group) *rows_per_group = gg.Mb;
  const int64_t rows = (int64_t)gg.G * gg.Mb;
  for (int64_t i = 0; i < rows && i < map_rows; ++i) {
    if (xmap) xmap[i] = gg.xmap[(size_t)i];
    if (ymap) ymap[i] = gg.ymap[(size_t)i];
  }
  return gg.G;
}

void aq_testing_set_wait_limit_ns(uint64_t ns) { aq::testing_set_mv_wait_ns(ns); }
void aq_testing_set_start_delay_ns(uint64_t ns) { aq::testing_set_mv_delay_ns(ns); }
void aq_testing_set_qmv_kernel(int which) { g_qmv_kernel.store(which, std::memory_order_relaxed); }
aq_status aq_testing_clear_device_errors(void) {
  g_err[0] = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = aq::testing_clear_device_error_qmv_mma();
  return cuda_status(e, "aq_testing_clear_device_errors");
}

unsigned aq_device_errors(void) {
  unsigned v = 0, w = 0;
  if (aq::read_device_error_qmm(&v) != cudaSuccess) return 0xFFFFFFFFu;
  if (aq::read_device_error_conv(&w) != cudaSuccess) return 0xFFFFFFFFu;
  unsigned t = 0, u = 0;
  if (aq::read_device_error_qmv_tc(&t) != cudaSuccess) return 0xFFFFFFFFu;
  if (aq::read_device_error_qmv_mma(&u) != cudaSuccess) return 0xFFFFFFFFu;
  return v | w | t | u;
}

aq_status aq_qconv2d_nhwc(const void* x, const void* w_q, const void* scales,
                          const void* biases, void* y, int B, int H, int W, int Cin,
                          int Cout, int kh, int kw, int stride_h, int stride_w, int pad_h,
                          int pad_w, int groups, int bits, int group_size, aq_dtype dtype,
                          void* workspace, size_t workspace_bytes, aq_stream_t stream) {
  g_err[0] = 0;
  (void)workspace; (void)workspace_bytes;
  aq_status st = check_format(bits, group_size, AQ_MODE_AFFINE, dtype);
  if (st != AQ_OK) return st;
  if (B < 0 || H < 0 || W < 0 || Cin <= 0 || Cout <= 0 || kh <= 0 || kw <= 0 ||
      stride_h <= 0 || stride_w <= 0 || pad_h < 0 || pad_w < 0 || groups <= 0)
    return fail(AQ_ERR_INVALID_ARG, "conv sizes must be positive (pads >= 0)");
  if (Cin % groups || Cout % groups)
    return fail(AQ_ERR_INVALID_ARG, "Cin=%d and Cout=%d must be multiples of groups=%d", Cin, Cout, groups);
  if ((Cin / groups) % 8)
    return fail(AQ_ERR_UNSUPPORTED, "Cin/groups=%d must be a multiple of 8 (16-byte channel runs)", Cin / groups);
  const int64_t Ho = ((int64_t)H + 2 * pad_h - kh) / stride_h + 1;
  const int64_t Wo = ((int64_t)W + 2 * pad_w - kw) / stride_w + 1;
  if (H + 2 * pad_h < kh || W + 2 * pad_w < kw)
    return fail(AQ_ERR_INVALID_ARG, "kernel %dx%d larger than the padded input", kh, kw);
  const int64_t M = (int64_t)B * Ho * Wo;
  const int64_t Kreal = (int64_t)kh * kw * (Cin / groups);
  const int64_t Kp = (Kreal + group_size - 1) / group_size * group_size;
  if (M > kMaxDim || Kp > kMaxDim || (int64_t)B * H * W * Cin > ((int64_t)1 << 40))
    return fail(AQ_ERR_INVALID_ARG, "conv problem too large");
  if (M == 0) return AQ_OK;
  if (!x || !y || !w_q || !scales || !biases)
    return fail(AQ_ERR_INVALID_ARG, "x, y, w_q, scales and biases must not be NULL");
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(w_q, 16))
    return fail(AQ_ERR_MISALIGNED, "x, y and w_q must be 16-byte aligned");
  if (!aligned(scales, 2) || !aligned(biases, 2))
    return fail(AQ_ERR_MISALIGNED, "scales and biases must be 2-byte aligned");
  return cuda_status(aq::launch_qconv(x, w_q, scales, biases, y, B, H, W, Cin, Cout, kh, kw,
                                      stride_h, stride_w, pad_h, pad_w, groups, bits, group_size,
                                      dtype, (cudaStream_t)stream),
                     "aq_qconv2d_nhwc launch");
}

size_t aq_workspace_size(aq_op op, int64_t M, int64_t N, int64_t K, int bits, int group_size,
                         aq_mode mode, int groups) {
  (void)groups;
  if (M <= 0 || N <= 0 || K <= 0 || group_size <= 0 || K % group_size) return 0;
  if (op == AQ_OP_QMV) {
    if (M > 16) return 0;
    // Which decode kernel runs also depends on the pointers' alignment, so
    // size for either.
    size_t need = 0;
    if (aq::qmv_mma_shape_ok(N, K, bits, group_size, mode))
      need = aq::qmv_mma_workspace(M, N, K, group_size);
    if (aq::qmv_tc_shape_ok(N, K, bits, group_size, mode))
      need = std::max(need, aq::qmv_tc_workspace(M, N, K, bits, group_size));
    return std::max(need, aq::plan_qmv(M, N, K, bits, group_size, mode).ws_bytes);
  }
  if (op == AQ_OP_QQMM) return qqmm_mm_bytes(M, N, K, group_size) + (size_t)(M * K) * 2;
  if (op == AQ_OP_QMM_NT) return aq::qmm_nt_workspace(M, N, K, bits);
  return 0;
}

}  // extern "C"
