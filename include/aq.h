/*
 * aq.h — C ABI of the group-wise affine quantized matmul library for NVIDIA
 * B200 (sm_100a).  libaq.so exports exactly the functions declared here.
 *
 * The operation (sources cited by page title and section):
 *   y = x . dequant(w_q, scales, biases)^T
 * "Add the 3bit packed qmm_t" (quantized_matmul with transpose=true): x is
 * [M, K], the weight has N rows of K elements, y is [M, N].
 *
 * Weight format ("mlx 1.0.0, mlx/backend/cpu/quantized.cpp": quantize,
 * get_pack_factor, get_bytes_per_pack, extract_bits, FP4_LUT,
 * dequantize_scale):
 *   - Affine mode: each row is cut into K/group_size groups of group_size
 *     (32, 64, 128) consecutive elements; group g of row n has one scale
 *     s[n, g] and one bias b[n, g] (dtype T) and codes q in [0, 2^bits - 1];
 *     w_hat = s * q + b.  bits is 2, 3, 4, 5, 6 or 8.
 *   - Packing: row n of w_q is K*bits/8 bytes.  Code k of the row occupies
 *     bits [k*bits, (k+1)*bits) of the row read as a little-endian bit
 *     stream.  For 2/4/8 bits this is 32/bits codes per uint32 word, low bits
 *     first; 3- and 5-bit put 8 codes in 3 and 5 bytes, 6-bit puts 4 codes
 *     in 3 bytes.
 *   - FP4 mode: 4-bit E2M1 codes (2 per byte, low nibble first, value table
 *     +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}) with one uint8 scale per group and no
 *     bias: group_size 32 -> E8M0 scale (bf16 bit pattern s == 0 ? 0x40 :
 *     s << 7, so 255 decodes to +inf), group_size 16 -> FP8 E4M3 scale (OCP
 *     E4M3FN).  The scale is converted to T before use; w_hat = LUT[q] * s_T.
 *   - scales / biases are [N, K/group_size] row-major.
 *
 * Conventions for every entry point:
 *   - Every pointer except aq_last_error's result is a DEVICE pointer owned
 *     by the caller.  The library allocates nothing on the device, frees
 *     nothing and retains no pointer after it returns.
 *   - Every call is asynchronous on `stream` (NULL = legacy default stream):
 *     it validates its arguments on the host, enqueues kernels and returns
 *     without synchronising.  Outputs are overwritten, never accumulated.
 *   - Row-major dense layouts; leading dimensions equal the row lengths.
 *   - Errors: a non-AQ_OK status is returned before anything is enqueued
 *     (argument errors) or right after a launch fails (AQ_ERR_CUDA).  A
 *     thread-local message is available from aq_last_error().  No call
 *     throws, aborts or writes to stdout/stderr.
 *   - Alignment: x, y and w (T data) 16 bytes; w_q 16 bytes; scales and
 *     biases 2 bytes (1 byte in FP4 mode); workspace 256 bytes.
 */
#ifndef AQ_H_
#define AQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AQ_API __attribute__((visibility("default")))
#else
#define AQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream; NULL is the default stream. */
typedef struct CUstream_st* aq_stream_t;

typedef enum {
  AQ_OK = 0,
  AQ_ERR_INVALID_ARG = 1,   /* shape, NULL pointer, or inconsistent sizes */
  AQ_ERR_UNSUPPORTED = 2,   /* bits / group_size / dtype / mode outside the set */
  AQ_ERR_MISALIGNED = 3,    /* a pointer below its required alignment */
  AQ_ERR_CUDA = 4,          /* a CUDA runtime or driver call failed */
  AQ_ERR_WORKSPACE = 5      /* workspace NULL or smaller than aq_workspace_size */
} aq_status;

typedef enum { AQ_F16 = 0, AQ_BF16 = 1 } aq_dtype;

typedef enum {
  AQ_MODE_AFFINE = 0,       /* bits in {2,3,4,5,6,8}, group_size in {32,64,128} */
  AQ_MODE_FP4 = 1           /* bits = 4; group_size 32 (E8M0) or 16 (E4M3); biases NULL */
} aq_mode;

typedef enum {
  AQ_OP_QMV = 0, AQ_OP_QMM = 1, AQ_OP_QCONV2D = 2, AQ_OP_QQMM = 3, AQ_OP_QMM_NT = 4
} aq_op;

/*
 * aq_quantize — affine group quantizer ("mlx 1.0.0, .../quantized.cpp",
 * quantize; "Improvements in the quantizer and dequantization kernel",
 * item 1).  Per group, in fp32 with IEEE division and ties-to-even rint:
 *   lo, hi = min, max;  at_min = |lo| > |hi|
 *   s = max((hi - lo) / (2^bits - 1), 1e-7), negated unless at_min
 *   edge = at_min ? lo : hi;  q0 = rint(edge / s)
 *   if q0 != 0: s = edge / q0, b = edge   (so 0 is exactly code -q0)
 *   else:       b = 0
 *   q = clamp(rint((w - b) / s), 0, 2^bits - 1);  store T(s), T(b)
 * The scale is negative when the bias sits at the maximum.
 *   w      [N, K] T (input)
 *   w_q    [N, K*bits/8] bytes (output)
 *   scales [N, K/group_size] T (output); biases likewise.
 * Requires K % group_size == 0.  Affine mode only.
 */
AQ_API aq_status aq_quantize(const void* w, void* w_q, void* scales, void* biases, int64_t N,
                      int64_t K, int bits, int group_size, aq_dtype dtype,
                      aq_stream_t stream);

/*
 * aq_quantize_fp4 — FP4 (E2M1) quantizer with per-group scales ("mlx 1.0.0,
 * mlx/backend/cpu/quantized.cpp": the steps of fp_quantize_dequantize,
 * to_fp8_e8m0 and to_fp4_e2m1, up to the codes and the scale byte).  It
 * writes the FP4 weights that aq_qmv / aq_qmm / aq_dequantize take in
 * AQ_MODE_FP4.  Per group of group_size consecutive elements of a row, in
 * fp32:
 *   absmax = max |w| (NaN elements ignored);  scale = absmax / 6
 *   group_size 32: byte = E8M0 of scale: 0xFF for NaN / inf, else
 *                  round(log2(scale)) (the exact nearest power of two on a
 *                  log scale; 0 -> -127), clamped to [-127, 127], + 127
 *   group_size 16: byte = E4M3FN of scale (ties to even, saturating at 448)
 *   s = the byte decoded (E8M0: 2^(byte-127), byte 0 -> 2^-127; E4M3FN)
 *   code = E2M1 of (s == 0 ? 0 : w / s): round to nearest (ties to even),
 *          saturating at +-6, sign kept (-0 -> code 8), NaN -> code 7.
 *   w      [N, K] T, row-major;  K a multiple of 32.
 *   codes  [N, K/2] bytes: code k in the low nibble of byte k/2 for even k,
 *          the high nibble for odd k.
 *   scales [N, K/group_size] bytes.
 * Bit-exact with the definition above.  Returns AQ_ERR_UNSUPPORTED for
 * group_size other than 16 / 32 or a dtype other than fp16 / bf16.
 */
AQ_API aq_status aq_quantize_fp4(const void* w, void* codes, void* scales, int64_t N, int64_t K,
                                 int group_size, aq_dtype dtype, aq_stream_t stream);

/*
 * aq_dequantize — writes w_out [N, K] T with every element rounded once
 * (to nearest, ties to even) from the exact value s*q + b (affine) or
 * LUT[q] * s_T (FP4).  Same weight arguments as aq_qmm.
 */
AQ_API aq_status aq_dequantize(const void* w_q, const void* scales, const void* biases, void* w_out,
                        int64_t N, int64_t K, int bits, int group_size, aq_mode mode,
                        aq_dtype dtype, aq_stream_t stream);

/*
 * aq_qmv — y = x . w_hat^T for small M (1 <= M <= 16): the weight-streaming
 * path ("Add the 3bit packed qmm_t", affine_packed_qmv_fast, which keeps the
 * dot product in fp32 and hoists scale and bias out of each group).
 *   x [M, K] T, y [M, N] T.  For every output
 *     y[m, n] = sum_g ( s[n,g] * P[g] + b[n,g] * X[g] ),
 *     P[g] = sum_{k in g} q[n,k] x[m,k],  X[g] = sum_{k in g} x[m,k],
 *   in fp32, with s and b (or the FP4 scale in T) applied in fp32: w_hat is
 *   never rounded to T.
 * When the packed rows (K * bits / 8 bytes) and the rows of scales (K /
 * group_size elements) are 16-byte multiples and scales / biases are
 * 16-byte aligned, the products P and the sums X come from tcgen05 tensor-
 * core MMAs over the exact integer codes, and K may be split over several
 * CTAs whose fp32 partials meet in `workspace`; other shapes run an fp32
 * CUDA-core kernel that needs no workspace.
 * Workspace: aq_workspace_size(AQ_OP_QMV, M, N, K, bits, group_size, mode,
 * 1) bytes, 256-byte aligned, ZERO-FILLED before its first use.  Its first
 * 65536 bytes hold per-tile counters that every call which completes leaves
 * zero again; the rest holds fp32 partial sums that each call writes before
 * it reads them.  So one buffer serves any sequence of calls on one stream;
 * calls that may run at the same time (other streams) need separate
 * buffers.  After a device error (aq_device_errors() != 0) zero it again.
 * Returns AQ_ERR_WORKSPACE when a needed workspace is NULL or too small.
 * Returns AQ_ERR_INVALID_ARG for M outside 1..16.
 */
AQ_API aq_status aq_qmv(const void* x, const void* w_q, const void* scales, const void* biases,
                 void* y, int64_t M, int64_t N, int64_t K, int bits, int group_size,
                 aq_mode mode, aq_dtype dtype, void* workspace, size_t workspace_bytes,
                 aq_stream_t stream);

/* One problem of aq_qmv_batched: y [M, N] = x [M, K] . dequant(w)^T. */
typedef struct aq_qmv_problem {
  const void* x;        /* [M, K] T */
  const void* w_q;      /* [N, K*bits/8] packed codes */
  const void* scales;   /* [N, K/group_size] */
  const void* biases;   /* [N, K/group_size] T (affine), NULL (FP4) */
  void* y;              /* [M, N] T */
  int64_t N, K;
} aq_qmv_problem;

/*
 * aq_qmv_batched — `count` independent aq_qmv problems that share M, bits,
 * group_size, mode and dtype (e.g. the projections of a decode step, or the
 * experts selected for a batch), computed by persistent CTAs that stream the
 * weights of all of them back to back: one launch per 40 problems instead of
 * one per problem.  Each problem's result is the one aq_qmv defines (same
 * fp32 arithmetic).  `problems` is a host array read before the call
 * returns.  Every problem must satisfy the tensor-core conditions of aq_qmv
 * (16-byte packed and scale rows, 16-byte aligned scales / biases, N, K > 0),
 * else AQ_ERR_UNSUPPORTED names it.  Workspace as aq_qmv, sized by
 * aq_qmv_batched_workspace_size.  Outputs must not overlap one another or any
 * input.
 */
AQ_API aq_status aq_qmv_batched(const aq_qmv_problem* problems, int count, int64_t M, int bits,
                                int group_size, aq_mode mode, aq_dtype dtype, void* workspace,
                                size_t workspace_bytes, aq_stream_t stream);

/*
 * aq_qmm_nt — the non-transposed product of a quantized weight ("Add the
 * 3bit packed qmm_t": quantized_matmul with transpose = false, the product
 * its VJP forms for x):
 *   y [M, K] = x [M, N] . w_hat [N, K]
 * with w_q / scales / biases exactly as aq_qmv / aq_qmm take them (N rows of
 * K codes quantized along K), so one stored weight serves both x . w_hat^T
 * and x . w_hat.  x [M, N] T (2-byte aligned), y [M, K] T (16-byte aligned).
 * fp32 arithmetic on the exact w_hat (scale and bias kept as factors of the
 * codes); each y is rounded to T once.  Runs 16 rows of x per launch (the
 * weight is streamed once per 16 rows).  Workspace:
 * aq_workspace_size(AQ_OP_QMM_NT, M, N, K, bits, group_size, mode, 1) bytes
 * under aq_qmv's rules (partial sums after the first 64 KB, which the call
 * leaves untouched).
 */
AQ_API aq_status aq_qmm_nt(const void* x, const void* w_q, const void* scales, const void* biases,
                           void* y, int64_t M, int64_t N, int64_t K, int bits, int group_size,
                           aq_mode mode, aq_dtype dtype, void* workspace, size_t workspace_bytes,
                           aq_stream_t stream);

/*
 * aq_gather_qmm — batched matmul over index pairs ("Add the 3bit packed
 * qmm_t": gather_qmm in the ops and bindings, GatherQMM, and the per-matrix
 * offsets of adjust_matrix_offsets): for pair i,
 *   y[i] [M, N] = x[lhs_indices[i]] [M, K] . dequant(w[rhs_indices[i]])^T
 * e.g. the experts a mixture-of-experts layer routes each token block to.
 *   x        [x_batch, M, K] T;   y [n_pairs, M, N] T
 *   w_q      [w_batch, N, K*bits/8];  scales / biases [w_batch, N, K/group_size]
 *   lhs_indices, rhs_indices: HOST arrays of n_pairs int32 (read before the
 *            call returns; NULL means index i), each in range or
 *            AQ_ERR_INVALID_ARG.
 * Each pair's result is the one aq_qmv (M <= 16) or aq_qmm defines.  Pairs of
 * decode size whose matrices meet aq_qmv_batched's conditions run as one
 * batch (one launch per 40 problems); when pairs share a weight matrix and
 * M <= 8 (and K, N are multiples of 8), up to 16 / M of them form one
 * problem first: their x rows are copied together into the workspace and
 * the problem's y rows copied back (two extra launches), so each matrix is
 * streamed once per call.  The other pairs run one call per pair, and every
 * pair's pointers must then meet that call's alignment rules (the error
 * names the pair).  Workspace: aq_gather_qmm_workspace_size bytes, under
 * aq_qmv's rules.
 */
AQ_API aq_status aq_gather_qmm(const void* x, const void* w_q, const void* scales,
                               const void* biases, const int32_t* lhs_indices,
                               const int32_t* rhs_indices, void* y, int64_t n_pairs, int64_t M,
                               int64_t N, int64_t K, int64_t x_batch, int64_t w_batch, int bits,
                               int group_size, aq_mode mode, aq_dtype dtype, void* workspace,
                               size_t workspace_bytes, aq_stream_t stream);

/* Workspace bytes for aq_gather_qmm with these sizes (0 for M > 16). */
AQ_API size_t aq_gather_qmm_workspace_size(int64_t n_pairs, int64_t M, int64_t N, int64_t K,
                                           int bits, int group_size, aq_mode mode);

/*
 * aq_qmv_noalloc — aq_qmv for callers that cannot allocate device memory or
 * manage a workspace buffer: e.g. code that runs after a serving process has
 * fixed its device memory (no cudaMalloc allowed past start-up), or that has
 * no allocator handle to obtain a workspace from.  The pages have no
 * counterpart: this is the same computation as aq_qmv (the same kernel and
 * result), run on a fixed scratch array inside the library instead of a
 * caller workspace.
 *   Arguments as aq_qmv, minus the workspace.  Only shapes that run the
 *   warp-MMA decode kernel: 4-bit affine weights, 1 <= M <= 16, N, K > 0, K a
 *   multiple of 512 (1024 for group_size 128), 16-byte aligned scales and
 *   biases; others return AQ_ERR_UNSUPPORTED.
 *   Limit: the scratch holds 4 MiB (64 KB of counters plus fp32 split-K
 *   partials).  A shape that needs more returns AQ_ERR_UNSUPPORTED with the
 *   size in aq_last_error(); e.g. every projection of a Llama-3.2-1B-sized
 *   layer at M <= 16 fits.
 *   Allocates nothing: no cudaMalloc / cudaFree and no allocating library
 *   call.  The first call on a device (with that device current) looks up
 *   the scratch array's device address once (cudaGetSymbolAddress); make
 *   that first call before any stream capture.
 *   The scratch is shared by every call on the device: its counters start at
 *   zero and every call that completes leaves them zero; calls whose kernels
 *   may overlap on the GPU (different streams without ordering) race on it.
 *   After a device error (aq_device_errors() != 0) the scratch counters may
 *   be left non-zero: do not use this entry point again in the process.
 */
AQ_API aq_status aq_qmv_noalloc(const void* x, const void* w_q, const void* scales,
                                const void* biases, void* y, int64_t M, int64_t N, int64_t K,
                                int bits, int group_size, aq_mode mode, aq_dtype dtype,
                                aq_stream_t stream);

/* Workspace bytes aq_qmv_batched needs for these problems (0 if none). */
AQ_API size_t aq_qmv_batched_workspace_size(const aq_qmv_problem* problems, int count,
                                            int64_t M, int bits, int group_size, aq_mode mode);

/*
 * aq_qmm — y = x . w_hat^T for any M >= 1 ("Add the 3bit packed qmm_t",
 * affine_packed_qmm_t): each weight tile is dequantized once into T (the
 * values aq_dequantize writes), stored in tensor memory as the A operand of
 * tcgen05 MMAs whose B operand is the x tile (TMA, shared memory), with fp32
 * accumulation in tensor memory.  Arguments as aq_qmv; M may be any size.
 * Needs no workspace (K-splits reduce inside a thread block cluster;
 * workspace may be NULL).
 */
AQ_API aq_status aq_qmm(const void* x, const void* w_q, const void* scales, const void* biases,
                 void* y, int64_t M, int64_t N, int64_t K, int bits, int group_size,
                 aq_mode mode, aq_dtype dtype, void* workspace, size_t workspace_bytes,
                 aq_stream_t stream);

/*
 * aq_qconv2d_nhwc — quantized 2-D convolution as an implicit GEMM
 * ("[Feature] Quantized Convolution 2D - Possible PR?": quantize_weights and
 * img2col followed by quantized_matmul), without materialising im2col.
 *   x [B, H, W, Cin] T;  y [B, Ho, Wo, Cout] T with Ho = (H + 2 pad_h - kh) /
 *   stride_h + 1 (likewise Wo).
 *   Conv group g reads input channels [g Cg, (g+1) Cg), Cg = Cin / groups,
 *   and writes output channels [g Ng, (g+1) Ng), Ng = Cout / groups.
 *   Weight row co (of Cout) is the filter flattened in (kh, kw, Cg) order and
 *   zero-padded to Kp = ceil(kh kw Cg / group_size) * group_size before it is
 *   quantized with aq_quantize(N = Cout, K = Kp): w_q is [Cout, Kp*bits/8]
 *   bytes, scales/biases [Cout, Kp/group_size].
 *   Image borders and the K..Kp-1 pad read zero activations.  No conv bias.
 * Affine mode only.  Workspace rules as aq_qmv (AQ_OP_QCONV2D sizing).
 */
AQ_API aq_status aq_qconv2d_nhwc(const void* x, const void* w_q, const void* scales,
                          const void* biases, void* y, int B, int H, int W, int Cin,
                          int Cout, int kh, int kw, int stride_h, int stride_w, int pad_h,
                          int pad_w, int groups, int bits, int group_size, aq_dtype dtype,
                          void* workspace, size_t workspace_bytes, aq_stream_t stream);

/*
 * aq_quantize_dequantize_fp — fake quantization of activations ("mlx 1.0.0,
 * mlx/backend/cpu/quantized.cpp", fp_quantize_dequantize: the step that
 * QQMatmul applies to x).  Per group of group_size consecutive elements of a
 * row, in fp32:
 *   scale = absmax / (bits == 4 ? 6 : 448)   (NaN elements ignored)
 *   s     = scale through its byte and back: E8M0 for group_size 32, E4M3FN
 *           for 16 (the same encodings as aq_quantize_fp4)
 *   e     = s == 0 ? 0 : x / s
 *   out   = T(s * v), v = the E2M1 value of e (bits 4; NaN -> 6) or its
 *           E4M3FN value (bits 8; ties to even, saturating at 448, NaN stays
 *           NaN); one fp32 multiplication, one rounding to T.
 *   x, out [N, K] T row-major (out may equal x); K a multiple of 32.
 * Bit-exact with the definition.  AQ_ERR_UNSUPPORTED for bits other than
 * 4 / 8, group_size other than 16 / 32, or a dtype other than fp16 / bf16.
 */
AQ_API aq_status aq_quantize_dequantize_fp(const void* x, void* out, int64_t N, int64_t K,
                                           int bits, int group_size, aq_dtype dtype,
                                           aq_stream_t stream);

/*
 * aq_qqmm — W4A4 matmul, y = fq(x) . w_hat^T ("mlx 1.0.0,
 * mlx/backend/cpu/quantized.cpp", QQMatmul::eval_cpu: x fake-quantized with
 * the weights' FP4 format, then the FP4 matmul; the page runs it for one row
 * of x, this call for any M).  fq is aq_quantize_dequantize_fp with bits 4 and
 * the weights' group_size; w_q / scales are FP4 weights as aq_qmv / aq_qmm
 * take them (aq_quantize_fp4 writes them).  x [M, K] T, y [M, N] T, K a
 * multiple of 32.  Two launches on `stream`: the fake quantization into the
 * workspace, then aq_qmv (M <= 16) or aq_qmm.  The matmul tolerance is
 * aq_qmv's / aq_qmm's over fq(x).
 * Workspace: aq_workspace_size(AQ_OP_QQMM, M, N, K, 4, group_size,
 * AQ_MODE_FP4, 1) bytes, 256-byte aligned, under aq_qmv's rules (zero-filled
 * before its first use): aq_qmv's workspace first (M <= 16), then fq(x),
 * which never starts inside the first 64 KB (the counters that every call
 * leaves zero).  So one buffer serves aq_qmv and aq_qqmm calls on one
 * stream.
 */
AQ_API aq_status aq_qqmm(const void* x, const void* w_q, const void* scales, void* y, int64_t M,
                         int64_t N, int64_t K, int group_size, aq_dtype dtype, void* workspace,
                         size_t workspace_bytes, aq_stream_t stream);

/*
 * aq_workspace_size — bytes of workspace the given call needs (0 if none).
 * For AQ_OP_QCONV2D pass M = B*Ho*Wo, N = Cout / groups, K = Kp and the
 * number of conv groups in `groups`; for the others pass groups = 1 (and for
 * AQ_OP_QQMM bits = 4, mode = AQ_MODE_FP4).
 */
AQ_API size_t aq_workspace_size(aq_op op, int64_t M, int64_t N, int64_t K, int bits, int group_size,
                         aq_mode mode, int groups);

/*
 * Device-side error bits accumulated since the library was loaded on the
 * current device (0 = none).  Bit 0: a kernel's bounded wait on an mbarrier
 * timed out (after 2 s); the kernel stopped, freed its tensor memory and left
 * its output incomplete.  Synchronises with the device (reads a __device__
 * variable).  Returns 0xFFFFFFFF if the read itself fails.
 */
AQ_API unsigned aq_device_errors(void);

/*
 * Weight prefetch across kernel boundaries (a setting of the CALLING THREAD,
 * default 0 = off; it affects only the calls this thread makes afterwards).
 * Every qmv / qmm / conv kernel is launched with programmatic dependent
 * launch, so it may start while the previous kernel on its stream is still
 * running; it always waits for that kernel before reading x or writing y
 * and the workspace.  With prefetch on, it also streams w_q, scales and
 * biases before that wait, which hides most of a small matmul's start-up
 * behind the previous kernel.  Turn it on only when no kernel launched just
 * before a matmul on the same stream writes that matmul's weights (e.g. not
 * directly after aq_quantize of the same weights without a synchronising
 * operation in between).
 */
AQ_API void aq_set_weight_prefetch(int enable);
AQ_API int aq_get_weight_prefetch(void);

/*
 * Input prefetch (a setting of the calling thread, default 0 = off).  With
 * it on, a matmul that starts while the previous kernel on its stream is
 * still running also reads x before waiting for that kernel; it still waits
 * before writing y, so y is ordered after everything earlier on the stream.
 * Turn it on only when no kernel that may still be running when a matmul
 * starts writes that matmul's x: for instance calls whose x were all written
 * before the first of them was launched (projections that share an input,
 * experts of one batch, a sweep over fixed activations).
 */
AQ_API void aq_set_input_prefetch(int enable);
AQ_API int aq_get_input_prefetch(void);

/* Message for the last non-AQ_OK status on the calling thread ("" if none). */
AQ_API const char* aq_last_error(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
AQ_API int aq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* AQ_H_ */
