// qmv_tc.cu — decode-sized quantized matmul (1 <= M <= 16 rows of x) on the
// tensor cores, with the scale and bias applied in fp32 per group:
//   y[m, n] = sum_g ( s[n,g] * sum_{k in g} q[n,k] x[m,k]  +  b[n,g] * sum_{k in g} x[m,k] )
// for one problem (aq_qmv) or for a list of independent problems in one
// launch (aq_qmv_batched).  4-bit affine weights whose K is a multiple of the
// 512-column sub-slice run the warp-MMA kernel of qmv_mma.cu instead; this
// kernel serves the other widths (2, 3, 5, 6, 8 bits), FP4 and the other
// shapes with 16-byte packed and scale rows.
//
// Prior art: affine_packed_qmv_fast in "Add the 3bit packed qmm_t" keeps the
// dot product in fp32 and hoists scale and bias out of each group (result +=
// s * accum + b * sum); the FP4 path of "mlx 1.0.0, .../quantized.cpp"
// (fp_qmm_t) hoists the group scale the same way.  This kernel keeps that
// arithmetic and moves the inner products onto the tensor cores:
//   * The codes themselves are the MMA's A operand: every code is an integer
//     that T holds exactly, so the 128 x 16 tcgen05 MMAs of one group form
//     sum_k q x with exact products and fp32 accumulation, into that group's
//     own TMEM slot.  Under bf16 (widths up to 6) the operand is the bit
//     pattern 0x4300 | q, i.e. 128 + q, and the epilogue uses b - 128 s in
//     place of b; fp16 codes and 8-bit bf16 codes are converted to the exact
//     integer.
//   * The epilogue warps (one weight row per thread, its TMEM lane) read each
//     group's 16-column result and apply s and b in fp32 FMAs to it and to
//     the group's x sums.  w_hat is never rounded to T.
// Work decomposition, B200-first:
//   * A unit is 128 weight rows x one K-slice of one problem.  CTAs are
//     persistent (2 per SM, grid <= 2 * SMs) and walk the units round-robin;
//     the weight, scale and x rings run on across unit boundaries, so the
//     weight stream does not drain between units or problems.
//   * A 128 x 16 x 16 MMA costs a warp about 90 cycles to issue whatever its
//     N, so two warps per CTA issue them (groups alternate between the two):
//     four issuers per SM keep up with the weight stream at HBM speed.
//   * Roles: warp 0 streams packed weight chunks (128 rows x 128 bytes,
//     128-byte swizzle) and scale/bias chunks (128 rows x 16 bytes) by TMA in
//     K order; warps 1-2 issue the MMAs (warp 1 owns TMEM); warps 3-6 turn
//     codes into A operands in TMEM (tcgen05.st) and also prepare x: each
//     thread copies one 16-byte run of the 16-row x tile by cp.async two
//     stages ahead (every CTA reads the same few lines of x, which the LSU
//     path serves much better than TMA boxes queued behind the weights), then
//     sums it into per-group row sums and, for 2- and 4-bit codes, reorders it
//     in place to the order in which the codes are unpacked (the unpack then
//     needs one shift and one logic op per pair of codes); warps 7-10 run the
//     epilogue.
//   * K-slices of a row tile reduce through the caller's workspace: every
//     slice stores its fp32 partial rows, and the last slice to arrive (a
//     per-warp counter) adds the slices in slice order and writes y, then
//     resets the counter.  The order of the sum does not depend on which
//     slice arrives last.
//   * Every mbarrier wait is bounded (2 s); a timeout sets a device error
//     bit, every role stops issuing work, TMA copies in flight are waited for
//     (bounded) and the CTA frees its TMEM.
#include <algorithm>
#include <atomic>
#include <climits>

#include "qmm_kernel.cuh"

namespace aq {
namespace {

constexpr int kDecMaxProblems = 40;     // problems per launch of the batched entry
// Tile counters at the start of the workspace (4 per split row tile); the
// fp32 partials follow, so no call's partials ever overlap any call's counters.
constexpr int kDecMaxSplitTiles = 4096;
constexpr int64_t kDecCntWords = 4 * kDecMaxSplitTiles;

struct DecProblem {
  CUtensorMap w;        // [N, K*bits/8] u8, box {128 bytes, 128 rows}, 128-byte swizzle
  CUtensorMap s;        // [N, G] scales, box {16 bytes, 128 rows}
  CUtensorMap b;        // [N, G] biases (affine), likewise
  const void* x;        // [M, K] T
  void* y;              // [M, N] T
  int N, K;
  int splits;           // K-slices per row tile
  int kslice;           // K columns per slice (a multiple of 64 and of group_size)
  int cnt0;             // first tile counter (in units of 4 words) of this problem
  int pad_;
  int64_t ws_part;      // word offset of the fp32 partials
};

template <int P>
struct DecParams {
  DecProblem prob[P];
  int unit_end[P];      // units of problems 0..p (inclusive prefix sums)
  int count;            // problems in this launch
  int M;
  int gs_log2;
  int weights_early;    // issue weight / scale loads before the dependency wait
  int x_early;          // issue x loads before the dependency wait
  uint32_t* ws;         // workspace (counters, then partials); NULL when no problem splits K
};

struct DecShape {
  static constexpr int kWarpLoad = 0, kWarpMma0 = 1, kMmaWarps = 2, kWarpDq0 = 3, kWarpEp0 = 7;
  static constexpr int kThreads = 32 * 11;
  static constexpr int kST = 5;                       // A stages in TMEM, 64 K each
  static constexpr int kXS = 7;                       // x tiles (16 rows x 64 columns, 2 KB)
  static constexpr int kWS = 4;                       // weight chunk slots, 16 KB each
  static constexpr int kSS = 4;                       // scale chunk slots, 4 KB each
  // x-sum slots (per group: [16 rows] fp32).  A slot is rewritten 32 groups
  // later, which the stage and D rings order after the epilogue's read of it
  // (the writer has seen the MMAs of 5 stages back, which waited for the
  // epilogue to finish 6 groups before those): no barrier of its own.
  static constexpr int kXGS = 32;
  static constexpr int kDS = 6;                       // D slots (one group each, 16 TMEM columns)
  static constexpr int kWChunk = kRowsW * 128;
  static constexpr int kSChunk = kRowsW * 16 * 2;
  static constexpr int kXTile = 16 * kBK * 2;
  static constexpr int kWOff = 0;
  static constexpr int kXOff = kWOff + kWS * kWChunk;
  static constexpr int kSOff = kXOff + kXS * kXTile;
  static constexpr int kXsOff = kSOff + kSS * kSChunk;
  static constexpr int kDataBytes = kXsOff + kXGS * 16 * 4;
  // barriers: A full (codes and x), stage empty [kST]; w full/empty [kWS];
  // s full/empty [kSS]; d full/empty [kDS]; done [2]
  static constexpr int kBars = 2 * kST + 2 * kWS + 2 * kSS + 2 * kDS + kMmaWarps;
  static constexpr int kSmem = 1024 + kDataBytes + 1024;
  // TMEM (256 columns, two CTAs per SM): A stages in [0, 32 kST), D slots of
  // 16 columns from kDCol0.
  static constexpr int kTmemCols = 256;
  static constexpr int kDCol0 = 32 * kST;
  static_assert(kDCol0 + 16 * kDS <= kTmemCols, "TMEM columns");
  static_assert(kBars * 8 + 16 <= 1024, "barrier area");
  static_assert(2 * kSmem <= 228 * 1024, "two CTAs per SM");
};

// The A operand holds code + kOff exactly: under bf16 the pattern 0x4300 | q
// is 128 + q for q < 128; otherwise the exact code.
template <typename T, int BITS, bool FP4> struct CodeA {
  static constexpr bool kMagic = !FP4 && std::is_same<T, __nv_bfloat16>::value && BITS <= 6;
  static constexpr float kOff = kMagic ? 128.0f : 0.0f;
  // 2- and 4-bit codes are unpacked as (code i, code i + 8 / 4) pairs; the
  // x-prep warp reorders x to match.
  static constexpr bool kPermX = !FP4 && (BITS == 2 || BITS == 4);
};

struct Unit {
  int p, tile, slice, n0, k0, k1;
};

template <int P>
__device__ __forceinline__ Unit unit_at(const DecParams<P>& pr, int u) {
  int p = 0;
#pragma unroll 1
  for (; p + 1 < pr.count && u >= pr.unit_end[p]; ++p) {}
  const int v = u - (p ? pr.unit_end[p - 1] : 0);
  const DecProblem& q = pr.prob[p];
  Unit r;
  r.p = p;
  r.tile = v / q.splits;
  r.slice = v - r.tile * q.splits;
  r.n0 = r.tile * kRowsW;
  r.k0 = r.slice * q.kslice;
  r.k1 = min(q.K, r.k0 + q.kslice);
  return r;
}

// A operand pair J (0..3) of the 8 codes that word-chunk C of a row's 64
// codes covers.  2-bit and 4-bit: code i of a word with code i + 16/BITS
// (one shift and one logic op per pair; x is reordered to match); other
// widths: codes (2J, 2J+1) in K order.
template <typename T, int BITS, int C, int J>
__device__ __forceinline__ uint32_t a_pair(const Packed<BITS>& p) {
  constexpr bool kMagic = CodeA<T, BITS, false>::kMagic;
  constexpr int k0 = 8 * C + 2 * J;
  if constexpr (BITS == 8 && std::is_same<T, __nv_bfloat16>::value) {
    // 128 + q does not fit bf16's significand for q >= 128: convert exactly
    return Pair<T>::from_f2(u_to_f_exact(code_at<8, k0>(p.w)), u_to_f_exact(code_at<8, k0 + 1>(p.w)));
  } else {
    uint32_t v;
    if constexpr (BITS == 4) {
      // word C holds codes 8C + i at bits 4i: pair (i, i + 4) is (w >> 4i) & 0x000F000F
      v = ((p.w[C] >> (4 * J)) & 0x000F000Fu) | Pair<T>::kMagic;
    } else if constexpr (BITS == 2) {
      // word C/2 holds codes 16(C/2) + i at bits 2i: pair (i, i + 8) is (w >> 2i) & 0x00030003
      v = ((p.w[C >> 1] >> (2 * (4 * (C & 1) + J))) & 0x00030003u) | Pair<T>::kMagic;
    } else {
      v = code_at<BITS, k0>(p.w) | (code_at<BITS, k0 + 1>(p.w) << 16) | Pair<T>::kMagic;
    }
    if constexpr (kMagic) return v;
    else return Pair<T>::sub_magic(v);
  }
}

// Chunk C's four pairs into o[4 (C - C0) ...].
template <typename T, int BITS, bool FP4, int C, int C0 = 0>
__device__ __forceinline__ void a_chunk(const Packed<BITS>& p, uint32_t (&o)[16]) {
  constexpr int i = 4 * (C - C0);
  if constexpr (FP4) {
    fp4_quad<T>(p.w[C], o[i], o[i + 1]);
    fp4_quad<T>(p.w[C] >> 16, o[i + 2], o[i + 3]);
  } else {
    o[i] = a_pair<T, BITS, C, 0>(p);
    o[i + 1] = a_pair<T, BITS, C, 1>(p);
    o[i + 2] = a_pair<T, BITS, C, 2>(p);
    o[i + 3] = a_pair<T, BITS, C, 3>(p);
  }
}

// x in the order a_pair produces codes: within each run of 16 / BITS * 2
// elements (8 for 4-bit, 16 for 2-bit) element i is followed by element
// i + half.  `lo` and `hi` are the two 16-byte runs (2-bit) or the same run.
__device__ __forceinline__ void perm_x4(uint4& v) {
  const uint32_t a = __byte_perm(v.x, v.z, 0x5410), b = __byte_perm(v.x, v.z, 0x7632);
  const uint32_t c = __byte_perm(v.y, v.w, 0x5410), d = __byte_perm(v.y, v.w, 0x7632);
  v = make_uint4(a, b, c, d);
}
__device__ __forceinline__ void perm_x2(uint4& lo, uint4& hi) {
  const uint4 l = lo, h = hi;
  lo = make_uint4(__byte_perm(l.x, h.x, 0x5410), __byte_perm(l.x, h.x, 0x7632),
                  __byte_perm(l.y, h.y, 0x5410), __byte_perm(l.y, h.y, 0x7632));
  hi = make_uint4(__byte_perm(l.z, h.z, 0x5410), __byte_perm(l.z, h.z, 0x7632),
                  __byte_perm(l.w, h.w, 0x5410), __byte_perm(l.w, h.w, 0x7632));
}

// Sum of eight T values held in a 16-byte run, in fp32 (fixed order).
template <typename T>
__device__ __forceinline__ float sum8(uint4 v) {
  float s = 0.0f;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      s += __uint_as_float(w[i] << 16);
      s += __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      s += f.x;
      s += f.y;
    }
  }
  return s;
}

// One row's 64 codes at byte `off` of a unit whose first weight chunk is
// global chunk `cbase`, from the swizzled chunk ring.
template <int BITS>
__device__ __forceinline__ void load_codes(Packed<BITS>& pk, const uint8_t* wring, int cbase,
                                           int off, int r) {
  constexpr int kB = 8 * BITS;
  constexpr int U = (kB % 16 == 0) ? 16 : 8;
#pragma unroll
  for (int u = 0; u < kB / U; ++u) {
    const int o = off + U * u;
    const uint8_t* src = wring + ((cbase + (o >> 7)) % DecShape::kWS) * DecShape::kWChunk +
                         wchunk_off(o & 127, r);
    if constexpr (U == 16) {
      const uint4 v = *reinterpret_cast<const uint4*>(src);
      pk.w[4 * u] = v.x; pk.w[4 * u + 1] = v.y; pk.w[4 * u + 2] = v.z; pk.w[4 * u + 3] = v.w;
    } else {
      const uint2 v = *reinterpret_cast<const uint2*>(src);
      pk.w[2 * u] = v.x; pk.w[2 * u + 1] = v.y;
    }
  }
}

// Element e (0..7) of eight 16-bit T values, as float.
template <typename T>
__device__ __forceinline__ float t_elem(uint4 v, int e) {
  const uint32_t w = (e & 4) ? ((e & 2) ? v.w : v.z) : ((e & 2) ? v.y : v.x);
  const uint32_t h = (e & 1) ? (w >> 16) : (w & 0xFFFFu);
  if constexpr (std::is_same<T, __nv_bfloat16>::value) return __uint_as_float(h << 16);
  else return __half2float(__ushort_as_half((unsigned short)h));
}
__device__ __forceinline__ uint32_t byte_elem(uint4 v, int e) {
  const uint32_t w = (e & 8) ? ((e & 4) ? v.w : v.z) : ((e & 4) ? v.y : v.x);
  return (w >> (8 * (e & 3))) & 0xFFu;
}

// Wait for the last issued phase of every slot of a TMA ring (bounded), so
// that no copy is still writing shared memory when the CTA exits.
__device__ __forceinline__ void drain_ring(const uint64_t* bars, int slots, int issued,
                                           volatile int* abort_flag) {
  for (int c = issued - 1; c >= 0 && c >= issued - slots; --c) {
    const uint32_t bar = smem_u32(bars + (c % slots));
    const uint32_t par = (c / slots) & 1;
    if (mbar_try_wait(bar, par)) continue;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, par))
      if (globaltimer_ns() - t0 > 1000000000ull) { *abort_flag = 1; break; }
  }
}

template <typename T, int BITS, bool FP4, int P>
__global__ void __launch_bounds__(DecShape::kThreads, 2)
qmv_tc_kernel(const __grid_constant__ DecParams<P> pr) {
  using S = DecShape;
  constexpr int ST = S::kST, WS = S::kWS, SS = S::kSS, XGS = S::kXGS, DS = S::kDS;
  constexpr int NMMA = S::kMmaWarps;
  constexpr int kPB = 8 * BITS;                           // packed bytes per row per 64 codes
  constexpr int SGC = FP4 ? 16 : 8;                       // groups per scale chunk (16 bytes)
  constexpr float kOff = CodeA<T, BITS, FP4>::kOff;
  constexpr bool kPermX = CodeA<T, BITS, FP4>::kPermX;
  constexpr bool kSums = !FP4;                            // the bias term needs the x sums
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* wring = smem + S::kWOff;
  uint8_t* xring = smem + S::kXOff;
  uint8_t* sring = smem + S::kSOff;
  float* xsring = reinterpret_cast<float*>(smem + S::kXsOff);   // [XGS][16]: x sums per group
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kDataBytes);
  uint64_t* full_a = bars;                                // A stage and x tile ready (count 4)
  uint64_t* empty_st = full_a + ST;                       // MMA warps: A slot free (count 2)
  uint64_t* full_w = empty_st + ST;
  uint64_t* empty_w = full_w + WS;
  uint64_t* full_s = empty_w + WS;
  uint64_t* empty_s = full_s + SS;
  uint64_t* full_d = empty_s + SS;
  uint64_t* empty_d = full_d + DS;
  uint64_t* done_bar = empty_d + DS;                      // [NMMA]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + S::kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto B = [](uint64_t* b, int i) { return smem_u32(b + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = pr.unit_end[pr.count - 1];
  const int gs = 1 << pr.gs_log2;
  const int M = pr.M;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(B(full_a, i), 4);
      mbar_init(B(empty_st, i), NMMA);
    }
    for (int i = 0; i < WS; ++i) { mbar_init(B(full_w, i), 1); mbar_init(B(empty_w, i), 4); }
    for (int i = 0; i < SS; ++i) { mbar_init(B(full_s, i), 1); mbar_init(B(empty_s, i), 4); }
    for (int i = 0; i < DS; ++i) { mbar_init(B(full_d, i), 1); mbar_init(B(empty_d, i), 4); }
    for (int i = 0; i < NMMA; ++i) mbar_init(B(done_bar, i), 1);
    *abort_flag = 0;
    fence_mbar_init();
    if constexpr (P == 1) {
      prefetch_tensormap(&pr.prob[0].w);
      prefetch_tensormap(&pr.prob[0].s);
      if constexpr (!FP4) prefetch_tensormap(&pr.prob[0].b);
    }
  }
  if (warp == S::kWarpMma0) {
    tmem_alloc(smem_u32(tmem_slot), S::kTmemCols);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();

  if (warp == S::kWarpLoad) {
    // ------------------------------------------ weight and scale chunks
    int cw = 0, cs = 0;                                   // chunks issued (global)
    if (lane == 0) {
      if (!pr.weights_early) pdl_wait();
      const uint64_t pol = l2_policy_evict_first();
      bool ok = true;
      for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
        const Unit un = unit_at(pr, u);
        const DecProblem& q = pr.prob[un.p];
        if constexpr (P > 1) {
          prefetch_tensormap(&q.w);
          prefetch_tensormap(&q.s);
          if constexpr (!FP4) prefetch_tensormap(&q.b);
        }
        const int wb0 = un.k0 * BITS / 8;                 // a multiple of 128 bytes (host plan)
        const int nwc = ((un.k1 - un.k0) * BITS / 8 + 127) >> 7;
        const int sc0 = (un.k0 >> pr.gs_log2) / SGC;
        const int nsc = (((un.k1 - 1) >> pr.gs_log2) / SGC) - sc0 + 1;
        int c = 0, j = 0;
        while (ok && (c < nwc || j < nsc)) {
          // K position (codes from k0) where each chunk starts; weight first on a tie
          const int kw = c < nwc ? (int)((int64_t)c * 1024 / BITS) : INT_MAX;
          const int ks = j < nsc ? (sc0 + j) * SGC * gs - un.k0 : INT_MAX;
          if (kw <= ks) {
            const int slot = cw % WS;
            ok = mbar_wait(B(empty_w, slot), ((cw / WS) & 1) ^ 1, abort_flag);
            if (!ok) break;
            mbar_arrive_expect_tx(B(full_w, slot), S::kWChunk);
            tma_load_2d_hint(smem_u32(wring + slot * S::kWChunk), &q.w, B(full_w, slot),
                             wb0 + 128 * c, un.n0, pol);
            ++c; ++cw;
          } else {
            const int slot = cs % SS;
            ok = mbar_wait(B(empty_s, slot), ((cs / SS) & 1) ^ 1, abort_flag);
            if (!ok) break;
            const uint32_t dst = smem_u32(sring + slot * S::kSChunk);
            mbar_arrive_expect_tx(B(full_s, slot), FP4 ? kRowsW * 16 : 2 * kRowsW * 16);
            tma_load_2d_hint(dst, &q.s, B(full_s, slot), (sc0 + j) * SGC, un.n0, pol);
            if constexpr (!FP4)
              tma_load_2d_hint(dst + kRowsW * 16, &q.b, B(full_s, slot), (sc0 + j) * SGC, un.n0, pol);
            ++j; ++cs;
          }
        }
      }
      drain_ring(full_w, WS, cw, abort_flag);
      drain_ring(full_s, SS, cs, abort_flag);
    }
    __syncwarp();
  } else if (warp >= S::kWarpMma0 && warp < S::kWarpMma0 + NMMA) {
    // ------------------------------------------------------- MMA issuers
    // Both warps visit every stage (warp-uniform waits); warp w issues the
    // MMAs of the groups g with g % 2 == w from an elected lane into the
    // group's D slot, and both release the stage with a commit.
    const int w = warp - S::kWarpMma0;
    constexpr uint32_t idesc = idesc_f16(std::is_same<T, __nv_bfloat16>::value, kRowsW, 16);
    int js = 0, gi = 0;                                   // stages and groups (global)
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      const Unit un = unit_at(pr, u);
      const int ns = (un.k1 - un.k0 + kBK - 1) / kBK;
      const int ng = (un.k1 - un.k0) >> pr.gs_log2;
      for (int st = 0; st < ns; ++st, ++js) {
        const int a = js % ST;
        ok = __all_sync(0xffffffffu, mbar_wait(B(full_a, a), (js / ST) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_col = tmem + (uint32_t)(32 * a);
        const uint32_t x_addr = smem_u32(xring + (js % S::kXS) * S::kXTile);
        // the groups of this stage: one (gs >= 64) or 64 / gs
        int g_lo, g_hi;
        if (gs >= kBK) {
          g_lo = st / (gs / kBK);
          g_hi = g_lo + 1;
        } else {
          g_lo = st * (kBK / gs);
          g_hi = min(ng, g_lo + kBK / gs);
        }
        for (int g = g_lo; g < g_hi && ok; ++g) {
          const int gg = gi + g;
          if ((gg % NMMA) != w) continue;
          const int slot = gg % DS;
          const bool first = gs >= kBK ? (st % (gs / kBK)) == 0 : true;
          const bool last = gs >= kBK ? ((st + 1) % (gs / kBK)) == 0 : true;
          if (first) {
            ok = __all_sync(0xffffffffu,
                            mbar_wait(B(empty_d, slot), ((gg / DS) & 1) ^ 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
          }
          // 16-column K chunks of this group within the stage
          const int kc0 = gs >= kBK ? 0 : (g - g_lo) * (gs / 16);
          const int kcn = gs >= kBK ? kBK / 16 : gs / 16;
          const uint32_t d_col = tmem + (uint32_t)(S::kDCol0 + 16 * slot);
          if (elect_one()) {
            for (int kc = kc0; kc < kc0 + kcn; ++kc)
              mma_f16_tmem_a(d_col, a_col + 8 * kc, sdesc_sw128(x_addr + kc * 32), idesc,
                             (first && kc == kc0) ? 0u : 1u);
            if (last) mma_commit(B(full_d, slot));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) mma_commit(B(empty_st, a));
        __syncwarp();
      }
      gi += ng;
    }
    // every MMA issued has completed before TMEM is freed
    if (elect_one()) mma_commit(B(done_bar, w));
    __syncwarp();
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(B(done_bar, w), 0))
      if (globaltimer_ns() - t0 > 1000000000ull) { *abort_flag = 1; break; }
  } else if (warp >= S::kWarpDq0 && warp < S::kWarpEp0) {
    // ------------------------------------------------------- code unpack and x
    // One weight row per thread (its TMEM lane): 64 codes per stage into the
    // A stage in TMEM.  The same thread also owns one 16-byte run of x per
    // stage: t = 32 (warp % 4) + lane is row t / 8, run t % 8 of the 16-row x
    // tile (rows below M only; other rows feed outputs that are never read).
    // The run is copied by cp.async kXAhead stages ahead into the x ring,
    // then summed and (2-/4-bit codes) reordered in place to the order in
    // which the codes are unpacked, so x is prepared by 128 threads in
    // parallel with the codes.  Stage js uses x slot js % kXS; the x ring is
    // deeper than the stage ring by kXAhead, so a slot is free once the stage
    // ring's own wait has seen the MMAs of stage js - kST complete.
    constexpr int kXAhead = S::kXS - S::kST;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int xrow = r >> 3, xrun = r & 7;
    const bool xmine = xrow < M;
    int js = 0, cbase = 0, w_ready = 0, w_freed = 0, gx = 0;
    float carry = 0.f;                                    // first stage of a 128-column group
    // x issue cursor: unit lu, its x, K and end column, next column lk
    int lu = blockIdx.x, lk = 0, lK = 0, lk1 = 0, issued = 0;
    const T* lxp = nullptr;
    auto x_unit = [&]() {
      const Unit ul = unit_at(pr, lu);
      const DecProblem& ql = pr.prob[ul.p];
      lxp = reinterpret_cast<const T*>(ql.x);
      lK = ql.K;
      lk = ul.k0;
      lk1 = ul.k1;
    };
    auto x_issue = [&]() {
      const int col = lk + 8 * xrun;
      if (xmine && col < lK)
        cp_async_16(smem_u32(xring + (issued % S::kXS) * S::kXTile + xrow * 128 +
                             ((xrun ^ (xrow & 7)) << 4)),
                    lxp + (int64_t)xrow * lK + col);
      cp_async_commit();                                  // one group per stage, even if empty
      ++issued;
      lk += kBK;
      if (lk >= lk1) {
        lu += gridDim.x;
        if (lu < total) x_unit();
      }
    };
    if (lu < total) x_unit();
    if (!pr.x_early) pdl_wait();                          // x may come from the previous kernel
    for (int i = 0; i < kXAhead && lu < total; ++i) x_issue();
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      const Unit un = unit_at(pr, u);
      const int ns = (un.k1 - un.k0 + kBK - 1) / kBK;
      const int ngu = (un.k1 - un.k0) >> pr.gs_log2;
      const int nwc = ((un.k1 - un.k0) * BITS / 8 + 127) >> 7;
      for (int st = 0; st < ns; ++st, ++js) {
        const int off = st * kPB;
        const int c_hi = cbase + ((off + kPB - 1) >> 7);
        for (; w_ready <= c_hi && ok; ++w_ready)
          ok = mbar_wait(B(full_w, w_ready % WS), (w_ready / WS) & 1, abort_flag);
        const int a = js % ST;
        ok = __all_sync(0xffffffffu, ok && mbar_wait(B(empty_st, a), ((js / ST) & 1) ^ 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        // ---- codes -> A stage in TMEM (two halves of 32 codes)
        Packed<BITS> pk;
        load_codes<BITS>(pk, wring, cbase, off, r);
        const uint32_t a_addr = tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(32 * a);
        {
          uint32_t o[16];
          a_chunk<T, BITS, FP4, 0>(pk, o);
          a_chunk<T, BITS, FP4, 1>(pk, o);
          a_chunk<T, BITS, FP4, 2>(pk, o);
          a_chunk<T, BITS, FP4, 3>(pk, o);
          tmem_st_16(a_addr, o);
        }
        {
          uint32_t o[16];
          a_chunk<T, BITS, FP4, 4, 4>(pk, o);
          a_chunk<T, BITS, FP4, 5, 4>(pk, o);
          a_chunk<T, BITS, FP4, 6, 4>(pk, o);
          a_chunk<T, BITS, FP4, 7, 4>(pk, o);
          tmem_st_16(a_addr + 16, o);
        }
        // ---- x run of this stage: copied kXAhead stages ago
        if (issued - js - 1 >= kXAhead - 1) {
          if constexpr (kXAhead >= 2) cp_async_wait_group<kXAhead - 1>();
          else cp_async_wait_group<0>();
        } else {
          cp_async_wait_group<0>();
        }
        float hs = 0.f;
        {
          uint4* xp = reinterpret_cast<uint4*>(xring + (js % S::kXS) * S::kXTile + xrow * 128 +
                                               ((xrun ^ (xrow & 7)) << 4));
          uint4 cur = xmine ? *xp : make_uint4(0u, 0u, 0u, 0u);   // past K: never used
          if constexpr (BITS == 2 && kPermX) {
            // runs (2w, 2w + 1) pair up across lanes l and l ^ 1 (same row)
            const uint4 other = make_uint4(__shfl_xor_sync(0xffffffffu, cur.x, 1),
                                           __shfl_xor_sync(0xffffffffu, cur.y, 1),
                                           __shfl_xor_sync(0xffffffffu, cur.z, 1),
                                           __shfl_xor_sync(0xffffffffu, cur.w, 1));
            if (xmine) {
              hs = sum8<T>(cur);
              uint4 lo = (xrun & 1) ? other : cur, hi = (xrun & 1) ? cur : other;
              perm_x2(lo, hi);
              *xp = (xrun & 1) ? hi : lo;
            }
          } else if (xmine) {
            if constexpr (kSums) hs = sum8<T>(cur);
            if constexpr (kPermX) {
              perm_x4(cur);
              *xp = cur;
            }
          }
        }
        // the next x run in flight (its slot was freed with stage js - kST)
        if (lu < total) x_issue();
        if constexpr (kSums) {
          // runs of a row half sit in lanes 8r' + {0..3} / {4..7} of this warp
          hs += __shfl_xor_sync(0xffffffffu, hs, 1);
          hs += __shfl_xor_sync(0xffffffffu, hs, 2);
          const float full = hs + __shfl_xor_sync(0xffffffffu, hs, 4);
          // one vector of 16 row sums per group (this warp writes rows
          // 4 q4 .. 4 q4 + 3): a half (group 32), the stage (group 64) or two
          // stages (group 128)
          auto put = [&](float v, int src) -> bool {
            if ((lane & 7) == src && xmine) xsring[(gx % XGS) * 16 + xrow] = v;
            ++gx;
            return true;
          };
          if (gs == 32) {
            if (2 * st < ngu) ok = put(hs, 0);
            if (ok && 2 * st + 1 < ngu) ok = put(hs, 4);
          } else if (gs == 64) {
            ok = put(full, 0);
          } else if ((st & 1) == 0) {
            carry = full;
          } else {
            ok = put(carry + full, 0);
          }
          if (!ok) break;
        }
        fence_proxy_async_smem();                         // x writes -> tensor core reads
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B(full_a, a));
        // chunks that end before the next stage starts are done
        const int w_done = cbase + (st + 1 < ns ? (((st + 1) * kPB) >> 7) : nwc);
        for (; w_freed < w_done; ++w_freed)
          if (lane == 0) mbar_arrive(B(empty_w, w_freed % WS));
      }
      cbase += nwc;
    }
    cp_async_wait_all();                                  // no copy lands after the CTA exits
  } else if (warp >= S::kWarpEp0) {
    // ------------------------------------------------------- epilogue
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    int gi = 0, sbase = 0, s_ready = 0, s_freed = 0, s_have = -1;
    uint4 sv = make_uint4(0, 0, 0, 0), bv = make_uint4(0, 0, 0, 0);
    bool ok = true, waited = false;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x) {
      const Unit un = unit_at(pr, u);
      const DecProblem& q = pr.prob[un.p];
      const int ng = (un.k1 - un.k0) >> pr.gs_log2;
      const int ga0 = un.k0 >> pr.gs_log2;                // absolute group of the unit's first
      const int sc0 = ga0 / SGC;
      const int nsc = (((un.k1 - 1) >> pr.gs_log2) / SGC) - sc0 + 1;
      float acc[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) acc[m] = 0.0f;
      for (int g = 0; g < ng; ++g) {
        const int gg = gi + g, slot = gg % DS;
        ok = __all_sync(0xffffffffu, mbar_wait(B(full_d, slot), (gg / DS) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        // the group's products for rows of x 0-7 (and 8-15 when M > 8)
        const uint32_t d_addr = tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(S::kDCol0 + 16 * slot);
        uint32_t v0[8], v1[8];
        tmem_ld_8(d_addr, v0);
        if (M > 8) tmem_ld_8(d_addr + 8, v1);
        tmem_ld_wait();
        tc_fence_before();
        auto dval = [&](int m) { return __uint_as_float(m < 8 ? v0[m & 7] : v1[m & 7]); };
        // this group's scale (and bias) from the scale chunk ring
        const int ga = ga0 + g;
        const int cj = sbase + (ga / SGC - sc0);
        if (cj != s_have) {
          for (; s_ready <= cj && ok; ++s_ready)
            ok = mbar_wait(B(full_s, s_ready % SS), (s_ready / SS) & 1, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          const uint8_t* sp = sring + (cj % SS) * S::kSChunk + r * 16;
          sv = *reinterpret_cast<const uint4*>(sp);
          if constexpr (!FP4) bv = *reinterpret_cast<const uint4*>(sp + kRowsW * 16);
          __syncwarp();
          for (; s_freed < cj; ++s_freed)
            if (lane == 0) mbar_arrive(B(empty_s, s_freed % SS));
          s_have = cj;
        }
        const int e = ga % SGC;
        if constexpr (FP4) {
          const float sf = fp4_scale_t<T>(byte_elem(sv, e), gs);
#pragma unroll
          for (int m = 0; m < 16; ++m)
            if (m < M) acc[m] = fmaf(sf, dval(m), acc[m]);
        } else {
          // the x sums of this group (16 rows), written before the group's
          // last A stage was handed to the MMA
          const int xslot = gg % XGS;
          const float sf = t_elem<T>(sv, e);
          const float bf = fmaf(-kOff, sf, t_elem<T>(bv, e));
          const float4* xv4 = reinterpret_cast<const float4*>(xsring + xslot * 16);
#pragma unroll
          for (int m4 = 0; m4 < 4; ++m4) {
            if (4 * m4 < M) {
              const float4 t = xv4[m4];
              const float xv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
              for (int i = 0; i < 4; ++i)
                if (4 * m4 + i < M)
                  acc[4 * m4 + i] = fmaf(sf, dval(4 * m4 + i), fmaf(bf, xv[i], acc[4 * m4 + i]));
            }
          }
        }
        // the D slot and this group's x sums are no longer read
        __syncwarp();
        if (lane == 0) mbar_arrive(B(empty_d, slot));
      }
      if (!ok) break;
      // the unit's scale chunks are done
      __syncwarp();
      for (; s_freed < sbase + nsc; ++s_freed)
        if (lane == 0) mbar_arrive(B(empty_s, s_freed % SS));
      s_have = -1;
      sbase += nsc;
      gi += ng;
      // ------------------------------------------- output of the unit
      if (!waited) {
        pdl_wait();                                       // y and the workspace are ordered
        waited = true;
      }
      const bool row_ok = un.n0 + r < q.N;
      T* yp = reinterpret_cast<T*>(q.y) + un.n0 + r;
      if (q.splits == 1) {
        if (row_ok) {
#pragma unroll
          for (int m = 0; m < 16; ++m)
            if (m < M) yp[(int64_t)m * q.N] = TT<T>::from_f(acc[m]);
        }
      } else {
        uint32_t* cnt = pr.ws + 4 * (q.cnt0 + un.tile) + q4;
        float* part = reinterpret_cast<float*>(pr.ws + q.ws_part) +
                      (int64_t)un.tile * q.splits * M * kRowsW;
        float* mine = part + (int64_t)un.slice * M * kRowsW + r;
#pragma unroll
        for (int m = 0; m < 16; ++m)
          if (m < M) __stcg(mine + m * kRowsW, acc[m]);
        __threadfence();
        __syncwarp();
        unsigned old = 0;
        if (lane == 0) old = atomicAdd(cnt, 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old == (unsigned)(q.splits - 1)) {
          // the last slice: add the slices in slice order
          __threadfence();
          float tot[16];
#pragma unroll
          for (int m = 0; m < 16; ++m) tot[m] = 0.0f;
          for (int sl = 0; sl < q.splits; ++sl) {
            const float* ps = part + (int64_t)sl * M * kRowsW + r;
#pragma unroll
            for (int m = 0; m < 16; ++m)
              if (m < M) tot[m] += sl == un.slice ? acc[m] : __ldcg(ps + m * kRowsW);
          }
          if (row_ok) {
#pragma unroll
            for (int m = 0; m < 16; ++m)
              if (m < M) yp[(int64_t)m * q.N] = TT<T>::from_f(tot[m]);
          }
          __syncwarp();
          if (lane == 0) atomicExch(cnt, 0u);
        }
      }
    }
    if (!waited) pdl_wait();
  }

  __syncthreads();
  if (warp == S::kWarpMma0) {
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(&g_aq_device_error, 1u);
}

// ------------------------------------------------------------------- host
// K columns per slice: a multiple of 64 and of the group size whose packed
// bytes fill whole 128-byte weight chunks (no chunk is read by two slices).
int dec_kgran(int bits, int gs) {
  const int low = bits & -bits;                       // 1, 2, 4 or 8
  return std::max(1024 / low, std::max(gs, kBK));
}

struct DecSplit {
  int splits, kslice;
};

// Split K so that the units of one problem fill `slots` CTAs, or so that a
// unit carries about `unit_bytes` of packed weights (batched launches).
DecSplit dec_split(int64_t N, int64_t K, int bits, int gs, int64_t slots, int64_t unit_bytes) {
  const int64_t tiles = (N + kRowsW - 1) / kRowsW;
  const int kgran = dec_kgran(bits, gs);
  const int64_t max_splits = std::max<int64_t>(1, (K + kgran - 1) / kgran);
  int64_t want;
  if (unit_bytes > 0) {
    want = (kRowsW * K * bits / 8 + unit_bytes / 2) / unit_bytes;
  } else {
    want = (slots + tiles / 2) / tiles;
    // at least four stages per slice
    want = std::min<int64_t>(want, std::max<int64_t>(1, K / (4 * kBK)));
  }
  want = std::max<int64_t>(1, std::min(want, max_splits));
  int64_t kslice = (K + want - 1) / want;
  kslice = (kslice + kgran - 1) / kgran * kgran;
  DecSplit d;
  d.kslice = (int)kslice;
  d.splits = (int)((K + kslice - 1) / kslice);
  return d;
}

constexpr int64_t kSlots = 2 * 148;

// Plan of one launch: per problem its split, first tile counter and the word
// offset of its partials; `words` is the workspace the launch needs.
struct DecGroupPlan {
  DecSplit sp[kDecMaxProblems];
  int cnt0[kDecMaxProblems];
  int64_t part[kDecMaxProblems];
  int64_t words;
};

void dec_plan_group(DecGroupPlan& g, const QmvProblemDesc* probs, int count, int64_t M, int bits,
                    int gs, int64_t unit_bytes) {
  int tiles_used = 0;                                 // split tiles given counters so far
  int64_t part = kDecCntWords;
  bool any = false;
  for (int i = 0; i < count; ++i) {
    DecSplit d = dec_split(probs[i].N, probs[i].K, bits, gs, kSlots, unit_bytes);
    const int64_t tiles = (probs[i].N + kRowsW - 1) / kRowsW;
    if (d.splits > 1 && tiles_used + tiles > kDecMaxSplitTiles) {
      d.splits = 1;                                   // out of counters: whole rows per unit
      d.kslice = (int)probs[i].K;
    }
    g.sp[i] = d;
    g.cnt0[i] = tiles_used;
    g.part[i] = part;
    if (d.splits > 1) {
      any = true;
      tiles_used += (int)tiles;
      part += (tiles * d.splits * M * kRowsW + 31) / 32 * 32;
    }
  }
  g.words = any ? part : 0;
}

template <typename T, int BITS, bool FP4, int P>
cudaError_t launch_dec(const DecParams<P>& pr, int grid, cudaStream_t st) {
  auto kern = qmv_tc_kernel<T, BITS, FP4, P>;
  static std::atomic<bool> attr_done[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !attr_done[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DecShape::kSmem);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_done[dev].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(DecShape::kThreads, 1, 1);
  cfg.dynamicSmemBytes = DecShape::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, pr);
}

template <typename T, int P>
cudaError_t dec_by_bits(const DecParams<P>& pr, int grid, int bits, int mode, cudaStream_t st) {
  if (mode == AQ_MODE_FP4) return launch_dec<T, 4, true, P>(pr, grid, st);
  switch (bits) {
    case 2: return launch_dec<T, 2, false, P>(pr, grid, st);
    case 3: return launch_dec<T, 3, false, P>(pr, grid, st);
    case 4: return launch_dec<T, 4, false, P>(pr, grid, st);
    case 5: return launch_dec<T, 5, false, P>(pr, grid, st);
    case 6: return launch_dec<T, 6, false, P>(pr, grid, st);
    case 8: return launch_dec<T, 8, false, P>(pr, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

// Fill problem slot `i` (maps, sizes, split plan, workspace offsets).
cudaError_t dec_problem(DecProblem& dp, const QmvProblemDesc& d, int64_t M, int bits, int gs,
                        int mode, int dtype, const DecSplit& sp, int cnt0, int64_t part) {
  memset(&dp, 0, sizeof(dp));
  const CUtensorMapDataType tt =
      dtype == AQ_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  (void)tt;
  dp.x = d.x;
  const int64_t row_bytes = d.K * bits / 8;
  cudaError_t e = make_map(&dp.w, d.w_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d.N, row_bytes, 128, kRowsW,
               CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const int esz = mode == AQ_MODE_FP4 ? 1 : 2;
  const CUtensorMapDataType st_t =
      mode == AQ_MODE_FP4 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
  const int64_t G = d.K / gs;
  e = make_map(&dp.s, d.scales, st_t, esz, d.N, G, 16 / esz, kRowsW, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;
  if (mode != AQ_MODE_FP4) {
    e = make_map(&dp.b, d.biases, st_t, esz, d.N, G, 16 / esz, kRowsW, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
  }
  dp.y = d.y;
  dp.N = (int)d.N;
  dp.K = (int)d.K;
  dp.splits = sp.splits;
  dp.kslice = sp.kslice;
  dp.cnt0 = cnt0;
  dp.ws_part = part;
  return cudaSuccess;
}

template <int P>
cudaError_t dec_launch_group(const QmvProblemDesc* probs, int count, int64_t M, int bits, int gs,
                             int mode, int dtype, void* ws, int64_t unit_bytes, cudaStream_t st) {
  static_assert(sizeof(DecParams<P>) <= 32000, "kernel parameter space");
  DecGroupPlan g;
  dec_plan_group(g, probs, count, M, bits, gs, unit_bytes);
  if (g.words > 0 && !ws) return cudaErrorInvalidValue;
  DecParams<P> pr;
  memset(&pr, 0, sizeof(pr));
  int units = 0;
  for (int i = 0; i < count; ++i) {
    cudaError_t e = dec_problem(pr.prob[i], probs[i], M, bits, gs, mode, dtype, g.sp[i], g.cnt0[i],
                                g.part[i]);
    if (e != cudaSuccess) return e;
    units += (int)((probs[i].N + kRowsW - 1) / kRowsW) * g.sp[i].splits;
    pr.unit_end[i] = units;
  }
  pr.count = count;
  pr.M = (int)M;
  pr.gs_log2 = ilog2i(gs);
  pr.weights_early = weight_prefetch_enabled();
  pr.x_early = input_prefetch_enabled();
  pr.ws = reinterpret_cast<uint32_t*>(ws);
  const int grid = (int)std::min<int64_t>(units, kSlots);
  return dtype == AQ_F16 ? dec_by_bits<__half, P>(pr, grid, bits, mode, st)
                         : dec_by_bits<__nv_bfloat16, P>(pr, grid, bits, mode, st);
}

}  // namespace

bool qmv_tc_applies(int64_t M, int64_t N, int64_t K, int bits, int gs, int mode,
                    const void* scales, const void* biases) {
  if (M < 1 || M > 16 || N < 1 || K < 1) return false;
  return qmv_tc_shape_ok(N, K, bits, gs, mode) && ((uintptr_t)scales & 15) == 0 &&
         (mode == AQ_MODE_FP4 || ((uintptr_t)biases & 15) == 0);
}

bool qmv_tc_shape_ok(int64_t N, int64_t K, int bits, int gs, int mode) {
  const int64_t row_bytes = K * bits / 8;
  const int esz = mode == AQ_MODE_FP4 ? 1 : 2;
  return N >= 1 && K >= 1 && row_bytes % 16 == 0 && ((K / gs) * esz) % 16 == 0 &&
         N <= kMaxRowsDec && K <= kMaxRowsDec;
}

size_t qmv_tc_workspace(int64_t M, int64_t N, int64_t K, int bits, int gs) {
  const QmvProblemDesc d{nullptr, nullptr, nullptr, nullptr, nullptr, N, K};
  DecGroupPlan g;
  dec_plan_group(g, &d, 1, M, bits, gs, 0);
  return (size_t)g.words * 4;
}

size_t qmv_tc_batched_workspace(const QmvProblemDesc* probs, int count, int64_t M, int bits,
                                int gs) {
  int64_t best = 0;
  for (int i0 = 0; i0 < count; i0 += kDecMaxProblems) {
    DecGroupPlan g;
    dec_plan_group(g, probs + i0, std::min(count - i0, kDecMaxProblems), M, bits, gs, kDecUnitBytes);
    best = std::max(best, g.words);
  }
  return (size_t)best * 4;
}

cudaError_t launch_qmv_tc(const void* x, const void* w_q, const void* scales, const void* biases,
                          void* y, int64_t M, int64_t N, int64_t K, int bits, int gs, int mode,
                          int dtype, void* ws, cudaStream_t st) {
  QmvProblemDesc d{x, w_q, scales, biases, y, N, K};
  return dec_launch_group<1>(&d, 1, M, bits, gs, mode, dtype, ws, 0, st);
}

cudaError_t launch_qmv_tc_batched(const QmvProblemDesc* probs, int count, int64_t M, int bits,
                                  int gs, int mode, int dtype, void* ws, cudaStream_t st) {
  for (int i0 = 0; i0 < count; i0 += kDecMaxProblems) {
    const int n = std::min(count - i0, kDecMaxProblems);
    cudaError_t e = dec_launch_group<kDecMaxProblems>(probs + i0, n, M, bits, gs, mode, dtype, ws,
                                                      kDecUnitBytes, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t read_device_error_qmv_tc(unsigned* out) { return read_tu_error(out); }

}  // namespace aq
