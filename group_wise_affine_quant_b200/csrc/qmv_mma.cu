// qmv_mma.cu — decode-sized quantized matmul (1 <= M <= 16 rows of x) for
// 4-bit affine weights, streaming the packed weights at HBM speed:
//   y[m, n] = sum_g ( s[n,g] * sum_{k in g} q[n,k] x[m,k]  +  b[n,g] * sum_{k in g} x[m,k] )
// for one problem (aq_qmv) or a list of independent problems (aq_qmv_batched).
//
// Prior art: affine_packed_qmv_fast in "Add the 3bit packed qmm_t" keeps the
// dot product in fp32 and hoists scale and bias out of each group (result +=
// s * accum + b * sum); the "Improvements in the quantizer and dequantization
// kernel" page keeps qmv in fp32 throughout.  This kernel keeps that
// arithmetic (w_hat is never rounded to T) and runs the inner products on
// the tensor cores:
//   * The codes are the MMA's A operand.  Under bf16 the pattern 0x4300 | q
//     is the exact value 128 + q (fp16: 0x6400 | q = 1024 + q), so a warp-level
//     m16n8k16 MMA forms sum_k (off + q) x with exact products and fp32
//     accumulation, one group at a time in registers; the group's result is
//     folded into the output as s * D + (b - off * s) * sum_k x in fp32.
//   * Decode is bound by the weight stream, not by the tensor pipe: a
//     128-byte piece of 4-bit codes (16 rows x 16 K) costs one MMA per 8 rows
//     of x, about 2 SM cycles, against the ~5.5 cycles HBM needs to deliver
//     it.  Warp-level MMAs keep A, B and the accumulators in registers, so
//     the per-group fp32 epilogue costs a few FMAs and no tensor-memory round
//     trip or cross-warp hand-off.
// Work decomposition, B200-first:
//   * A unit is 128 weight rows x one K-slice of one problem.  CTAs are
//     persistent (grid <= SMs x resident CTAs) and walk the units round-robin;
//     the weight ring runs on across unit boundaries.
//   * Warp roles: warps 0-7 each own a 16-row tile and run MMAs; warp 8
//     issues the TMA copies (weights: 128 rows x 128 bytes per stage, 128-byte
//     swizzle; scales and biases: 128 rows x one sub-slice of groups); warps
//     9-10 prepare each 512-column sub-slice (1024 for group size 128): they
//     turn the raw scales and biases into fp32 (s, b - off * s) pairs, copy
//     the x columns into shared memory in the order the codes unpack, and add
//     the per-group x sums (fp32, a fixed shuffle tree over a group's lanes).
//     Sub-slice buffers are double-buffered, so the MMA warps' inner loop
//     waits only on weight stages.
//   * Unpack: a 32-bit word holds codes c0..c7 at bits 4i; the pair
//     (c_i, c_{i+4}) is ((w >> 4i) & 0x000F000F) | magic, which is one
//     bf16x2 / fp16x2 A register.  x is stored as (x0,x4),(x2,x6),(x1,x5),
//     (x3,x7) per 8 columns so that one 16-byte shared-memory load gives both
//     K-steps' B registers of a word.
//   * K-slices of a row tile reduce through the caller's workspace: every
//     slice stores its fp32 partial tile, and the last slice to arrive (a
//     per-tile counter) adds the slices in slice order and writes y, then
//     resets the counter.  The order of the sum does not depend on which
//     slice arrives last.
//   * Every mbarrier wait is bounded (2 s); a timeout sets a device error
//     bit, every role stops, and the TMA copies in flight are waited for
//     (bounded) before the CTA exits.
#include <algorithm>
#include <atomic>

#include "qmm_kernel.cuh"

namespace aq {
namespace {

constexpr int kMvRows = 128;                 // weight rows per unit (8 warps x 16)
constexpr int kMvMaxProblems = 40;           // problems per launch of the batched entry
constexpr int kMvSchedWords = 16;            // workspace words 0, 1: unit counter, exit counter
constexpr int kMvMaxSplitTiles = 16384 - kMvSchedWords;  // 16-row tiles with a counter
constexpr int kMvCntWords = 16384;           // the counter area: the first 64 KB of the workspace
constexpr int kMvQ = 8;                      // unit-queue depth (producer -> prep and MMA warps)

struct MvProblem {
  CUtensorMap w;        // [N, K/2] u8, box {128 bytes, 128 rows}, 128-byte swizzle
  CUtensorMap s;        // [N, G] scales (2-byte), box {groups of a sub-slice, 128 rows}
  CUtensorMap b;        // [N, G] biases, likewise
  const void* x;        // [M, K] T
  void* y;              // [M, N] T
  int N, K;
  int splits;           // K-slices per row block
  int kslice;           // K columns per slice (a multiple of the sub-slice)
  int cnt0;             // first tile counter of this problem
  int pad_;
  int64_t ws_part;      // word offset of the fp32 partials
};

template <int P>
struct MvParams {
  MvProblem prob[P];
  int unit_end[P];      // cumulative unit counts
  int count;
  int M;
  int weights_early;    // stream weights / scales / biases before the grid dependency wait
  int pad_;
  uint32_t* ws;
  uint64_t wait_ns;     // bound of every mbarrier wait
  uint64_t delay_ns;    // test hook: TMA warp start delay (0 = none)
};

// K columns per sub-slice: 8 groups (the scale boxes are 16-byte rows),
// and at least one 256-column weight stage.  Host and device use this one
// definition.
constexpr int mv_subk(int gs) { return gs * 8 > 256 ? gs * 8 : 256; }

template <int GS, int NT, int R>
struct MvShape {
  static constexpr int kMmaWarps = 8 / R;                       // R 16-row tiles per MMA warp
  static constexpr int kThreads = 32 * (kMmaWarps + 3);
  static constexpr int kWarpLoad = kMmaWarps, kWarpPrep0 = kMmaWarps + 1;
  static constexpr int kSubK = mv_subk(GS);                    // K per sub-slice (8 groups)
  static constexpr int kGps = kSubK / GS;                      // groups per sub-slice
  static constexpr int kStageK = 256;                          // 128 bytes of 4-bit codes per row
  static constexpr int kSps = kSubK / kStageK;                 // stages per sub-slice
  static constexpr int kST = NT == 1 ? 4 : 3;                  // weight stages (shared memory: 2 CTAs per SM)
  static constexpr int kStage = kMvRows * 128;                 // 16 KB
  static constexpr int kXP = kSubK * 2 + 64;                   // x row pitch: 64 mod 128 bytes
  static constexpr int kXBuf = 8 * NT * kXP;
  static constexpr int kXsBuf = kGps * 16 * 4;                 // [group][16 rows of x] fp32
  static constexpr int kTabPitch = kGps + 2;                   // float2 per weight row (16-byte rows)
  static constexpr int kTabBuf = kMvRows * kTabPitch * 8;
  static constexpr int kSbArr = kMvRows * kGps * 2;            // one raw scale or bias box
  static constexpr int kRingOff = 0;
  static constexpr int kXOff = kRingOff + kST * kStage;
  static constexpr int kXsOff = kXOff + 2 * kXBuf;
  static constexpr int kTabOff = kXsOff + 2 * kXsBuf;
  static constexpr int kSbOff = kTabOff + 2 * kTabBuf;
  static constexpr int kBarOff = kSbOff + 4 * kSbArr;
  static constexpr int kBars = 2 * kST + 10 + 2 * kMvQ;
  static constexpr int kSmem = 1024 + kBarOff + kBars * 8 + 16 + 4 * kMvQ;
  static_assert(kXP % 128 == 64, "x pitch");
  static_assert(kSbOff % 128 == 0 && kXOff % 1024 == 0, "TMA destinations");
  static_assert((kGps * 2) % 16 == 0, "scale box rows are 16-byte multiples");
};

template <typename T> struct Magic4;
template <> struct Magic4<__nv_bfloat16> {
  static constexpr uint32_t kM = 0x43004300u;    // bf16 128 + q
  static constexpr float kOff = 128.0f;
};
template <> struct Magic4<__half> {
  static constexpr uint32_t kM = 0x64006400u;    // fp16 1024 + q
  static constexpr float kOff = 1024.0f;
};

template <typename T>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// The same MMA with a zero accumulator (the first K-step of a group).
template <typename T>
__device__ __forceinline__ void mma16816_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                           uint32_t b1) {
  const float z = 0.0f;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(z));
  } else {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(z));
  }
}

// (v & mask) | magic in one logic op.
__device__ __forceinline__ uint32_t and_or(uint32_t v, uint32_t mask, uint32_t magic) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(v), "r"(mask), "r"(magic));
  return r;
}

// Atomic add at GPU scope with release semantics: the calling thread's prior
// writes, and those it has observed (a warp's, after __syncwarp), are visible
// before the addition is.
__device__ __forceinline__ unsigned atom_add_release_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.release.gpu.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ float t_to_f(uint32_t h, bool bf16) {
  return bf16 ? __uint_as_float(h << 16) : __half2float(__ushort_as_half((unsigned short)h));
}

struct MvUnit {
  int p, rb, sp, k0, nsub;
};

template <int P, int SUBK>
__device__ __forceinline__ MvUnit mv_unit(const MvParams<P>& pr, int u) {
  // the problem whose cumulative unit range holds u (binary search)
  int lo = 0, hi = pr.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (u >= pr.unit_end[mid]) lo = mid + 1;
    else hi = mid;
  }
  const int p = lo;
  const MvProblem& q = pr.prob[p];
  const int local = u - (p ? pr.unit_end[p - 1] : 0);
  const int rbs = (q.N + kMvRows - 1) / kMvRows;
  MvUnit un;
  un.p = p;
  un.rb = local % rbs;
  un.sp = local / rbs;
  un.k0 = un.sp * q.kslice;
  un.nsub = (min(q.kslice, q.K - un.k0)) / SUBK;
  return un;
}

// Next unit id from the CTA's unit queue (-1: no more units; -2: a wait gave up).
__device__ __forceinline__ int mv_take(volatile int* uq, uint64_t* uqf, uint64_t* uqe, int k,
                                       int lane, volatile int* abort_flag, uint64_t wl) {
  const int qs = k % kMvQ;
  if (!mbar_wait(smem_u32(uqf + qs), (k / kMvQ) & 1, abort_flag, wl)) return -2;
  const int u = uq[qs];
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_u32(uqe + qs));
  return u;
}

__device__ __forceinline__ void mv_drain(const uint64_t* bars, int slots, int issued,
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

// Bit pattern of T(1.0) twice: the A operand that turns an MMA into row sums of x.
template <typename T> constexpr uint32_t ones2() {
  return std::is_same<T, __nv_bfloat16>::value ? 0x3F803F80u : 0x3C003C00u;
}

// Up to this many rows of x, the prep warp adds the per-group x sums (fp32
// adds and a shuffle tree); above it the MMA warps do, with an all-ones MMA
// each for its share of the groups, because the prep warp's adds over more
// rows would fall behind the weight stream.
constexpr int kMvPrepSumsMaxM = 4;

template <typename T, int GS, int NT, int R, int P>
__global__ void __launch_bounds__(MvShape<GS, NT, R>::kThreads, 2)
qmv_mma_kernel(const __grid_constant__ MvParams<P> pr) {
  using S = MvShape<GS, NT, R>;
  constexpr int kMvWarps = S::kMmaWarps;
  constexpr int ST = S::kST, GPS = S::kGps, SUBK = S::kSubK;
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kMag = Magic4<T>::kM;
  constexpr float kOff = Magic4<T>::kOff;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* full = bars;                 // weight stage landed (TMA bytes)
  uint64_t* empty = full + ST;           // weight stage consumed (the MMA warps)
  uint64_t* sbf = empty + ST;            // raw scales / biases of a sub-slice landed (TMA bytes)
  uint64_t* sbe = sbf + 2;               // raw scales / biases converted (its prep warp)
  uint64_t* xf = sbe + 2;                // sub-slice prepared (its prep warp)
  uint64_t* xe = xf + 2;                 // sub-slice consumed (the MMA warps)
  uint64_t* xsr = xe + 2;                // per-group x sums written (the MMA warps, M > kMvPrepSumsMaxM)
  uint64_t* uqf = xsr + 2;               // unit id posted (producer)
  uint64_t* uqe = uqf + kMvQ;            // unit id read (every prep and MMA warp)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + S::kBars);
  volatile int* uq = reinterpret_cast<volatile int*>(bars + S::kBars) + 4;   // [kMvQ] unit ids
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int M = pr.M;
  const int total = pr.unit_end[pr.count - 1];
  const uint64_t wl = pr.wait_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(empty + i), kMvWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(sbf + i), 1);
      mbar_init(smem_u32(sbe + i), 1);
      mbar_init(smem_u32(xf + i), 1);
      mbar_init(smem_u32(xe + i), kMvWarps);
      mbar_init(smem_u32(xsr + i), kMvWarps);
    }
    for (int i = 0; i < kMvQ; ++i) {
      mbar_init(smem_u32(uqf + i), 1);
      mbar_init(smem_u32(uqe + i), kMvWarps + 2);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == S::kWarpLoad) {
    // ------------------------------------------------------------ TMA issue
    int wc = 0, sc = 0;
    if (lane == 0) {
      bool waited = !pr.weights_early;
      if (waited) pdl_wait();
      if (pr.delay_ns) {                       // test hook: hold back the first copy
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < pr.delay_ns && !*abort_flag) {
        }
      }
      const uint64_t pol = l2_policy_evict_first();
      // Units: the first one of each CTA is blockIdx.x; later ones are claimed
      // from the launch's unit counter (after the wait on the previous kernel,
      // which leaves the counter at zero), so the CTAs stay evenly loaded.
      int posted = 0;
      auto post = [&](int uu) -> bool {
        const int qs = posted % kMvQ;
        if (!mbar_wait(smem_u32(uqe + qs), ((posted / kMvQ) & 1) ^ 1, abort_flag, wl)) return false;
        uq[qs] = uu;
        mbar_arrive(smem_u32(uqf + qs));
        ++posted;
        return true;
      };
      for (int u = blockIdx.x; u < total && !*abort_flag;) {
        if (!post(u)) break;
        const MvUnit un = mv_unit<P, SUBK>(pr, u);
        const MvProblem& q = pr.prob[un.p];
        const int row0 = un.rb * kMvRows;
        bool ok = true;
        for (int j = 0; j < un.nsub && ok; ++j) {
          const int kk = un.k0 + j * SUBK;
          const int buf = sc & 1;
          if (!mbar_wait(smem_u32(sbe + buf), ((sc >> 1) & 1) ^ 1, abort_flag, wl)) break;
          mbar_arrive_expect_tx(smem_u32(sbf + buf), 2 * S::kSbArr);
          uint8_t* sb = smem + S::kSbOff + buf * 2 * S::kSbArr;
          tma_load_2d(smem_u32(sb), &q.s, smem_u32(sbf + buf), kk / GS, row0);
          tma_load_2d(smem_u32(sb + S::kSbArr), &q.b, smem_u32(sbf + buf), kk / GS, row0);
          ++sc;
          for (int st = 0; st < S::kSps; ++st) {
            const int slot = wc % ST;
            if (!mbar_wait(smem_u32(empty + slot), ((wc / ST) & 1) ^ 1, abort_flag, wl)) { ok = false; break; }
            mbar_arrive_expect_tx(smem_u32(full + slot), S::kStage);
            tma_load_2d_hint(smem_u32(smem + S::kRingOff + slot * S::kStage), &q.w,
                             smem_u32(full + slot), (kk + st * S::kStageK) / 2, row0, pol);
            ++wc;
          }
        }
        if (!ok) break;
        if (!waited) {
          pdl_wait();
          waited = true;
        }
        u = (int)gridDim.x + (int)atomicAdd(pr.ws, 1u);
      }
      if (!*abort_flag) post(-1);                           // no more units
      // This CTA claims no more units: count it out, and the last CTA to do so
      // puts the launch's unit counter back to zero (every claim of the launch
      // has then been made), off the critical path of the last unit.
      if (!waited) {
        pdl_wait();
        waited = true;
      }
      if (atomicAdd(pr.ws + 1, 1u) == gridDim.x - 1) {
        atomicExch(pr.ws, 0u);
        atomicExch(pr.ws + 1, 0u);
      }
      mv_drain(full, ST, wc, abort_flag);
      mv_drain(sbf, 2, sc, abort_flag);
    }
  } else if (warp >= S::kWarpPrep0) {
    // ------------------------------------------------ sub-slice preparation
    // Prep warp b prepares the sub-slices c with c % 2 == b, into buffer b.
    const int b = warp - S::kWarpPrep0;
    pdl_wait();
    int c = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = mv_take(uq, uqf, uqe, k, lane, abort_flag, wl);
      if (u < 0) { ok = u == -1; break; }
      const MvUnit un = mv_unit<P, SUBK>(pr, u);
      const MvProblem& q = pr.prob[un.p];
      const T* xg = reinterpret_cast<const T*>(q.x);
      for (int j = 0; j < un.nsub; ++j, ++c) {
        if ((c & 1) != b) continue;
        const uint32_t par = (c >> 1) & 1;
        uint8_t* xb = smem + S::kXOff + b * S::kXBuf;
        if (!mbar_wait(smem_u32(xe + b), par ^ 1, abort_flag, wl)) { ok = false; break; }
        // x columns of the sub-slice (natural order; 64-byte blocks of 32 columns
        // at a row pitch of 64 mod 128 bytes), copied with cp.async
        const int kk = un.k0 + j * SUBK;
        constexpr int kCpr = SUBK / 8;                         // 16-byte chunks per x row
        const int nch = M * kCpr;
        for (int i = lane; i < nch; i += 32) {
          const int m = i / kCpr, ch = i % kCpr;
          cp_async_16(smem_u32(xb + m * S::kXP + ch * 16),
                     reinterpret_cast<const uint4*>(xg + (int64_t)m * q.K + kk) + ch);
        }
        // fp32 (s, b - off * s) per weight row and group (while the x copy is in flight)
        if (!mbar_wait(smem_u32(sbf + b), par, abort_flag, wl)) {
          cp_async_wait_all();                              // no copy may outlive the CTA
          ok = false;
          break;
        }
        const uint16_t* sraw = reinterpret_cast<const uint16_t*>(smem + S::kSbOff + b * 2 * S::kSbArr);
        const uint16_t* braw = sraw + kMvRows * GPS;
        float2* tab = reinterpret_cast<float2*>(smem + S::kTabOff + b * S::kTabBuf);
        for (int i = lane; i < kMvRows * (GPS / 8); i += 32) {
          const int row = i / (GPS / 8), g8 = 8 * (i % (GPS / 8));
          const uint4 sv = *reinterpret_cast<const uint4*>(sraw + row * GPS + g8);
          const uint4 bv = *reinterpret_cast<const uint4*>(braw + row * GPS + g8);
          const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w}, bw[4] = {bv.x, bv.y, bv.z, bv.w};
          float4* dst = reinterpret_cast<float4*>(tab + row * S::kTabPitch + g8);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float s0 = t_to_f(sw[e] & 0xFFFFu, kBf16), s1 = t_to_f(sw[e] >> 16, kBf16);
            const float b0 = t_to_f(bw[e] & 0xFFFFu, kBf16), b1 = t_to_f(bw[e] >> 16, kBf16);
            dst[e] = make_float4(s0, fmaf(-kOff, s0, b0), s1, fmaf(-kOff, s1, b1));
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(sbe + b));
        cp_async_wait_all();
        // Reorder each 8-column chunk in place to the order the codes unpack,
        // (x0,x4), (x2,x6), (x1,x5), (x3,x7), and add the per-group x sums: a
        // group's GS/8 chunks sit on GS/8 consecutive lanes of one pass (a row
        // has a multiple of 32 chunks), which add their chunk sums by a fixed
        // shuffle tree.
        float* xs = reinterpret_cast<float*>(smem + S::kXsOff + b * S::kXsBuf);
        constexpr int kSeg = GS / 8;                          // lanes per group
        static_assert(kCpr % 32 == 0, "a pass of the warp covers whole groups of one row");
        for (int i0 = 0; i0 < nch; i0 += 32) {
          const int i = i0 + lane;                            // nch is a multiple of 32
          const int m = i / kCpr, ch = i % kCpr;
          uint4* pc = reinterpret_cast<uint4*>(xb + m * S::kXP + ch * 16);
          const uint4 v = *pc;
          const uint32_t r[4] = {v.x, v.y, v.z, v.w};
          if (M <= kMvPrepSumsMaxM) {                         // warp-uniform
            float sum = 0.0f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              sum += t_to_f(r[e] & 0xFFFFu, kBf16);
              sum += t_to_f(r[e] >> 16, kBf16);
            }
#pragma unroll
            for (int o = 1; o < kSeg; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if ((lane & (kSeg - 1)) == 0) xs[(ch / kSeg) * 16 + m] = sum;
          }
          uint4 ov;
          ov.x = __byte_perm(v.x, v.z, 0x5410);
          ov.y = __byte_perm(v.y, v.w, 0x5410);
          ov.z = __byte_perm(v.x, v.z, 0x7632);
          ov.w = __byte_perm(v.y, v.w, 0x7632);
          *pc = ov;
        }
        __syncwarp();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(xf + b));
      }
    }
  } else {
    // ------------------------------------------------------------ MMA warps
    // Warp w owns rows 16Rw .. 16R(w + 1) - 1 of the unit: R 16-row tiles.
    pdl_wait();                                   // y and the workspace are ordered
    int wc = 0, c = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int u = mv_take(uq, uqf, uqe, k, lane, abort_flag, wl);
      if (u < 0) { ok = u == -1; break; }
      const MvUnit un = mv_unit<P, SUBK>(pr, u);
      const MvProblem& q = pr.prob[un.p];
      float acc[R][NT][4];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[r][nt][i] = 0.0f;
      for (int j = 0; j < un.nsub && ok; ++j) {
        const int buf = c & 1;
        if (!mbar_wait(smem_u32(xf + buf), (c >> 1) & 1, abort_flag, wl)) { ok = false; break; }
        const uint8_t* xb = smem + S::kXOff + buf * S::kXBuf + t * 16;
        float* xsw = reinterpret_cast<float*>(smem + S::kXsOff + buf * S::kXsBuf);
        if (M > kMvPrepSumsMaxM) {
          // Per-group sums of each x row, GPS / kMvWarps groups per warp: an MMA
          // with an all-ones A operand adds the K-steps' columns.
          const uint32_t one[4] = {ones2<T>(), ones2<T>(), ones2<T>(), ones2<T>()};
          constexpr int kGpw = GPS / kMvWarps;
          static_assert(GPS % kMvWarps == 0, "groups per sub-slice split over the MMA warps");
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            float dd[kGpw][4];
#pragma unroll
            for (int bl = 0; bl < GS / 32; ++bl) {
#pragma unroll
              for (int j2 = 0; j2 < kGpw; ++j2) {
                const int gi = warp * kGpw + j2;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (g + 8 * nt < M)
                  v = *reinterpret_cast<const uint4*>(xb + (g + 8 * nt) * S::kXP + (gi * (GS / 32) + bl) * 64);
                if (bl == 0) mma16816_z<T>(dd[j2], one, v.x, v.y);
                else mma16816<T>(dd[j2], one, v.x, v.y);
                mma16816<T>(dd[j2], one, v.z, v.w);
              }
            }
            if (g == 0) {
#pragma unroll
              for (int j2 = 0; j2 < kGpw; ++j2)
                *reinterpret_cast<float2*>(xsw + (warp * kGpw + j2) * 16 + 8 * nt + 2 * t) =
                    make_float2(dd[j2][0], dd[j2][1]);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(xsr + buf));
          if (!mbar_wait(smem_u32(xsr + buf), (c >> 1) & 1, abort_flag, wl)) { ok = false; break; }
        }
        const float* xs = xsw + 2 * t;
        const float2* tab = reinterpret_cast<const float2*>(smem + S::kTabOff + buf * S::kTabBuf) +
                            (warp * 16 * R + g) * S::kTabPitch;
        for (int st = 0; st < S::kSps; ++st) {
          const int slot = wc % ST;
          if (!mbar_wait(smem_u32(full + slot), (wc / ST) & 1, abort_flag, wl)) { ok = false; break; }
          const uint8_t* w0 = smem + S::kRingOff + slot * S::kStage + (warp * 16 * R + g) * 128 + t * 4;
          // NT == 1: two accumulators per tile (the aA and aB K-steps of a word),
          // so a group's MMAs form two chains of half the depth; the epilogue
          // adds them.  With the group's epilogue operands loaded at its first
          // step (below), this measured 1.4 % faster on the batched decode step
          // than one accumulator with the operands loaded at the last step.
          constexpr bool kTwoAcc = NT == 1;
          float d[R][NT][4], d2[R][NT][4];
          // codes of rows g and g + 8 of both tiles, and x, one step ahead
          uint32_t cw[R][2], cn[R][2];
          uint4 xc[NT], xn[NT];
          auto load_step = [&](int s, uint32_t (&w)[R][2], uint4 (&xv)[NT]) {
            const int off = ((s ^ g) << 4);
#pragma unroll
            for (int r = 0; r < R; ++r) {
              w[r][0] = *reinterpret_cast<const uint32_t*>(w0 + r * 16 * 128 + off);
              w[r][1] = *reinterpret_cast<const uint32_t*>(w0 + r * 16 * 128 + 8 * 128 + off);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              xv[nt] = make_uint4(0u, 0u, 0u, 0u);
              if (g + 8 * nt < M)
                xv[nt] = *reinterpret_cast<const uint4*>(xb + (g + 8 * nt) * S::kXP + (st * 8 + s) * 64);
            }
          };
          load_step(0, cw, xc);
          float2 pe0[R], pe1[R], psx[NT];             // the group's (s, b') rows and x sums
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            if ((s & (GS / 32 - 1)) == 0) {             // first step of a group
              const int gi0 = ((st * 8 + s) * 32) / GS;
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                psx[nt] = *reinterpret_cast<const float2*>(xs + gi0 * 16 + 8 * nt);
#pragma unroll
              for (int r = 0; r < R; ++r) {
                pe0[r] = tab[r * 16 * S::kTabPitch + gi0];
                pe1[r] = tab[(r * 16 + 8) * S::kTabPitch + gi0];
              }
            }
            if (s < 7) load_step(s + 1, cn, xn);
            constexpr int kFirstMask = GS / 32 - 1;
            constexpr uint32_t kLo = 0x000F000Fu;
#pragma unroll
            for (int r = 0; r < R; ++r) {
              const uint32_t wa = cw[r][0], wb = cw[r][1];
              uint32_t aA[4], aB[4];
              aA[0] = and_or(wa, kLo, kMag);
              aA[1] = and_or(wb, kLo, kMag);
              aA[2] = and_or(wa >> 8, kLo, kMag);                   // codes 2, 6
              aA[3] = and_or(wb >> 8, kLo, kMag);
              aB[0] = and_or(wa >> 4, kLo, kMag);                   // codes 1, 5
              aB[1] = and_or(wb >> 4, kLo, kMag);
              aB[2] = and_or(wa >> 12, kLo, kMag);                  // codes 3, 7
              aB[3] = and_or(wb >> 12, kLo, kMag);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                if (kTwoAcc) {
                  if ((s & kFirstMask) == 0) {
                    mma16816_z<T>(d[r][nt], aA, xc[nt].x, xc[nt].y);
                    mma16816_z<T>(d2[r][nt], aB, xc[nt].z, xc[nt].w);
                  } else {
                    mma16816<T>(d[r][nt], aA, xc[nt].x, xc[nt].y);
                    mma16816<T>(d2[r][nt], aB, xc[nt].z, xc[nt].w);
                  }
                } else {
                  if ((s & kFirstMask) == 0)
                    mma16816_z<T>(d[r][nt], aA, xc[nt].x, xc[nt].y);
                  else
                    mma16816<T>(d[r][nt], aA, xc[nt].x, xc[nt].y);
                  mma16816<T>(d[r][nt], aB, xc[nt].z, xc[nt].w);
                }
              }
            }
            if ((s & kFirstMask) == kFirstMask) {
              float2 sx[NT];
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) sx[nt] = psx[nt];
#pragma unroll
              for (int r = 0; r < R; ++r) {
                const float2 e0 = pe0[r];
                const float2 e1 = pe1[r];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                  if (kTwoAcc) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) d[r][nt][i] += d2[r][nt][i];
                  }
                  acc[r][nt][0] = fmaf(e0.x, d[r][nt][0], fmaf(e0.y, sx[nt].x, acc[r][nt][0]));
                  acc[r][nt][1] = fmaf(e0.x, d[r][nt][1], fmaf(e0.y, sx[nt].y, acc[r][nt][1]));
                  acc[r][nt][2] = fmaf(e1.x, d[r][nt][2], fmaf(e1.y, sx[nt].x, acc[r][nt][2]));
                  acc[r][nt][3] = fmaf(e1.x, d[r][nt][3], fmaf(e1.y, sx[nt].y, acc[r][nt][3]));
                }
              }
            }
            if (s < 7) {
#pragma unroll
              for (int r = 0; r < R; ++r) { cw[r][0] = cn[r][0]; cw[r][1] = cn[r][1]; }
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) xc[nt] = xn[nt];
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(empty + slot));
          ++wc;
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(xe + buf));
        ++c;
      }
      if (!ok) break;
      // ------------------------------------------------- output of the unit
      T* yp = reinterpret_cast<T*>(q.y);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int tile = un.rb * 8 + warp * R + r;            // 16-row tile of the problem
        const int r0 = tile * 16 + g;
        if (q.splits == 1) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int m = 8 * nt + 2 * t + (i & 1), row = r0 + 8 * (i >> 1);
              if (m < M && row < q.N) yp[(int64_t)m * q.N + row] = TT<T>::from_f(acc[r][nt][i]);
            }
        } else {
          uint32_t* cnt = pr.ws + q.cnt0 + tile;
          float* part = reinterpret_cast<float*>(pr.ws + q.ws_part) + (int64_t)tile * q.splits * M * 16;
          float* mine = part + (int64_t)un.sp * M * 16;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int m = 8 * nt + 2 * t + (i & 1), rr = g + 8 * (i >> 1);
              if (m < M) __stcg(mine + m * 16 + rr, acc[r][nt][i]);
            }
          __syncwarp();                                     // the warp's partial stores ...
          unsigned old = 0;
          if (lane == 0) old = atom_add_release_gpu(cnt, 1u); // ... released with the count
          old = __shfl_sync(0xffffffffu, old, 0);
          if (old == (unsigned)(q.splits - 1)) {
            __threadfence();
            float tot[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int i = 0; i < 4; ++i) tot[nt][i] = 0.0f;
            for (int sl = 0; sl < q.splits; ++sl) {
              const float* ps = part + (int64_t)sl * M * 16;
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int m = 8 * nt + 2 * t + (i & 1), rr = g + 8 * (i >> 1);
                  if (m < M) tot[nt][i] += sl == un.sp ? acc[r][nt][i] : __ldcg(ps + m * 16 + rr);
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int m = 8 * nt + 2 * t + (i & 1), row = r0 + 8 * (i >> 1);
                if (m < M && row < q.N) yp[(int64_t)m * q.N + row] = TT<T>::from_f(tot[nt][i]);
              }
            __syncwarp();
            if (lane == 0) atomicExch(cnt, 0u);
          }
        }
      }
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicOr(&g_aq_device_error, 1u);
}

// ------------------------------------------------------------------- host
// Test hooks (aq_testing.h): wait bound and TMA-warp start delay, in ns.
std::atomic<uint64_t> g_mv_wait_ns{0}, g_mv_delay_ns{0};

struct MvSplit {
  int splits, kslice;
};

// Split K so that the units of one problem fill `slots` CTAs, or so that a
// unit carries about `unit_bytes` of packed weights (batched launches).
MvSplit mv_split(int64_t N, int64_t K, int gs, int64_t slots, int64_t unit_bytes) {
  const int subk = mv_subk(gs);
  const int64_t rbs = (N + kMvRows - 1) / kMvRows;
  const int64_t max_splits = std::max<int64_t>(1, std::min<int64_t>(32, K / subk));
  int64_t want;
  if (unit_bytes > 0)
    want = (kMvRows * K / 2 + unit_bytes / 2) / unit_bytes;
  else
    want = (slots + rbs - 1) / rbs;
  want = std::max<int64_t>(1, std::min(want, max_splits));
  int64_t kslice = (K + want - 1) / want;
  kslice = (kslice + subk - 1) / subk * subk;
  MvSplit d;
  d.kslice = (int)kslice;
  d.splits = (int)((K + kslice - 1) / kslice);
  return d;
}

struct MvGroupPlan {
  MvSplit sp[kMvMaxProblems];
  int cnt0[kMvMaxProblems];
  int64_t part[kMvMaxProblems];
  int64_t words;
};

void mv_plan_group(MvGroupPlan& g, const QmvProblemDesc* probs, int count, int64_t M, int gs,
                   int64_t slots, int64_t unit_bytes) {
  int tiles_used = 0;
  int64_t part = kMvCntWords;
  for (int i = 0; i < count; ++i) {
    MvSplit d = mv_split(probs[i].N, probs[i].K, gs, slots, unit_bytes);
    const int64_t tiles = (probs[i].N + kMvRows - 1) / kMvRows * 8;
    if (d.splits > 1 && tiles_used + tiles > kMvMaxSplitTiles) {
      d.splits = 1;                                   // out of counters: whole rows per unit
      d.kslice = (int)probs[i].K;
    }
    g.sp[i] = d;
    g.cnt0[i] = kMvSchedWords + tiles_used;
    g.part[i] = part;
    if (d.splits > 1) {
      tiles_used += (int)tiles;
      part += (tiles * d.splits * M * 16 + 31) / 32 * 32;
    }
  }
  g.words = part;                                     // the counters are always needed
}

template <typename T, int GS, int NT, int P>
struct MvKernel {
  static constexpr int R = 1;                                 // one 16-row tile per MMA warp
  using S = MvShape<GS, NT, R>;
  static cudaError_t prepare(int* slots) {
    static std::atomic<int> occ[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int o = dev < 64 ? occ[dev].load(std::memory_order_acquire) : 0;
    if (o == 0) {
      auto kern = qmv_mma_kernel<T, GS, NT, R, P>;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
      if (e != cudaSuccess) return e;
      int per_sm = 0, sms = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, S::kThreads, S::kSmem);
      if (e != cudaSuccess) return e;
      e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return e;
      o = std::max(1, per_sm) * sms;
      if (dev < 64) occ[dev].store(o, std::memory_order_release);
    }
    *slots = o;
    return cudaSuccess;
  }
  static cudaError_t launch(const MvParams<P>& pr, int grid, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(S::kThreads, 1, 1);
    cfg.dynamicSmemBytes = S::kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, qmv_mma_kernel<T, GS, NT, R, P>, pr);
  }
};

cudaError_t mv_problem(MvProblem& dp, const QmvProblemDesc& d, int gs, const MvSplit& sp,
                       int cnt0, int64_t part) {
  memset(&dp, 0, sizeof(dp));
  cudaError_t e = make_map(&dp.w, d.w_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d.N, d.K / 2, 128,
                           kMvRows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const int64_t G = d.K / gs;
  const int gps = mv_subk(gs) / gs;
  e = make_map(&dp.s, d.scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, d.N, G, gps, kMvRows,
               CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;
  e = make_map(&dp.b, d.biases, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, d.N, G, gps, kMvRows,
               CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;
  dp.x = d.x;
  dp.y = d.y;
  dp.N = (int)d.N;
  dp.K = (int)d.K;
  dp.splits = sp.splits;
  dp.kslice = sp.kslice;
  dp.cnt0 = cnt0;
  dp.ws_part = part;
  return cudaSuccess;
}

template <typename T, int GS, int NT, int P>
cudaError_t mv_launch_group(const QmvProblemDesc* probs, int count, int64_t M, void* ws,
                            int64_t unit_bytes, cudaStream_t st) {
  static_assert(sizeof(MvParams<P>) <= 32000, "kernel parameter space");
  int slots = 0;
  cudaError_t e = MvKernel<T, GS, NT, P>::prepare(&slots);
  if (e != cudaSuccess) return e;
  // A single matmul runs one CTA per SM: the next kernel of the stream (launched
  // with programmatic dependent launch) then fits beside it and can start
  // streaming its weights while this one finishes.  Batched launches fill
  // both CTA slots of every SM.
  if (unit_bytes == 0) slots = std::max(1, slots / 2);
  MvGroupPlan g;
  mv_plan_group(g, probs, count, M, GS, slots, unit_bytes);
  if (!ws) return cudaErrorInvalidValue;
  MvParams<P> pr;
  memset(&pr, 0, sizeof(pr));
  int units = 0;
  for (int i = 0; i < count; ++i) {
    e = mv_problem(pr.prob[i], probs[i], GS, g.sp[i], g.cnt0[i], g.part[i]);
    if (e != cudaSuccess) return e;
    units += (int)((probs[i].N + kMvRows - 1) / kMvRows) * g.sp[i].splits;
    pr.unit_end[i] = units;
  }
  pr.count = count;
  pr.M = (int)M;
  pr.weights_early = weight_prefetch_enabled();
  pr.ws = reinterpret_cast<uint32_t*>(ws);
  const uint64_t wl = g_mv_wait_ns.load(std::memory_order_relaxed);
  pr.wait_ns = wl ? wl : 2000000000ull;
  pr.delay_ns = g_mv_delay_ns.load(std::memory_order_relaxed);
  const int grid = std::min(units, slots);
  return MvKernel<T, GS, NT, P>::launch(pr, grid, st);
}

template <int P>
cudaError_t mv_dispatch(const QmvProblemDesc* probs, int count, int64_t M, int gs, int dtype,
                        void* ws, int64_t unit_bytes, cudaStream_t st) {
#define AQ_MV_GS(T, NT)                                                                   \
  switch (gs) {                                                                           \
    case 32: return mv_launch_group<T, 32, NT, P>(probs, count, M, ws, unit_bytes, st);   \
    case 64: return mv_launch_group<T, 64, NT, P>(probs, count, M, ws, unit_bytes, st);   \
    case 128: return mv_launch_group<T, 128, NT, P>(probs, count, M, ws, unit_bytes, st); \
    default: return cudaErrorInvalidValue;                                                \
  }
  if (dtype == AQ_F16) {
    if (M <= 8) { AQ_MV_GS(__half, 1) } else { AQ_MV_GS(__half, 2) }
  } else {
    if (M <= 8) { AQ_MV_GS(__nv_bfloat16, 1) } else { AQ_MV_GS(__nv_bfloat16, 2) }
  }
#undef AQ_MV_GS
}

}  // namespace

bool qmv_mma_shape_ok(int64_t N, int64_t K, int bits, int gs, int mode) {
  if (mode != AQ_MODE_AFFINE || bits != 4) return false;
  if (!(gs == 32 || gs == 64 || gs == 128)) return false;
  return N >= 1 && K >= 1 && N <= kMaxRowsDec && K <= kMaxRowsDec && K % mv_subk(gs) == 0;
}

bool qmv_mma_applies(int64_t M, int64_t N, int64_t K, int bits, int gs, int mode,
                     const void* scales, const void* biases) {
  if (M < 1 || M > 16) return false;
  return qmv_mma_shape_ok(N, K, bits, gs, mode) && ((uintptr_t)scales & 15) == 0 &&
         ((uintptr_t)biases & 15) == 0;
}

size_t qmv_mma_workspace(int64_t M, int64_t N, int64_t K, int gs) {
  const QmvProblemDesc d{nullptr, nullptr, nullptr, nullptr, nullptr, N, K};
  // The split depends on the resident CTA count; plan for the most splits
  // any device can ask for (up to every sub-slice its own slice).
  MvGroupPlan g;
  mv_plan_group(g, &d, 1, M, gs, 1 << 30, 0);
  return (size_t)g.words * 4;
}

size_t qmv_mma_batched_workspace(const QmvProblemDesc* probs, int count, int64_t M, int gs) {
  int64_t best = 0;
  for (int i0 = 0; i0 < count; i0 += kMvMaxProblems) {
    MvGroupPlan g;
    mv_plan_group(g, probs + i0, std::min(count - i0, kMvMaxProblems), M, gs, 0, kDecUnitBytes);
    best = std::max(best, g.words);
  }
  return (size_t)best * 4;
}

cudaError_t launch_qmv_mma(const void* x, const void* w_q, const void* scales,
                           const void* biases, void* y, int64_t M, int64_t N, int64_t K, int gs,
                           int dtype, void* ws, cudaStream_t st) {
  QmvProblemDesc d{x, w_q, scales, biases, y, N, K};
  return mv_dispatch<1>(&d, 1, M, gs, dtype, ws, 0, st);
}

cudaError_t launch_qmv_mma_batched(const QmvProblemDesc* probs, int count, int64_t M, int gs,
                                   int dtype, void* ws, cudaStream_t st) {
  for (int i0 = 0; i0 < count; i0 += kMvMaxProblems) {
    const int n = std::min(count - i0, kMvMaxProblems);
    cudaError_t e = mv_dispatch<kMvMaxProblems>(probs + i0, n, M, gs, dtype, ws, kDecUnitBytes, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t read_device_error_qmv_mma(unsigned* out) { return read_tu_error(out); }

void testing_set_mv_wait_ns(uint64_t ns) { g_mv_wait_ns.store(ns, std::memory_order_relaxed); }
void testing_set_mv_delay_ns(uint64_t ns) { g_mv_delay_ns.store(ns, std::memory_order_relaxed); }
cudaError_t testing_clear_device_error_qmv_mma() {
  const unsigned z = 0;
  return cudaMemcpyToSymbol(g_aq_device_error, &z, sizeof(z));
}

// ------------------------------------------------ no-allocation entry point
// Scratch of aq_qmv_noalloc, in place of a caller-supplied workspace: the
// unit and split-K counters (its first 64 KB, which must start at zero: the
// array is zero when the module loads, and every call that completes leaves
// them zero) and the fp32 split-K partials.  Every call on a device shares
// it, so calls whose kernels may overlap on the GPU (other streams, or no
// ordering between them) race on it.
static __device__ __align__(256) unsigned char g_qmv_scratch[kQmvNoallocScratchBytes];

namespace {
std::atomic<void*> g_scratch_ptr[64];
}  // namespace

cudaError_t launch_qmv_noalloc(const void* x, const void* w_q, const void* scales,
                               const void* biases, void* y, int64_t M, int64_t N, int64_t K,
                               int gs, int dtype, cudaStream_t st, size_t* need) {
  *need = qmv_mma_workspace(M, N, K, gs);
  if (*need > kQmvNoallocScratchBytes) return cudaErrorMemoryAllocation;   // caller reports
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64) return cudaErrorInvalidDevice;
  // Set-up on the first call on this device (with it current): the address
  // of the scratch array in this device's copy of the module.
  void* ptr = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!ptr) {
    e = cudaGetSymbolAddress(&ptr, g_qmv_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev].store(ptr, std::memory_order_release);
  }
  return launch_qmv_mma(x, w_q, scales, biases, y, M, N, K, gs, dtype, ptr, st);
}

}  // namespace aq
