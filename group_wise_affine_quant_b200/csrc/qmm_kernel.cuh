// qmm_kernel.cuh — the tcgen05 quantized-matmul kernel template shared by the
// dense entry (qmm.cu) and the implicit-GEMM conv entry (conv.cu).
#pragma once
//
// Tensor-core quantized matmul y = x . dequant(W)^T (tcgen05 + TMEM).
//
// Prior art: affine_packed_qmm_t in "Add the 3bit packed qmm_t" (a block
// loader dequantizes a weight tile into threadgroup memory, then a simdgroup
// MMA).  The B200 design, per CTA and output tile of 128 weight rows x BT
// rows of x:
//   * The weight is the MMA's A operand (M = 128 rows of N) and x is the B
//     operand (N = BT in 16..256 rows of M), so a decode-sized M still fills a
//     full 128-row MMA: one wave of tiles covers M = 1..64 at the weight
//     stream's cost.
//   * Warp 0 is the x producer: a warp-uniform loop whose elected lane issues
//     each x tile's TMA into 128-byte-swizzled shared memory (or, for the
//     conv, 4-D boxes per filter tap / a cp.async gather).  Warp 1 allocates
//     TMEM and issues the tcgen05.mma (kind::f16, fp32 accumulate in TMEM)
//     from an elected lane, one wait and one commit per stage.  The last warp
//     streams the packed codes and the scale / bias chunks by TMA (128 rows x
//     128 bytes, 128-byte swizzle) into a ring, or by cp.async when the rows
//     are not 16-byte multiples.  Warps 2 .. 2+4G-1 are G groups of four
//     dequantizers on interleaved K-stages (one weight row per thread): they
//     form w_hat = s*q + b in T with packed FMAs (single rounding, the value
//     aq_dequantize writes) and store it into tensor memory with
//     tcgen05.st; the MMA reads its A operand from TMEM, so the dequantized
//     tile never passes through shared memory.  Stages hand over through
//     mbarriers; the MMA's commit frees an operand slot for both producers.
//   * K-step 64 (one 128-byte swizzle atom of 16-bit values); a K tail of 32
//     reads zero x through TMA's out-of-bounds fill and writes zero w_hat.
//   * The epilogue (the dequantizer warps) reads TMEM with tcgen05.ld and
//     stores y through shared memory in 16-byte runs.  With split-K the
//     K-slices of a tile form a thread block cluster: each CTA parks its fp32
//     tile in shared memory and the slices are added in slice order through
//     distributed shared memory.  No workspace, no global atomics.
//   * Every mbarrier wait is bounded (2 s); a timeout sets a device error
//     flag, every role stops issuing work and the CTA frees its TMEM.
#include <atomic>
#include <cooperative_groups.h>

#include <string.h>

#include <type_traits>

#include "common.cuh"
#include "sm100.cuh"

namespace cg = cooperative_groups;

namespace aq {

namespace {

// Per translation unit; bit 0: a kernel's bounded wait timed out.
__device__ unsigned int g_aq_device_error = 0u;

using namespace sm100;

constexpr int kBK = 64;                  // K elements per stage (128 bytes of T)
constexpr int kRowsW = 128;              // weight rows per tile (MMA M)
constexpr int kProducerWarp0 = 2;        // warps 2 .. : dequantizer groups of 4 warps

template <int BT, int BITS, bool FAST>
struct QmmShape {
  // Small token tiles (BT <= 32, the weight-streaming regime) use a light
  // CTA (2 dequantizer groups, about 95 KB of shared memory) so that two
  // CTAs fit on an SM: the next kernel of a stream can then start streaming
  // its weights while this one finishes.  Larger tiles use a deeper pipeline.
  static constexpr bool kLight = BT <= 32;
  // Operand stages: K-stage i fills slot i % kStages of both rings, the
  // dequantized A tile in tensor memory (the dequantizers refill it from
  // shared memory; the MMA reads A from TMEM, which keeps the A tile out of
  // the shared-memory bandwidth) and the x tile in shared memory (TMA from
  // L2/HBM).  One "full" barrier per slot takes the dequantizers' arrivals
  // and the x tile's, and one MMA commit frees both halves of the slot, so
  // the MMA issuer waits once and commits once per stage.  (Deeper rings,
  // 5 slots at BT = 256 and 8 below, measured a few percent slower.)
  static constexpr int kStages = kLight ? 3 : 4;
  static constexpr int kBStages = kStages;
  static constexpr int kBBytes = BT * kBK * 2;                       // BT * 128
  static constexpr int kPB = 8 * BITS;                               // packed bytes / row / stage
  // cp.async path: one slot per stage, rows at a bank-spreading pitch.
  static constexpr int kPStages = kLight ? 4 : BT >= 256 ? 4 : BT >= 128 ? 6 : 8;
  static constexpr int kRP = (kPB % 32 == 0) ? kPB + 16 : kPB;
  static constexpr int kPSlot = kRowsW * kRP + kRowsW * 16;
  // TMA path: weight chunks of 128 rows x 128 bytes (128-byte swizzle) and
  // scale chunks of 128 rows x 16 bytes (scales, then biases).
  // A chunk slot is refilled only after every group has passed the chunk,
  // and the refill comes from HBM (a few microseconds): four slots cover 16
  // K-stages of 4-bit codes (8 of 8-bit), so the refill lands before the
  // first group reaches it.
  static constexpr int kWChunk = kRowsW * 128;                       // 16 KB
  static constexpr int kWSlots = kLight ? 2 : 4;
  static constexpr int kSChunk = kRowsW * 16 * 2;                    // 4 KB
  static constexpr int kSSlots = kLight ? 2 : 4;
  static constexpr int kLoadBytes = FAST ? kWSlots * kWChunk + kSSlots * kSChunk : kPStages * kPSlot;
  static constexpr int kRedBytes = BT * kRowsW * 4;                  // split-K parking
  static constexpr int kRingBytes = kBStages * kBBytes;
  static constexpr int kOpBytes = kRingBytes > kRedBytes ? kRingBytes : kRedBytes;
  static constexpr int kDataBytes = kOpBytes + kLoadBytes;
  // TMEM: the fp32 accumulator in columns [0, kACol0), then kStages A
  // stages of 32 columns (64 16-bit values per lane).
  static constexpr int kACol0 = BT < 32 ? 32 : BT;
  static constexpr int kTmemNeed = kACol0 + 32 * kStages;
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                   : kTmemNeed <= 256 ? 256 : 512;
  // Dequantizer groups: group g takes K-stages i with i % kGroups == g.  A
  // group's consecutive stages are kGroups apart and its operand-slot wait
  // is a phase-parity wait, which is unambiguous only while the slot's
  // previous phase is already complete: that needs kGroups <= kStages.
  static constexpr int kGroups = kLight ? 2 : (kStages < 4 ? kStages : 4);
  static constexpr int kLoaderWarp = kProducerWarp0 + 4 * kGroups;
  static constexpr int kThreads = 32 * (kLoaderWarp + 1);
  static constexpr int kBars = 2 * kStages + 2 * (FAST ? kWSlots + kSSlots : kPStages) + 1;
  static constexpr int kSmem = 1024 + kDataBytes + 512;             // align slack, barriers
  static_assert(kGroups <= kStages, "parity waits need kGroups <= kStages");
  static_assert(kOpBytes >= 4 * kGroups * 1024, "epilogue staging: 1 KB per dequantizer warp");
  static_assert(kBars * 8 + 16 <= 512, "barrier area");
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

struct QmmArgs {
  const uint8_t* wq;
  const void* scales;
  const void* biases;
  void* y;
  int M, N, K;
  int gs_log2;
  int k_tiles;          // ceil(K / 64)
  int k_tiles_split;    // k-tiles per split
  int splits;
  int vec;              // widest cp.async (16, 8 or 4 bytes) the packed rows allow
  int64_t row_bytes;
  // Output tiles are numbered t = tile0 + blockIdx.x; tile t covers x rows
  // [(t / nt_all) * BT, +BT) and column block c = t % nt_all, which holds
  // weight rows g * n_limit + [nt * 128, nt * 128 + 128) with g = c / ntg and
  // nt = c % ntg; rows at or past n_limit (within the block's group) are
  // zero.  y[m, g * n_limit + row] at stride ldy.  Dense: one group.
  int ldy, n_limit, ntg;
  int nt_all;           // column blocks over all groups (ntg * groups)
  int tile0;            // first tile of this launch
  // Implicit-GEMM conv geometry (x is NHWC [Bn, H, W, Cin]; K index =
  // (i * kw + j) * Cg + c over the k_real = kh * kw * Cg real columns).
  int Cin, Cg, H, W, Ho, Wo, kh, kw, sh, sw, ph, pw, k_real;
  const void* x;        // conv gather path
  int weights_early;    // load weights/scales before waiting on the previous kernel
  int x_early;          // read x before waiting on the previous kernel
  int scale_copy;       // TMA path: scale rows are not 16-byte multiples, copy them
  int y_vec;            // y rows and the group's columns allow 16-byte stores (set at launch)
};

struct QmmMaps {
  CUtensorMap x;        // dense: [M, K] T, box {64, BT}, 128-byte swizzle;
                        // conv: [Bn, H, W, Cin] T, box {16, bw, bh, 1}, 32-byte swizzle
  CUtensorMap w;        // [N, row_bytes] u8, box {128, 128}, 128-byte swizzle (TMA path)
  CUtensorMap s;        // [N, G] scales, box {16 bytes, 128} (TMA path)
  CUtensorMap b;        // [N, G] biases, likewise (affine)
};

// ------------------------------------------------------------ cp.async
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
// 16-byte copy reading `src_bytes` (0 or 16) bytes; the rest is zero-filled.
__device__ __forceinline__ void cp_async_16_zfill(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Copy the two 4-byte words starting at the 4-byte boundary at or below
// `p` (a 2- or 1-byte element of an array that ends at `end`) into dst.
// Words that stick out of the array are filled with byte loads of their
// in-bounds part (and zeros) and plain shared stores.
__device__ __forceinline__ void copy_window(uint32_t dst, const uint8_t* p, const uint8_t* begin,
                                            const uint8_t* end) {
  const uint8_t* w0 = reinterpret_cast<const uint8_t*>((uintptr_t)p & ~(uintptr_t)3);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint8_t* w = w0 + 4 * i;
    if (w >= begin && w + 4 <= end) {
      cp_async_4(dst + 4 * i, w);
    } else {
      uint32_t v = 0;
      for (int j = 0; j < 4; ++j)
        if (w + j >= begin && w + j < end) v |= (uint32_t)w[j] << (8 * j);
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(dst + 4 * i), "r"(v) : "memory");
    }
  }
}

// ------------------------------------------------------------- dequantizer
// Per thread and stage: the 64 codes of one weight row as 2*BITS words.
template <int BITS>
struct Packed {
  static constexpr int kWords = 2 * BITS;
  uint32_t w[kWords];
};

template <int BITS>
__device__ __forceinline__ void lds_packed(Packed<BITS>& p, const uint8_t* src) {
  if constexpr ((8 * BITS) % 16 == 0) {
#pragma unroll
    for (int i = 0; i < BITS / 2; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * i);
      p.w[4 * i] = v.x; p.w[4 * i + 1] = v.y; p.w[4 * i + 2] = v.z; p.w[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) {
      const uint2 v = *reinterpret_cast<const uint2*>(src + 8 * i);
      p.w[2 * i] = v.x; p.w[2 * i + 1] = v.y;
    }
  }
}

template <typename T> struct Pair;
template <> struct Pair<__half> {
  static constexpr uint32_t kMagic = 0x64006400u;            // 1024.0 in each half
  static __device__ __forceinline__ uint32_t sub_magic(uint32_t v) {
    __half2 h = *reinterpret_cast<__half2*>(&v);
    h = __hsub2(h, __half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400)));
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ uint32_t fma(uint32_t q, uint32_t s, uint32_t b) {
    __half2 r = __hfma2(*reinterpret_cast<__half2*>(&q), *reinterpret_cast<__half2*>(&s),
                        *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
  static __device__ __forceinline__ uint32_t mul(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
  static __device__ __forceinline__ uint32_t from_f2(float lo, float hi) {
    __half2 r = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
  }
  static constexpr int kMagicMaxCode = 1023;
};
template <> struct Pair<__nv_bfloat16> {
  static constexpr uint32_t kMagic = 0x43004300u;            // 128.0 in each half
  static __device__ __forceinline__ uint32_t sub_magic(uint32_t v) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&v);
    h = __hsub2(h, __nv_bfloat162(__ushort_as_bfloat16(0x4300), __ushort_as_bfloat16(0x4300)));
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ uint32_t fma(uint32_t q, uint32_t s, uint32_t b) {
    __nv_bfloat162 r = __hfma2(*reinterpret_cast<__nv_bfloat162*>(&q),
                               *reinterpret_cast<__nv_bfloat162*>(&s),
                               *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
  static __device__ __forceinline__ uint32_t mul(uint32_t a, uint32_t b) {
    __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a),
                               *reinterpret_cast<__nv_bfloat162*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
  }
  static __device__ __forceinline__ uint32_t from_f2(float lo, float hi) {
    __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
  }
  static constexpr int kMagicMaxCode = 127;
};

// Exact codes of elements (2j, 2j+1) of chunk c as a T pair.
template <typename T, int BITS, int C, int J>
__device__ __forceinline__ uint32_t code_pair(const Packed<BITS>& p) {
  constexpr int k0 = 8 * C + 2 * J;
  if constexpr (BITS == 4) {
    // byte J of word C holds codes 2J (low nibble) and 2J+1 (high nibble):
    // put byte J of w at byte 0 and byte J of w >> 4 at byte 2, keep the low
    // nibbles, OR in the magic exponent and subtract it.
    const uint32_t w = p.w[C];
    constexpr uint32_t sel = (uint32_t)J | ((uint32_t)J << 4) | ((uint32_t)(J + 4) << 8) |
                             ((uint32_t)(J + 4) << 12);
    const uint32_t t = __byte_perm(w, w >> 4, sel);
    return Pair<T>::sub_magic((t & 0x000F000Fu) | Pair<T>::kMagic);
  } else if constexpr (BITS == 8 && std::is_same<T, __nv_bfloat16>::value) {
    const float lo = u_to_f_exact(code_at<8, k0>(p.w));
    const float hi = u_to_f_exact(code_at<8, k0 + 1>(p.w));
    return Pair<T>::from_f2(lo, hi);
  } else {
    const uint32_t lo = code_at<BITS, k0>(p.w);
    const uint32_t hi = code_at<BITS, k0 + 1>(p.w);
    return Pair<T>::sub_magic(lo | (hi << 16) | Pair<T>::kMagic);
  }
}

// E2M1 magnitudes (code & 7: 0, 0.5, 1, 1.5, 2, 3, 4, 6) as T, split into
// high and low bytes so that one byte permute looks up four codes at once.
template <typename T> struct Fp4Bytes;
template <> struct Fp4Bytes<__nv_bfloat16> {
  static constexpr uint32_t kHi0 = 0x3F3F3F00u, kHi1 = 0x40404040u;   // 0x00 0x3F 0x3F 0x3F | 0x40 x4
  static constexpr uint32_t kLo0 = 0xC0800000u, kLo1 = 0xC0804000u;   // 0x00 0x00 0x80 0xC0 | 0x00 0x40 0x80 0xC0
};
template <> struct Fp4Bytes<__half> {
  static constexpr uint32_t kHi0 = 0x3E3C3800u, kHi1 = 0x46444240u;   // 0x00 0x38 0x3C 0x3E | 0x40 0x42 0x44 0x46
  static constexpr uint32_t kLo0 = 0u, kLo1 = 0u;
};

// The four E2M1 codes in the low 16 bits of h (code i in bits 4i..4i+3,
// bit 3 the sign) as two T pairs in code order: exact values, no rounding.
template <typename T>
__device__ __forceinline__ void fp4_quad(uint32_t h, uint32_t& pa, uint32_t& pb) {
  const uint32_t sel = h & 0x7777u;                     // magnitude index per code
  const uint32_t sg = h & 0x8888u;                      // sign bits
  uint32_t hi = __byte_perm(Fp4Bytes<T>::kHi0, Fp4Bytes<T>::kHi1, sel);
  // sign of code i into bit 7 of byte i: bytes of (sg << 4) carry codes 0 and
  // 2 at bit 7, bytes of sg carry codes 1 and 3 there
  hi |= __byte_perm(sg << 4, sg, 0x5140) & 0x80808080u;
  const uint32_t lo = __byte_perm(Fp4Bytes<T>::kLo0, Fp4Bytes<T>::kLo1, sel);
  pa = __byte_perm(lo, hi, 0x5140);                     // (code 0, code 1)
  pb = __byte_perm(lo, hi, 0x7362);                     // (code 2, code 3)
}

// Dequantize chunk C (8 elements) into 16 bytes.
template <typename T, int BITS, bool FP4, int C>
__device__ __forceinline__ uint4 dequant_chunk(const Packed<BITS>& p, uint32_t s2, uint32_t b2) {
  uint4 o;
  if constexpr (FP4) {
    // 8 codes of chunk C are word C (4-bit, low nibble first)
    uint32_t q0, q1, q2, q3;
    fp4_quad<T>(p.w[C], q0, q1);
    fp4_quad<T>(p.w[C] >> 16, q2, q3);
    o.x = Pair<T>::mul(q0, s2);
    o.y = Pair<T>::mul(q1, s2);
    o.z = Pair<T>::mul(q2, s2);
    o.w = Pair<T>::mul(q3, s2);
  } else {
    o.x = Pair<T>::fma(code_pair<T, BITS, C, 0>(p), s2, b2);
    o.y = Pair<T>::fma(code_pair<T, BITS, C, 1>(p), s2, b2);
    o.z = Pair<T>::fma(code_pair<T, BITS, C, 2>(p), s2, b2);
    o.w = Pair<T>::fma(code_pair<T, BITS, C, 3>(p), s2, b2);
  }
  return o;
}

template <typename T>
__device__ __forceinline__ uint32_t splat(T v) {
  const uint16_t u = *reinterpret_cast<const uint16_t*>(&v);
  return (uint32_t)u | ((uint32_t)u << 16);
}

// Scale/bias pairs (splatted T) for the two 32-element halves of a stage;
// FP4 at group 16 keeps its four quarter scales in s[0], s[1], b[0], b[1].
struct StageSB {
  uint32_t s[2], b[2];
};

__device__ __forceinline__ uint32_t u16_at(uint32_t w0, uint32_t w1, int byte_off) {
  const uint64_t v = ((uint64_t)w1 << 32) | w0;
  return (uint32_t)(v >> (8 * byte_off)) & 0xFFFFu;
}
__device__ __forceinline__ uint32_t u8_at(uint32_t w0, uint32_t w1, int byte_off) {
  const uint64_t v = ((uint64_t)w1 << 32) | w0;
  return (uint32_t)(v >> (8 * byte_off)) & 0xFFu;
}

// Decode the staged words of one row into the stage's scale/bias pairs.
template <typename T, bool FP4>
__device__ __forceinline__ StageSB sb_from_words(const uint4 wv, const QmmArgs& a, int64_t row,
                                                 int kt, int G, bool tail) {
  StageSB r;
  const int k = kt * kBK;
  const int g0 = k >> a.gs_log2;
  const int g1 = tail ? g0 : (k + 32) >> a.gs_log2;
  if constexpr (FP4) {
    const uint8_t* p = reinterpret_cast<const uint8_t*>(a.scales) + row * G + g0;
    const int off = (int)((uintptr_t)p & 3);
    auto sc = [&](int d) {
      return splat(TT<T>::from_f(fp4_scale_t<T>(u8_at(wv.x, wv.y, off + d), 1 << a.gs_log2)));
    };
    if (a.gs_log2 == 4) {
      r.s[0] = sc(0);
      r.s[1] = sc(1);
      r.b[0] = tail ? r.s[0] : sc(2);
      r.b[1] = tail ? r.s[0] : sc(3);
    } else {
      r.s[0] = sc(0);
      r.s[1] = sc(g1 - g0);
      r.b[0] = r.b[1] = 0u;
    }
  } else {
    const int offs = (int)(((uintptr_t)a.scales + 2 * (row * G + g0)) & 3);
    const int offb = (int)(((uintptr_t)a.biases + 2 * (row * G + g0)) & 3);
    const uint32_t s0 = u16_at(wv.x, wv.y, offs), s1 = u16_at(wv.x, wv.y, offs + 2 * (g1 - g0));
    const uint32_t b0 = u16_at(wv.z, wv.w, offb), b1 = u16_at(wv.z, wv.w, offb + 2 * (g1 - g0));
    r.s[0] = s0 | (s0 << 16);
    r.s[1] = s1 | (s1 << 16);
    r.b[0] = b0 | (b0 << 16);
    r.b[1] = b1 | (b1 << 16);
  }
  return r;
}

// Dequantize one weight row of a K-stage (64 codes) into 32 words (T pairs
// in K order), the layout of an A operand in tensor memory: lane = row, two
// 16-bit values per column.  With `tail` the upper 32 columns are zero.
// Raw scale / bias values of one row for K-stage kt, straight from global
// memory (rows of scales that TMA cannot address): affine {s(g0), s(g1),
// b(g0), b(g1)}; FP4 the scale bytes of the stage's groups (four at group
// 16, two at group 32).  g1 is the group of the stage's second half.
template <bool FP4>
__device__ __forceinline__ void load_stage_scales(uint32_t (&raw)[4], const void* scales,
                                                  const void* biases, int64_t row, int G, int kt,
                                                  int gs_log2, int K, bool valid) {
  raw[0] = raw[1] = raw[2] = raw[3] = 0u;
  if (!valid) return;
  const bool tail = (kt + 1) * 64 > K;
  const int g0 = (kt * 64) >> gs_log2;
  if constexpr (FP4) {
    const uint8_t* sp = reinterpret_cast<const uint8_t*>(scales) + row * G;
    if (gs_log2 == 4) {
      raw[0] = sp[g0]; raw[1] = sp[g0 + 1];
      if (!tail) { raw[2] = sp[g0 + 2]; raw[3] = sp[g0 + 3]; }
    } else {
      raw[0] = sp[g0]; raw[1] = tail ? raw[0] : sp[(kt * 64 + 32) >> gs_log2];
    }
  } else {
    const int g1 = tail ? g0 : ((kt * 64 + 32) >> gs_log2);
    const uint16_t* sp = reinterpret_cast<const uint16_t*>(scales) + row * G;
    const uint16_t* bp = reinterpret_cast<const uint16_t*>(biases) + row * G;
    raw[0] = sp[g0]; raw[1] = sp[g1]; raw[2] = bp[g0]; raw[3] = bp[g1];
  }
}

template <typename T, int BITS, bool FP4>
__device__ __forceinline__ void dequant_row(const Packed<BITS>& p, const StageSB& sb, bool fp4_g16,
                                            bool tail, uint32_t (&o)[32]) {
  auto put = [&](int c, uint4 v) { o[4 * c] = v.x; o[4 * c + 1] = v.y; o[4 * c + 2] = v.z; o[4 * c + 3] = v.w; };
  if constexpr (FP4) {
    // quarters of 16 elements: scales s0 s1 (group 16: b0 b1 hold quarters 2, 3)
    const uint32_t q0 = sb.s[0];
    const uint32_t q1 = fp4_g16 ? sb.s[1] : sb.s[0];
    const uint32_t q2 = fp4_g16 ? sb.b[0] : sb.s[1];
    const uint32_t q3 = fp4_g16 ? sb.b[1] : sb.s[1];
    put(0, dequant_chunk<T, BITS, FP4, 0>(p, q0, 0u));
    put(1, dequant_chunk<T, BITS, FP4, 1>(p, q0, 0u));
    put(2, dequant_chunk<T, BITS, FP4, 2>(p, q1, 0u));
    put(3, dequant_chunk<T, BITS, FP4, 3>(p, q1, 0u));
    put(4, dequant_chunk<T, BITS, FP4, 4>(p, q2, 0u));
    put(5, dequant_chunk<T, BITS, FP4, 5>(p, q2, 0u));
    put(6, dequant_chunk<T, BITS, FP4, 6>(p, q3, 0u));
    put(7, dequant_chunk<T, BITS, FP4, 7>(p, q3, 0u));
  } else {
    put(0, dequant_chunk<T, BITS, FP4, 0>(p, sb.s[0], sb.b[0]));
    put(1, dequant_chunk<T, BITS, FP4, 1>(p, sb.s[0], sb.b[0]));
    put(2, dequant_chunk<T, BITS, FP4, 2>(p, sb.s[0], sb.b[0]));
    put(3, dequant_chunk<T, BITS, FP4, 3>(p, sb.s[0], sb.b[0]));
    put(4, dequant_chunk<T, BITS, FP4, 4>(p, sb.s[1], sb.b[1]));
    put(5, dequant_chunk<T, BITS, FP4, 5>(p, sb.s[1], sb.b[1]));
    put(6, dequant_chunk<T, BITS, FP4, 6>(p, sb.s[1], sb.b[1]));
    put(7, dequant_chunk<T, BITS, FP4, 7>(p, sb.s[1], sb.b[1]));
  }
  if (tail) {
#pragma unroll
    for (int c = 16; c < 32; ++c) o[c] = 0u;
  }
}

// -------------------------------------------------------------------- kernel
// Shared memory offset of byte `o` of row r within a chain of 128-byte
// weight chunks (128-byte swizzle: 16-byte unit u of row r sits at unit
// u ^ (r % 8)).
__device__ __forceinline__ uint32_t wchunk_off(int o, int r) {
  return (uint32_t)(r * 128 + ((((o >> 4) & 7) ^ (r & 7)) << 4) + (o & 15));
}

// XMODE: 0 = dense x by 2-D TMA; 3 = conv pixels by one 4-D TMA box of 64
// channels per K-stage (Cg % 64 == 0, 128-byte swizzle); 1 = conv pixels by
// 4-D TMA boxes (one per
// 16-channel atom column of a K-stage, 32-byte swizzle); 2 = conv pixels
// gathered with cp.async (16-byte granules, zero-filled outside the image).
template <typename T, int BITS, bool FP4, int BT, bool FAST, int XMODE>
__global__ void __launch_bounds__(QmmShape<BT, BITS, FAST>::kThreads,
                                  QmmShape<BT, BITS, FAST>::kLight ? 2 : 1)
qmm_tc_kernel(const __grid_constant__ QmmMaps maps, const QmmArgs a) {
  using S = QmmShape<BT, BITS, FAST>;
  constexpr int kDqGroups = S::kGroups;
  constexpr int kLoaderWarp = S::kLoaderWarp;
  constexpr int kThreads = S::kThreads;
  constexpr int ST = S::kStages;                          // operand slots (A and B)
  constexpr int SB = S::kBStages;                         // == ST
  constexpr int PST = S::kPStages;
  constexpr int WS = S::kWSlots;
  constexpr int SS = S::kSSlots;
  constexpr int SGC = FP4 ? 16 : 8;                       // groups per scale chunk (16 bytes)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = smem;                                   // operand rings (and split-K parking)
  uint8_t* ring_b = smem;                                 // [SB] B BT*128
  uint8_t* pring = smem + S::kOpBytes;                    // loader area
  uint8_t* wring = pring;                                 // TMA path: [WS] weight chunks
  uint8_t* sring = pring + WS * S::kWChunk;               // TMA path: [SS] scale chunks
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kDataBytes);
  constexpr int NL = FAST ? WS + SS : PST;                // loader slots
  // bars: full[ST], empty[ST], full_l[NL], empty_l[NL], acc_full
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + S::kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = a.tile0 + (int)blockIdx.x;
  const int cblk = tile % a.nt_all;                       // column block
  const int cgrp = cblk / a.ntg;                          // conv group (0 when dense)
  const int nl0 = (cblk - cgrp * a.ntg) * kRowsW;         // first row within the group
  const int n0 = cgrp * a.n_limit + nl0;                  // first weight row
  const int m0 = (tile / a.nt_all) * BT;
  const int split = blockIdx.z;
  const int kt0 = split * a.k_tiles_split;
  const int kt1 = min(a.k_tiles, kt0 + a.k_tiles_split);
  const int nkt = kt1 - kt0;                              // >= 1
  const int G = a.K >> a.gs_log2;

  static_assert(SB == ST, "one barrier pair per operand slot");
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + ST + s); };
  auto full_l = [&](int s) { return smem_u32(bars + 2 * ST + s); };
  auto empty_l = [&](int s) { return smem_u32(bars + 2 * ST + NL + s); };
  const uint32_t acc_full = smem_u32(bars + 2 * ST + 2 * NL);

  // TMA path bookkeeping: weight chunk c covers bytes [wb0 + 128 c, +128) of
  // every row, scale chunk j covers groups [SGC j, SGC (j + 1)).
  const int64_t wb0 = (int64_t)kt0 * S::kPB;              // 16-byte aligned (host plan)
  const int nwc = (int)((nkt * S::kPB + 127) / 128);
  const int sc0 = ((kt0 * kBK) >> a.gs_log2) / SGC;
  const int sc1 = (((kt1 * kBK) - 1) >> a.gs_log2) / SGC;
  const int nsc = a.scale_copy ? 0 : sc1 - sc0 + 1;    // scale chunks (none: read from global)

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      // one arrive per dequantizer warp, plus the x tile's: the TMA
      // producer's arrive (with the tile's bytes as tx), or every gather lane
      mbar_init(full(s), 4 + (XMODE == 2 ? 32 : 1));
      mbar_init(empty(s), 1);           // MMA commit
    }
    for (int s = 0; s < NL; ++s) {
      mbar_init(full_l(s), FAST ? 1 : 32);   // TMA arrive + tx, or every loader lane
      // TMA path: every dequantizer group releases every chunk (after its
      // data has landed); cp.async path: one stage, one group.
      mbar_init(empty_l(s), FAST ? 4 * kDqGroups : 4);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), S::kTmemCols);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Programmatic dependent launch: the next kernel in the stream may start
  // its prologue now; it waits for this grid before touching its own inputs.
  pdl_launch_dependents();

  if (warp == 0) {
    if (!a.x_early) pdl_wait();                           // x may come from the previous kernel
    if constexpr (XMODE != 2) {
      // ------------------------------------------------- TMA producer (x)
      // The whole warp runs the loop (warp-uniform waits and coordinates);
      // one elected lane issues the copies.  Conv coordinates advance
      // incrementally: (tap, c) is the filter tap and the channel within the
      // conv group of the stage's first K column, (dy, dx) the tap's offset.
      //   XMODE 0: x rows [m0, m0 + BT) x K columns [kk, kk + 64), 2-D box;
      //   XMODE 3: one 64-channel 4-D box (Cg % 64 == 0: one tap per stage);
      //   XMODE 1: four 16-channel 4-D boxes, one per atom column.
      int bimg = 0, ho0 = 0, wo0 = 0, taps = 0, tap = 0, c = 0, dy = 0, dx = 0;
      int kk = kt0 * kBK;
      if constexpr (XMODE != 0) {
        const int hw = a.Ho * a.Wo;
        bimg = m0 / hw;
        const int rem = m0 - bimg * hw;
        ho0 = rem / a.Wo;
        wo0 = rem - ho0 * a.Wo;
        taps = a.kh * a.kw;
        tap = kk / a.Cg;
        c = kk - tap * a.Cg;
        dy = tap / a.kw;
        dx = tap - dy * a.kw;
      }
      for (int i = 0; i < nkt; ++i) {
        const int s = i % SB;
        const uint32_t par = ((i / SB) & 1) ^ 1;
        if (!__all_sync(0xffffffffu, mbar_wait(empty(s), par, abort_flag))) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(full(s), S::kBBytes);
          const uint32_t dst = smem_u32(ring_b + s * S::kBBytes);
          if constexpr (XMODE == 0) {
            tma_load_2d(dst, &maps.x, full(s), kk, m0);
          } else if constexpr (XMODE == 3) {
            const bool in = tap < taps && kk < a.k_real;   // else past the image: zero fill
            tma_load_4d(dst, &maps.x, full(s), in ? cgrp * a.Cg + c : 0, in ? wo0 - a.pw + dx : 0,
                        in ? ho0 - a.ph + dy : a.H, bimg);
          } else {
            int t2 = tap, c2 = c, dy2 = dy, dx2 = dx;
#pragma unroll
            for (int at = 0; at < 4; ++at) {
              const bool in = t2 < taps && kk + 16 * at < a.k_real;
              tma_load_4d(dst + at * (BT * 32), &maps.x, full(s), in ? cgrp * a.Cg + c2 : 0,
                          in ? wo0 - a.pw + dx2 : 0, in ? ho0 - a.ph + dy2 : a.H, bimg);
              c2 += 16;                                    // Cg % 16 == 0: exact wrap
              if (c2 >= a.Cg) {
                c2 = 0;
                ++t2;
                if (++dx2 == a.kw) { dx2 = 0; ++dy2; }
              }
            }
          }
        }
        __syncwarp();
        kk += kBK;
        if constexpr (XMODE != 0) {
          c += kBK;
          while (c >= a.Cg) {
            c -= a.Cg;
            ++tap;
            if (++dx == a.kw) { dx = 0; ++dy; }
          }
        }
      }
    } else {
      // ------------------ conv pixels: cp.async gather of 16-byte granules
      constexpr int kLagB = SB - 1;
      const int taps = a.kh * a.kw;
      const int hw = a.Ho * a.Wo;
      int published = 0;
      for (int i = 0; i < nkt; ++i) {
        const int s = i % SB;
        const uint32_t par = ((i / SB) & 1) ^ 1;
        if (!mbar_wait(empty(s), par, abort_flag)) break;
        const uint32_t dst = smem_u32(ring_b + s * S::kBBytes);
        for (int idx = lane; idx < BT * 8; idx += 32) {
          const int j = idx >> 3, q = idx & 7;           // pixel row, granule of 8 channels
          const int kk = (kt0 + i) * kBK + 8 * q;
          const int tap = kk / a.Cg, c = kk - (kk / a.Cg) * a.Cg;
          const int m = m0 + j;
          const T* src = reinterpret_cast<const T*>(a.x);
          bool valid = m < a.M && tap < taps && kk < a.k_real;
          if (valid) {
            const int bimg = m / hw, rem = m - (m / hw) * hw;
            const int ho = rem / a.Wo, wo = rem - (rem / a.Wo) * a.Wo;
            const int hi = ho * a.sh - a.ph + tap / a.kw;
            const int wi = wo * a.sw - a.pw + tap % a.kw;
            valid = hi >= 0 && hi < a.H && wi >= 0 && wi < a.W;
            if (valid)
              src += (((int64_t)bimg * a.H + hi) * a.W + wi) * a.Cin + cgrp * a.Cg + c;
          }
          // atom column q/2, half q%2; 32-byte swizzle: 16-byte chunk ^= row bit 2
          const uint32_t d = dst + (q >> 1) * (BT * 32) + j * 32 + ((((q & 1) ^ (j >> 2)) & 1) << 4);
          cp_async_16_zfill(d, src, valid ? 16 : 0);
        }
        cp_async_commit();
        if (i - kLagB >= 0) {
          cp_async_wait_group<kLagB>();
          mbar_arrive(full((i - kLagB) % SB));
          published = i - kLagB + 1;
        }
      }
      cp_async_wait_all();
      if (!*abort_flag) {
        for (int i = published; i < nkt; ++i) mbar_arrive(full(i % SB));
      }
    }
  } else if (warp == kLoaderWarp) {
    // Weights, scales and biases are read before the dependency wait only when
    // the caller has declared that no preceding kernel writes them.
    if (!a.weights_early) pdl_wait();
    if constexpr (FAST) {
      // ------------------- weight and scale chunks in K order
      // Weight and scale chunks by TMA (lane 0; the warp follows lane 0's
      // wait result, so a failed wait leaves the loop together).  When the
      // rows of scales are not 16-byte multiples there are no scale chunks:
      // the dequantizers read their scales from global memory.
      int c = 0, j = 0;
      while (c < nwc || j < nsc) {
        // K position (in codes, relative to kt0 * 64) where each chunk starts
        const int64_t kw = c < nwc ? (int64_t)c * 128 * 8 / BITS : INT64_MAX;
        const int64_t ks = j < nsc ? (int64_t)(sc0 + j) * SGC * (1 << a.gs_log2) - (int64_t)kt0 * kBK
                                   : INT64_MAX;
        if (kw <= ks) {
          const int slot = c % WS;
          bool ok = true;
          if (lane == 0) {
            ok = mbar_wait(empty_l(slot), ((c / WS) & 1) ^ 1, abort_flag);
            if (ok) {
              mbar_arrive_expect_tx(full_l(slot), S::kWChunk);
              tma_load_2d(smem_u32(wring + slot * S::kWChunk), &maps.w, full_l(slot),
                          (int)(wb0 + 128 * c), n0);
            }
          }
          if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
          ++c;
        } else {
          const int slot = j % SS;
          bool ok = true;
          if (lane == 0) {
            ok = mbar_wait(empty_l(WS + slot), ((j / SS) & 1) ^ 1, abort_flag);
            if (ok) {
              const uint32_t dst = smem_u32(sring + slot * S::kSChunk);
              mbar_arrive_expect_tx(full_l(WS + slot), FP4 ? kRowsW * 16 : 2 * kRowsW * 16);
              tma_load_2d(dst, &maps.s, full_l(WS + slot), (sc0 + j) * SGC, n0);
              if constexpr (!FP4)
                tma_load_2d(dst + kRowsW * 16, &maps.b, full_l(WS + slot), (sc0 + j) * SGC, n0);
            }
          }
          if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
          ++j;
        }
      }
      // On abort, the copies still in flight land before the CTA exits: a
      // bounded wait on the full barrier of every chunk issued in the last
      // lap of each ring (these barriers take only the TMA's bytes).
      if (*abort_flag && lane == 0) {
        auto drain = [&](int base, int slots, int issued) {
          for (int q = issued - 1; q >= 0 && q >= issued - slots; --q) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(full_l(base + q % slots), (q / slots) & 1))
              if (globaltimer_ns() - t0 > 1000000000ull) break;
          }
        };
        drain(0, WS, c);
        drain(WS, SS, j);
      }
      __syncwarp();
    } else {
      // ------------------ packed codes, scales, biases by cp.async
      // Each lane copies 4 rows per stage, one commit group per stage, and
      // keeps kLag stages in flight: after committing stage i it waits for
      // stage i - kLag and publishes it with a release arrive.
      constexpr int kLag = PST - 1;
      const uint8_t* s_begin = reinterpret_cast<const uint8_t*>(a.scales);
      const uint8_t* s_end = s_begin + (int64_t)a.N * G * (FP4 ? 1 : 2);
      const uint8_t* b_begin = reinterpret_cast<const uint8_t*>(a.biases);
      const uint8_t* b_end = b_begin + (int64_t)a.N * G * 2;
      int published = 0;
      for (int i = 0; i < nkt; ++i) {
        const int ps = i % PST;
        const uint32_t par = ((i / PST) & 1) ^ 1;
        if (!mbar_wait(empty_l(ps), par, abort_flag)) break;
        const int kt = kt0 + i;
        const bool tail = (kt + 1) * kBK > a.K;
        const uint32_t slot = smem_u32(pring + ps * S::kPSlot);
#pragma unroll
        for (int jj = 0; jj < kRowsW / 32; ++jj) {
          const int r = lane + 32 * jj;
          const int64_t row = n0 + r;
          if (row >= a.N) continue;
          const uint8_t* src = a.wq + row * a.row_bytes + (int64_t)kt * S::kPB;
          const uint32_t dst = slot + r * S::kRP;
          const int nbytes = tail ? S::kPB / 2 : S::kPB;
          if (a.vec == 16 && !tail) {
#pragma unroll
            for (int o = 0; o < S::kPB; o += 16) cp_async_16(dst + o, src + o);
          } else if (a.vec >= 8 && (nbytes % 8) == 0) {
            for (int o = 0; o < nbytes; o += 8) cp_async_8(dst + o, src + o);
          } else {
            for (int o = 0; o < nbytes; o += 4) cp_async_4(dst + o, src + o);
          }
          const uint32_t wdst = slot + kRowsW * S::kRP + r * 16;
          const int g0 = (kt * kBK) >> a.gs_log2;
          if constexpr (FP4) {
            copy_window(wdst, s_begin + row * G + g0, s_begin, s_end);
          } else {
            copy_window(wdst, s_begin + 2 * (row * G + g0), s_begin, s_end);
            copy_window(wdst + 8, b_begin + 2 * (row * G + g0), b_begin, b_end);
          }
        }
        cp_async_commit();
        if (i - kLag >= 0) {
          cp_async_wait_group<kLag>();
          mbar_arrive(full_l((i - kLag) % PST));
          published = i - kLag + 1;
        }
      }
      cp_async_wait_all();
      if (!*abort_flag) {
        for (int i = published; i < nkt; ++i) mbar_arrive(full_l(i % PST));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    // The whole warp runs the loop (warp-uniform waits and descriptors); one
    // elected lane issues the MMAs and the commits.  A single thread issuing
    // the same sequence spends about twice as long per stage.
    constexpr uint32_t idesc = idesc_f16(std::is_same<T, __nv_bfloat16>::value, kRowsW, BT);
    for (int i = 0; i < nkt; ++i) {
      const int s = i % ST;
      if (!__all_sync(0xffffffffu, mbar_wait(full(s), (i / ST) & 1, abort_flag))) break;
      tc_fence_after();
      const uint32_t a_col = tmem + S::kACol0 + 32 * s;
      const uint32_t b_addr = smem_u32(ring_b + s * S::kBBytes);
      if (elect_one()) {
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          const uint64_t bdesc = (XMODE == 0 || XMODE == 3) ? sdesc_sw128(b_addr + k * 32)
                                            : sdesc_sw32(b_addr + k * (BT * 32));
          mma_f16_tmem_a(tmem, a_col + 8 * k, bdesc, idesc, (i > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(empty(s));                    // frees the A and the x half of slot s
      }
      __syncwarp();
    }
    // Signals the epilogue once every issued MMA has completed (also on
    // abort, so nothing is in flight when TMEM is freed).  The elected lane
    // is the issuing lane (the lowest lane of the full warp).
    if (elect_one()) mma_commit(acc_full);
    __syncwarp();
    // This warp frees TMEM at the end: every MMA it issued has completed by
    // then, also on abort, when the epilogue does not wait for them (bounded).
    {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(acc_full, 0))
        if (globaltimer_ns() - t0 > 1000000000ull) { *abort_flag = 1; break; }
    }
    __syncwarp();
  } else {
    // ------------------------------------------- dequantizers (warps 2..5)
    const int grp = (warp - kProducerWarp0) >> 2;          // dequantizer group
    const int r = (warp & 3) * 32 + lane;                  // weight row in the tile = TMEM lane
    const int64_t row = n0 + r;
    const bool row_ok = nl0 + r < a.n_limit;
    const bool fp4_g16 = FP4 && a.gs_log2 == 4;
    int w_ready = 0, w_freed = 0;                          // TMA path: chunks waited / released
    int s_ready = 0, s_freed = 0;
    // Release weight chunks below w_done and scale chunks below s_done, in
    // the loader's K order (weight chunk first on a tie), waiting for each
    // chunk's data to land just before releasing it.  Every group releases
    // every chunk, so a chunk this group never reads is released too; the
    // wait makes the arrival count toward the right phase of its slot, and
    // the K order means the chunk waited for never sits behind a release this
    // group still owes the loader.
    auto release_upto = [&](int w_done, int s_done) -> bool {
      bool okr = true;
      while (okr && (w_freed < w_done || s_freed < s_done)) {
        const int64_t kw = w_freed < w_done ? (int64_t)w_freed * 128 * 8 / BITS : INT64_MAX;
        const int64_t ks = s_freed < s_done
                               ? (int64_t)(sc0 + s_freed) * SGC * (1 << a.gs_log2) - (int64_t)kt0 * kBK
                               : INT64_MAX;
        if (kw <= ks) {
          if (w_freed >= w_ready) {
            okr = mbar_wait(full_l(w_freed % WS), (w_freed / WS) & 1, abort_flag);
            w_ready = w_freed + 1;
          }
          __syncwarp();
          if (okr && lane == 0) mbar_arrive(empty_l(w_freed % WS));
          ++w_freed;
        } else {
          if (s_freed >= s_ready) {
            okr = mbar_wait(full_l(WS + s_freed % SS), (s_freed / SS) & 1, abort_flag);
            s_ready = s_freed + 1;
          }
          __syncwarp();
          if (okr && lane == 0) mbar_arrive(empty_l(WS + s_freed % SS));
          ++s_freed;
        }
      }
      return okr;
    };
    // scales straight from global memory: this group's next stage is loaded
    // one iteration ahead, so the load latency hides behind a stage
    uint32_t sraw[4] = {0u, 0u, 0u, 0u};
    if (FAST && a.scale_copy && grp < nkt)
      load_stage_scales<FP4>(sraw, a.scales, a.biases, row, G, kt0 + grp, a.gs_log2, a.K,
                             row_ok && row < a.N);
    for (int i = grp; i < nkt; i += kDqGroups) {
      const int kt = kt0 + i;
      const bool tail = (kt + 1) * kBK > a.K;
      Packed<BITS> pk;
      StageSB sb;
      if constexpr (FAST) {
        const int o0 = i * S::kPB;                         // row byte offset from wb0
        const int c_hi = (o0 + S::kPB - 1) >> 7;
        bool ok = true;
        for (; w_ready <= c_hi && ok; ++w_ready)
          ok = mbar_wait(full_l(w_ready % WS), (w_ready / WS) & 1, abort_flag);
        if (!a.scale_copy) {
          const int sj = (((kt * kBK) >> a.gs_log2) / SGC) - sc0;
          for (; s_ready <= sj && ok; ++s_ready)
            ok = mbar_wait(full_l(WS + s_ready % SS), (s_ready / SS) & 1, abort_flag);
        }
        if (!ok) break;
        if constexpr (S::kPB % 16 == 0) {
#pragma unroll
          for (int u = 0; u < S::kPB / 16; ++u) {
            const int o = o0 + 16 * u;
            const uint4 v = *reinterpret_cast<const uint4*>(
                wring + ((o >> 7) % WS) * S::kWChunk + wchunk_off(o & 127, r));
            pk.w[4 * u] = v.x; pk.w[4 * u + 1] = v.y; pk.w[4 * u + 2] = v.z; pk.w[4 * u + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int u = 0; u < S::kPB / 8; ++u) {
            const int o = o0 + 8 * u;
            const uint2 v = *reinterpret_cast<const uint2*>(
                wring + ((o >> 7) % WS) * S::kWChunk + wchunk_off(o & 127, r));
            pk.w[2 * u] = v.x; pk.w[2 * u + 1] = v.y;
          }
        }
        if (tail) {
#pragma unroll
          for (int w = BITS; w < 2 * BITS; ++w) pk.w[w] = 0u;
        }
        uint32_t raw[4];
        if (a.scale_copy) {
#pragma unroll
          for (int u = 0; u < 4; ++u) raw[u] = sraw[u];
          if (i + kDqGroups < nkt)
            load_stage_scales<FP4>(sraw, a.scales, a.biases, row, G, kt + kDqGroups, a.gs_log2, a.K,
                                   row_ok && row < a.N);
        } else {
          const uint8_t* sslot = sring + ((s_ready - 1) % SS) * S::kSChunk;
          const int g0 = (kt * kBK) >> a.gs_log2;
          const int g1 = tail ? g0 : ((kt * kBK + 32) >> a.gs_log2);
          if constexpr (FP4) {
            const uint8_t* sp = sslot + r * 16;
            if (fp4_g16) {
              raw[0] = sp[g0 % SGC]; raw[1] = sp[(g0 + 1) % SGC];
              raw[2] = sp[(g0 + 2) % SGC]; raw[3] = sp[(g0 + 3) % SGC];
            } else {
              raw[0] = sp[g0 % SGC]; raw[1] = sp[g1 % SGC]; raw[2] = raw[3] = 0u;
            }
          } else {
            const uint16_t* sp = reinterpret_cast<const uint16_t*>(sslot + r * 16);
            const uint16_t* bp = reinterpret_cast<const uint16_t*>(sslot + kRowsW * 16 + r * 16);
            raw[0] = sp[g0 % SGC]; raw[1] = sp[g1 % SGC];
            raw[2] = bp[g0 % SGC]; raw[3] = bp[g1 % SGC];
          }
        }
        if constexpr (FP4) {
          const int gs = 1 << a.gs_log2;
          auto sc = [&](uint32_t v) { return splat(TT<T>::from_f(fp4_scale_t<T>(v, gs))); };
          if (fp4_g16) {
            sb.s[0] = sc(raw[0]); sb.s[1] = sc(raw[1]);
            sb.b[0] = tail ? sb.s[0] : sc(raw[2]);
            sb.b[1] = tail ? sb.s[0] : sc(raw[3]);
          } else {
            sb.s[0] = sc(raw[0]); sb.s[1] = sc(raw[1]); sb.b[0] = sb.b[1] = 0u;
          }
        } else {
          sb.s[0] = raw[0] | (raw[0] << 16); sb.s[1] = raw[1] | (raw[1] << 16);
          sb.b[0] = raw[2] | (raw[2] << 16); sb.b[1] = raw[3] | (raw[3] << 16);
        }
        // release the chunks this group is done with: those that end before
        // its next stage starts (all of them after its last stage)
        const bool last = i + kDqGroups >= nkt;
        const int w_done = last ? nwc : (((i + kDqGroups) * S::kPB) >> 7);
        const int s_done = a.scale_copy ? 0
                           : last ? nsc : ((((kt + kDqGroups) * kBK) >> a.gs_log2) / SGC) - sc0;
        if (!release_upto(w_done, s_done)) break;
      } else {
        const int ps = i % PST;
        if (!mbar_wait(full_l(ps), (i / PST) & 1, abort_flag)) break;
        const uint8_t* slot = pring + ps * S::kPSlot;
        if (row_ok) {
          lds_packed<BITS>(pk, slot + r * S::kRP);
          if (tail) {
#pragma unroll
            for (int w = BITS; w < 2 * BITS; ++w) pk.w[w] = 0u;
          }
          const uint4 wv = *reinterpret_cast<const uint4*>(slot + kRowsW * S::kRP + r * 16);
          sb = sb_from_words<T, FP4>(wv, a, row, kt, G, tail);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_l(ps));
      }
      const int s = i % ST;
      if (!__all_sync(0xffffffffu, mbar_wait(empty(s), ((i / ST) & 1) ^ 1, abort_flag))) break;
      tc_fence_after();
      uint32_t o[32];
      if (row_ok) {
        dequant_row<T, BITS, FP4>(pk, sb, fp4_g16, tail, o);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = 0u;
      }
      tmem_st_32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + S::kACol0 + 32 * s, o);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(full(s));
    }
    if constexpr (FAST) {
      // Chunks past this group's last stage are released too.
      if (!*abort_flag) release_upto(nwc, nsc);
    }

    // ------------------------------------------------------- epilogue
    pdl_wait();                                           // before y is written
    const bool acc_ok = mbar_wait(acc_full, 0, abort_flag, 4000000000ull);
    tc_fence_after();
    const int q = warp & 3;                                 // TMEM lane quarter
    const int rr = q * 32 + lane;                           // tile row of this thread
    const int64_t orow = n0 + rr;
    const bool orow_ok = nl0 + rr < a.n_limit;
    float* red = reinterpret_cast<float*>(ring);            // [BT][128] when split
    if (acc_ok && !*abort_flag) {
#pragma unroll 1
      for (int c0 = 16 * grp; c0 < BT; c0 += 16 * kDqGroups) {
        uint32_t v[16];
        tmem_ld_16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, v);
        tmem_ld_wait();
        if (a.splits == 1 && a.y_vec) {
          // Through this warp's 1 KB of the (now idle) operand ring: the 16
          // columns x 32 rows go in as [column][row] T, and come out as
          // 16-byte runs of 8 rows, which are contiguous in y.
          T* stg = reinterpret_cast<T*>(ring) + (warp - kProducerWarp0) * 512;
#pragma unroll
          for (int j = 0; j < 16; ++j) stg[j * 32 + lane] = TT<T>::from_f(__uint_as_float(v[j]));
          __syncwarp();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int j = 8 * h + (lane >> 2), part = lane & 3;
            const int m = m0 + c0 + j;
            const int nl = nl0 + q * 32 + 8 * part;         // first of the 8 rows, within the group
            const uint4 val = *reinterpret_cast<const uint4*>(stg + j * 32 + 8 * part);
            // y_vec implies n_limit % 8 == 0: a run of 8 rows is whole or absent
            if (m < a.M && nl < a.n_limit)
              *reinterpret_cast<uint4*>(reinterpret_cast<T*>(a.y) + (int64_t)m * a.ldy +
                                        (n0 + q * 32 + 8 * part)) = val;
          }
          __syncwarp();
        } else if (a.splits == 1) {
          if (orow_ok) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int m = m0 + c0 + j;
              if (m < a.M)
                reinterpret_cast<T*>(a.y)[(int64_t)m * a.ldy + orow] = TT<T>::from_f(__uint_as_float(v[j]));
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) red[(c0 + j) * kRowsW + rr] = __uint_as_float(v[j]);
        }
      }
    }
  }

  // --------------------------------------------------------- split-K reduce
  if (a.splits > 1) {
    pdl_wait();
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (!*abort_flag) {
      // Rank `split` finishes a contiguous slice of the [BT][128] tile:
      // 16-byte loads of every rank's parked partials, added in rank order.
      const float4* red4 = reinterpret_cast<const float4*>(ring);
      constexpr int kE4 = BT * kRowsW / 4;
      const int per = (kE4 + a.splits - 1) / a.splits;
      const int f0 = split * per, f1 = min(kE4, f0 + per);
      for (int f = f0 + (int)threadIdx.x; f < f1; f += kThreads) {
        float4 acc = cluster.map_shared_rank(red4, 0)[f];
        for (int q = 1; q < a.splits; ++q) {
          const float4 v = cluster.map_shared_rank(red4, q)[f];
          acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        const int e = 4 * f;
        const int j = e / kRowsW, rr = e - j * kRowsW;     // 4 consecutive weight rows
        const int m = m0 + j;
        if (m >= a.M) continue;
        T* yrow = reinterpret_cast<T*>(a.y) + (int64_t)m * a.ldy + n0 + rr;
        const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
        if (a.y_vec && nl0 + rr + 4 <= a.n_limit) {
          const T o0 = TT<T>::from_f(vals[0]), o1 = TT<T>::from_f(vals[1]);
          const T o2 = TT<T>::from_f(vals[2]), o3 = TT<T>::from_f(vals[3]);
          uint2 pk;
          pk.x = (uint32_t)*reinterpret_cast<const uint16_t*>(&o0) |
                 ((uint32_t)*reinterpret_cast<const uint16_t*>(&o1) << 16);
          pk.y = (uint32_t)*reinterpret_cast<const uint16_t*>(&o2) |
                 ((uint32_t)*reinterpret_cast<const uint16_t*>(&o3) << 16);
          *reinterpret_cast<uint2*>(yrow) = pk;
        } else {
#pragma unroll
          for (int t = 0; t < 4; ++t)
            if (nl0 + rr + t < a.n_limit) yrow[t] = TT<T>::from_f(vals[t]);
        }
      }
    }
    cluster.sync();
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) atomicOr(&g_aq_device_error, 1u);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

// -------------------------------------------------------------------- host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  // Resolved once per process (a function-local static is initialised
  // exactly once even when several threads call at the same time).
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
  return fn;
}

// Encoded 2-D maps of the calling thread, keyed by every encode argument: a
// call that repeats a previous call's operands (the usual case for weights)
// copies the 128-byte map instead of encoding it again.  Direct-mapped, per
// thread, so no locking; a map only describes an address range and a shape,
// so an entry stays valid for as long as its arguments are passed again.
struct MapKey {
  const void* base;
  int64_t rows, cols;
  int type, esize, box_cols, box_rows, swz;
  bool operator==(const MapKey& o) const {
    return base == o.base && rows == o.rows && cols == o.cols && type == o.type &&
           esize == o.esize && box_cols == o.box_cols && box_rows == o.box_rows && swz == o.swz;
  }
};
struct MapEntry {
  MapKey key;
  bool used;
  CUtensorMap map;
};
constexpr int kMapCache = 256;

// 2-D tensor map over a row-major [rows, cols] array of 1- or 2-byte
// elements; zero fill out of bounds.
cudaError_t make_map(CUtensorMap* map, const void* base, CUtensorMapDataType type, int esize,
                     int64_t rows, int64_t cols, int box_cols, int box_rows,
                     CUtensorMapSwizzle swz) {
  thread_local MapEntry cache[kMapCache];
  const MapKey key{base, rows, cols, (int)type, esize, box_cols, box_rows, (int)swz};
  uint64_t h = (uint64_t)(uintptr_t)base * 0x9E3779B97F4A7C15ull;
  h ^= (uint64_t)(rows * 31 + cols) * 0xC2B2AE3D27D4EB4Full;
  h ^= (uint64_t)(((int)type * 8 + esize) * 1024 + box_cols * 4 + (int)swz) * 0x165667B19E3779F9ull;
  h ^= (uint64_t)box_rows << 17;
  MapEntry& slot = cache[(h >> 40) % kMapCache];
  if (slot.used && slot.key == key) {
    *map = slot.map;
    return cudaSuccess;
  }
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * esize)};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  slot.key = key;
  slot.map = *map;
  slot.used = true;
  return cudaSuccess;
}

// 4-D tensor map over an NHWC activation [Bn, H, W, C] of 2-byte elements,
// box {cbox channels, bw, bh, 1}: 16 channels with 32-byte swizzle or 64
// with 128-byte swizzle; zero fill out of bounds (which supplies the
// convolution's padding).
inline cudaError_t make_map_nhwc(CUtensorMap* map, const void* base, CUtensorMapDataType type,
                                 int Bn, int H, int W, int C, int bw, int bh, int cbox) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)Bn};
  cuuint64_t strides[3] = {(cuuint64_t)C * 2, (cuuint64_t)W * C * 2, (cuuint64_t)H * W * C * 2};
  cuuint32_t box[4] = {(cuuint32_t)cbox, (cuuint32_t)bw, (cuuint32_t)bh, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, type, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   cbox == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_32B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <typename T, int BITS, bool FP4, int BT, bool FAST, int XMODE>
cudaError_t launch_tc(const QmmPlan& p, const QmmMaps& maps, const QmmArgs& a, cudaStream_t st) {
  using S = QmmShape<BT, BITS, FAST>;
  auto kern = qmm_tc_kernel<T, BITS, FP4, BT, FAST, XMODE>;
  static std::atomic<bool> attr_done[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !attr_done[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_done[dev].store(true, std::memory_order_release);
  }
  // Part 0: tiles [0, tiles_main) with p.splits K-slices each; part 1 (the
  // partial last wave, when the plan splits it): the remaining tiles with
  // p.tail_splits slices each, so they spread over the idle SMs.
  const int64_t tiles = p.n_tiles * p.m_tiles;
  for (int part = 0; part < 2; ++part) {
    QmmArgs ap = a;
    ap.nt_all = (int)p.n_tiles;
    ap.y_vec = a.ldy % 8 == 0 && a.n_limit % 8 == 0 && ((uintptr_t)a.y & 15) == 0;
    int64_t count = tiles;
    if (part == 0) {
      count = p.tiles_main;
      ap.tile0 = 0;
    } else {
      count = tiles - p.tiles_main;
      if (count <= 0) break;
      ap.tile0 = (int)p.tiles_main;
      ap.splits = p.tail_splits;
      ap.k_tiles_split = p.tail_k_tiles_split;
    }
    if (count <= 0) continue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)count, 1, (unsigned)ap.splits);
    cfg.blockDim = dim3(S::kThreads, 1, 1);
    cfg.dynamicSmemBytes = S::kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = (unsigned)ap.splits;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, maps, ap);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename T, int BITS, bool FP4, bool FAST, int XMODE>
cudaError_t by_bt(const QmmPlan& p, const QmmMaps& maps, const QmmArgs& a, cudaStream_t st) {
  if constexpr (XMODE == 0) {
    switch (p.bt) {
      case 16: return launch_tc<T, BITS, FP4, 16, FAST, XMODE>(p, maps, a, st);
      case 32: return launch_tc<T, BITS, FP4, 32, FAST, XMODE>(p, maps, a, st);
      case 64: return launch_tc<T, BITS, FP4, 64, FAST, XMODE>(p, maps, a, st);
      case 128: return launch_tc<T, BITS, FP4, 128, FAST, XMODE>(p, maps, a, st);
      default: return launch_tc<T, BITS, FP4, 256, FAST, XMODE>(p, maps, a, st);
    }
  } else {
    switch (p.bt) {
      case 64: return launch_tc<T, BITS, FP4, 64, FAST, XMODE>(p, maps, a, st);
      case 128: return launch_tc<T, BITS, FP4, 128, FAST, XMODE>(p, maps, a, st);
      default: return launch_tc<T, BITS, FP4, 256, FAST, XMODE>(p, maps, a, st);
    }
  }
}

template <typename T, bool FAST, int XMODE>
cudaError_t by_bits_tc(const QmmPlan& p, const QmmMaps& maps, const QmmArgs& a, int bits,
                       int mode, cudaStream_t st) {
  if constexpr (XMODE == 0) {
    if (mode == AQ_MODE_FP4) return by_bt<T, 4, true, FAST, XMODE>(p, maps, a, st);
  }
  switch (bits) {
    case 2: return by_bt<T, 2, false, FAST, XMODE>(p, maps, a, st);
    case 3: return by_bt<T, 3, false, FAST, XMODE>(p, maps, a, st);
    case 4: return by_bt<T, 4, false, FAST, XMODE>(p, maps, a, st);
    case 5: return by_bt<T, 5, false, FAST, XMODE>(p, maps, a, st);
    case 6: return by_bt<T, 6, false, FAST, XMODE>(p, maps, a, st);
    case 8: return by_bt<T, 8, false, FAST, XMODE>(p, maps, a, st);
    default: return cudaErrorInvalidValue;
  }
}

// Prepare the weight-side tensor maps (TMA path) and the shared arguments;
// returns whether the TMA path applies.
inline cudaError_t weight_maps(QmmMaps& maps, QmmArgs& a, const void* w_q, const void* scales,
                               const void* biases, int64_t rows, int64_t K, int bits, int gs,
                               int mode, bool* fast) {
  a.row_bytes = K * bits / 8;
  // widest copy that every row start and stage offset (8*bits bytes) allows
  a.vec = (a.row_bytes % 16 == 0 && (8 * bits) % 16 == 0) ? 16
          : (a.row_bytes % 8 == 0 && (8 * bits) % 8 == 0) ? 8 : 4;
  const int64_t G = K / gs;
  const int esz = mode == AQ_MODE_FP4 ? 1 : 2;
  *fast = a.row_bytes % 16 == 0;
  if (!*fast) return cudaSuccess;
  // scale rows that TMA cannot address (stride or base not 16-byte aligned)
  // are copied by the loader warp instead
  a.scale_copy = !((G * esz) % 16 == 0 && ((uintptr_t)scales & 15) == 0 &&
                   (mode == AQ_MODE_FP4 || ((uintptr_t)biases & 15) == 0));
  cudaError_t e = make_map(&maps.w, w_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rows, a.row_bytes, 128,
                           kRowsW, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  if (a.scale_copy) return cudaSuccess;
  const CUtensorMapDataType st_t =
      mode == AQ_MODE_FP4 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
  e = make_map(&maps.s, scales, st_t, esz, rows, G, 16 / esz, kRowsW, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;
  if (mode != AQ_MODE_FP4)
    e = make_map(&maps.b, biases, st_t, esz, rows, G, 16 / esz, kRowsW, CU_TENSOR_MAP_SWIZZLE_NONE);
  return e;
}

// K-slice plan for p's tiles (n_tiles, m_tiles, k_tiles set) on `slots`
// resident CTAs.  Tiles that underfill the GPU split K over a cluster of up
// to 8; otherwise a last wave that is at most half full is launched apart,
// its tiles split in 2 or 4, so that it takes a fraction of a tile time on
// the SMs the full waves leave idle.  A K-slice starts on a 16-byte boundary
// of the packed rows (an even number of k-tiles for odd bit widths).
inline int slice_tiles(int64_t k_tiles, int splits, int bits) {
  int kts = (int)((k_tiles + splits - 1) / splits);
  if (bits & 1) kts += kts & 1;
  return kts;
}

inline void plan_splits(QmmPlan& p, int bits, int64_t slots) {
  const int64_t tiles = p.n_tiles * p.m_tiles;
  int splits = 1;
  while (splits < 8 && tiles * splits * 2 <= slots && p.k_tiles / (splits * 2) >= 2) splits *= 2;
  p.k_tiles_split = slice_tiles(p.k_tiles, splits, bits);
  p.splits = (p.k_tiles + p.k_tiles_split - 1) / p.k_tiles_split;
  p.tiles_main = tiles;
  p.tail_splits = 1;
  p.tail_k_tiles_split = p.k_tiles_split;
  if (p.splits != 1 || tiles <= slots) return;
  const int64_t rem = tiles % slots;
  int ts = 1;
  while (ts < 4 && rem > 0 && rem * ts * 2 <= slots && p.k_tiles / (ts * 2) >= 4) ts *= 2;
  if (ts == 1) return;
  const int kts = slice_tiles(p.k_tiles, ts, bits);
  ts = (p.k_tiles + kts - 1) / kts;
  if (ts < 2) return;
  p.tiles_main = tiles - rem;
  p.tail_splits = ts;
  p.tail_k_tiles_split = kts;
}

inline int ilog2i(int v) {
  int r = 0;
  while ((1 << (r + 1)) <= v) ++r;
  return r;
}

inline cudaError_t read_tu_error(unsigned* out) {
  return cudaMemcpyFromSymbol(out, g_aq_device_error, sizeof(unsigned));
}


}  // namespace
}  // namespace aq
