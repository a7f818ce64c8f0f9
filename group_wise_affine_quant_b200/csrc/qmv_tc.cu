// qmv_tc.cu — decode-sized quantized matmul (3 <= M <= 16 rows of x) on the
// tensor cores: y = x . dequant(W)^T with one 128 x 16 x K-slice tile per CTA.
//
// Prior art: affine_packed_qmv_fast in "Add the 3bit packed qmm_t" (a few
// rows per simdgroup, fp32 accumulation).  On B200 the fp32 pipe cannot keep
// up with the weight stream once M grows past two (one FMA per code per row
// of x), so this path dequantizes into shared memory and lets one 128 x 16
// tcgen05 MMA per 16 K-columns do the products.  The design is for latency:
//   * Every CTA owns 128 weight rows and one K-slice; the slices of a row
//     tile form a thread block cluster (split-K, up to 8).  About 90 KB of
//     shared memory, so two CTAs share an SM and the next kernel of a stream
//     can stream its weights while this one finishes.
//   * Warp 0 issues the packed weight chunks (128 rows x 128 bytes, 128-byte
//     swizzle) and the scale/bias chunks (128 rows x 16 bytes) by TMA in K
//     order, three weight chunks in flight; warp 2 loads the 16-row x tiles;
//     warp 1 owns TMEM and issues the MMAs.
//   * All eight dequantizer warps work on every 64-column stage: a thread
//     owns one weight row and one 32-column half, forms w_hat = s*q + b in T
//     with packed FMAs (the values aq_dequantize writes) and stores it in the
//     128-byte-swizzled K-major layout, so a stage is ready after one short
//     pass instead of one pass of a quarter of the threads.
//   * Split-K reduction without a cluster-wide barrier at the end: once its
//     own MMAs are done, the leader (rank 0) tells the other slices to send;
//     each pushes its fp32 partial (M columns of its 128 rows) into the
//     leader's shared memory with st.async, completing bytes on one leader
//     mbarrier, and leaves.  The leader adds the slices in rank order and
//     writes y.  No workspace, no global atomics.
//   * Every wait is bounded (2 s); a timeout sets a device error flag and the
//     CTA stops issuing work, frees its TMEM and exits.
#include "qmm_kernel.cuh"

namespace aq {
namespace {

struct DecShape {
  static constexpr int kDqWarps = 8;
  static constexpr int kWarpLoad = 0, kWarpMma = 1, kWarpX = 2, kWarpDq0 = 3;
  static constexpr int kThreads = 32 * (kWarpDq0 + kDqWarps);        // 352
  // A stage is 128 K-columns (two 64-column k-tiles).  Dequantized weight
  // stages live in TMEM: 64 columns each (two 16-bit values per lane and
  // column); the accumulator takes columns 0-15.
  static constexpr int kAStages = 3;
  static constexpr int kACol0 = 32;
  static constexpr int kTmemCols = 256;
  static constexpr int kWSlots = 4;                                  // 16 KB each
  static constexpr int kXStages = 4;                                 // 4 KB each
  static constexpr int kSSlots = 2;                                  // 4 KB each
  static constexpr int kWChunk = kRowsW * 128;
  static constexpr int kXAtom = 16 * kBK * 2;                        // 16 rows x 128 B
  static constexpr int kXBytes = 2 * kXAtom;
  static constexpr int kSChunk = kRowsW * 16 * 2;
  static constexpr int kWOff = 0;
  static constexpr int kXOff = kWOff + kWSlots * kWChunk;
  static constexpr int kSOff = kXOff + kXStages * kXBytes;
  // split-K: the partials this slice receives for the rows it owns, from
  // every other slice: (slices - 1) x ceil(128 / slices) rows x M fp32
  static constexpr int kRecvOff = kSOff + kSSlots * kSChunk;
  static constexpr int kRecvBytes = 8 * 1024;
  static constexpr int kDataBytes = kRecvOff + kRecvBytes;
  // full/empty pairs for the four rings, then acc_full, recv_full
  static constexpr int kBars = 2 * (kAStages + kWSlots + kXStages + kSSlots) + 2;
  static constexpr int kSmem = 1024 + kDataBytes + 512;
  static_assert(kBars * 8 + 16 <= 512, "barrier area");
  static_assert(kACol0 + 64 * kAStages <= kTmemCols, "TMEM columns");
};

struct DecArgs {
  void* y;
  int M, N, K;
  int gs_log2;
  int k_tiles;          // ceil(K / 64)
  int kts;              // k-tiles per slice (even)
  int splits;
  int mp;               // M rounded up to 4 (partial columns pushed per row)
  int weights_early;
  int x_early;           // read x before waiting on the previous kernel
};

// This thread's weight row for one k-tile (64 codes, 8 * BITS bytes at
// byte offset `off` of the slice) from the swizzled weight chunks.
template <int BITS, int WS>
__device__ __forceinline__ void load_row(Packed<BITS>& p, const uint8_t* wring, int off, int r) {
  constexpr int kB = 8 * BITS;
  constexpr int P = (kB % 16 == 0) ? 16 : 8;
#pragma unroll
  for (int u = 0; u < kB / P; ++u) {
    const int o = off + P * u;
    const uint8_t* src = wring + ((o >> 7) % WS) * (kRowsW * 128) + wchunk_off(o & 127, r);
    if constexpr (P == 16) {
      const uint4 v = *reinterpret_cast<const uint4*>(src);
      p.w[4 * u] = v.x; p.w[4 * u + 1] = v.y; p.w[4 * u + 2] = v.z; p.w[4 * u + 3] = v.w;
    } else {
      const uint2 v = *reinterpret_cast<const uint2*>(src);
      p.w[2 * u] = v.x; p.w[2 * u + 1] = v.y;
    }
  }
}


template <typename T, int BITS, bool FP4>
__global__ void __launch_bounds__(DecShape::kThreads, 2)
qmv_tc_kernel(const __grid_constant__ QmmMaps maps, const DecArgs a) {
  using S = DecShape;
  constexpr int AS = S::kAStages, WS = S::kWSlots, XS = S::kXStages, SS = S::kSSlots;
  constexpr int kPB = 8 * BITS;                           // packed bytes per row per k-tile
  constexpr int SGC = FP4 ? 16 : 8;                       // groups per scale chunk
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* wring = smem + S::kWOff;
  uint8_t* xring = smem + S::kXOff;
  uint8_t* sring = smem + S::kSOff;
  float* recv = reinterpret_cast<float*>(smem + S::kRecvOff);  // [splits-1][rows owned][mp]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kDataBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + S::kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  auto bar = [&](int i) { return smem_u32(bars + i); };
  auto full_a = [&](int s) { return bar(s); };
  auto empty_a = [&](int s) { return bar(AS + s); };
  auto full_w = [&](int s) { return bar(2 * AS + s); };
  auto empty_w = [&](int s) { return bar(2 * AS + WS + s); };
  auto full_x = [&](int s) { return bar(2 * (AS + WS) + s); };
  auto empty_x = [&](int s) { return bar(2 * (AS + WS) + XS + s); };
  auto full_s = [&](int s) { return bar(2 * (AS + WS + XS) + s); };
  auto empty_s = [&](int s) { return bar(2 * (AS + WS + XS) + SS + s); };
  const uint32_t acc_full = bar(2 * (AS + WS + XS + SS));
  const uint32_t recv_full = acc_full + 8;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kRowsW;
  const int split = blockIdx.z;
  const int kt0 = split * a.kts;                          // even (host plan)
  const int kt1 = min(a.k_tiles, kt0 + a.kts);
  const int nkt = kt1 - kt0;                              // >= 1 (host plan)
  const int nst = (nkt + 1) >> 1;                         // 128-column stages
  const bool clustered = a.splits > 1;
  // split-K: slice `split` owns rows [split * rpo, +rpo) of the tile and
  // receives those rows' partials from every other slice
  const int rpo = (kRowsW + a.splits - 1) / a.splits;
  const int own0 = min(kRowsW, split * rpo), own1 = min(kRowsW, own0 + rpo);
  // weight chunk c covers bytes [wb0 + 128 c, +128) of every row; scale chunk
  // j covers groups [SGC (sc0 + j), +SGC)
  const int wb0 = kt0 * kPB;                              // 16-byte aligned (host plan)
  const int nwc = (nkt * kPB + 127) >> 7;
  const int sc0 = ((kt0 * kBK) >> a.gs_log2) / SGC;
  const int nsc = ((((kt1 * kBK) - 1) >> a.gs_log2) / SGC) - sc0 + 1;

  // Weight and scale chunks in K order.  In the prologue (weights that no
  // earlier kernel writes) thread 0 issues what fits in the empty slots
  // before anything else; the loader warp continues from there.
  int lc = 0, lj = 0;
  auto load_chunks = [&](bool prologue) {
    while (lc < nwc || lj < nsc) {
      const int64_t kw = lc < nwc ? (int64_t)lc * 128 * 8 / BITS : INT64_MAX;
      const int64_t ks = lj < nsc ? (int64_t)(sc0 + lj) * SGC * (1 << a.gs_log2) - (int64_t)kt0 * kBK
                                  : INT64_MAX;
      if (kw <= ks) {
        const int slot = lc % WS;
        if (prologue ? lc >= WS : !mbar_wait(empty_w(slot), ((lc / WS) & 1) ^ 1, abort_flag)) return;
        mbar_arrive_expect_tx(full_w(slot), S::kWChunk);
        tma_load_2d_hint(smem_u32(wring + slot * S::kWChunk), &maps.w, full_w(slot), wb0 + 128 * lc, n0,
                         l2_policy_evict_first());
        ++lc;
      } else {
        const int slot = lj % SS;
        if (prologue ? lj >= SS : !mbar_wait(empty_s(slot), ((lj / SS) & 1) ^ 1, abort_flag)) return;
        const uint32_t dst = smem_u32(sring + slot * S::kSChunk);
        mbar_arrive_expect_tx(full_s(slot), FP4 ? kRowsW * 16 : 2 * kRowsW * 16);
        tma_load_2d_hint(dst, &maps.s, full_s(slot), (sc0 + lj) * SGC, n0, l2_policy_evict_first());
        if constexpr (!FP4)
          tma_load_2d_hint(dst + kRowsW * 16, &maps.b, full_s(slot), (sc0 + lj) * SGC, n0,
                           l2_policy_evict_first());
        ++lj;
      }
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < AS; ++s) { mbar_init(full_a(s), 4); mbar_init(empty_a(s), 1); }
    for (int s = 0; s < WS; ++s) { mbar_init(full_w(s), 1); mbar_init(empty_w(s), S::kDqWarps); }
    for (int s = 0; s < XS; ++s) { mbar_init(full_x(s), 1); mbar_init(empty_x(s), 1); }
    for (int s = 0; s < SS; ++s) { mbar_init(full_s(s), 1); mbar_init(empty_s(s), S::kDqWarps); }
    mbar_init(acc_full, 1);
    mbar_init(recv_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    // every other slice sends the owned rows' partials before this one adds
    if (clustered)
      mbar_arrive_expect_tx(recv_full, (uint32_t)((a.splits - 1) * (own1 - own0) * a.mp * 4));
    prefetch_tensormap(&maps.w);
    prefetch_tensormap(&maps.s);
    if constexpr (!FP4) prefetch_tensormap(&maps.b);
    if (a.weights_early) load_chunks(true);
  }
  if (warp == S::kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), S::kTmemCols);
    tc_fence_before();
  }
  if (warp == S::kWarpX && lane == 0) prefetch_tensormap(&maps.x);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (clustered) cluster_arrive();                        // barriers of every slice initialised
  pdl_launch_dependents();

  if (warp == S::kWarpLoad) {
    if (!a.weights_early) pdl_wait();
    if (lane == 0) load_chunks(false);
  } else if (warp == S::kWarpX) {
    // -------------------------------------------------------- x tiles by TMA
    if (!a.x_early) pdl_wait();                           // x may come from the previous kernel
    if (lane == 0) {
      for (int j = 0; j < nst; ++j) {
        const int s = j % XS;
        const bool two = 2 * j + 1 < nkt;
        if (!mbar_wait(empty_x(s), ((j / XS) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(full_x(s), two ? S::kXBytes : S::kXAtom);
        const uint32_t dst = smem_u32(xring + s * S::kXBytes);
        tma_load_2d_hint(dst, &maps.x, full_x(s), (kt0 + 2 * j) * kBK, 0, l2_policy_evict_last());
        if (two)
          tma_load_2d_hint(dst + S::kXAtom, &maps.x, full_x(s), (kt0 + 2 * j + 1) * kBK, 0,
                           l2_policy_evict_last());
      }
    }
  } else if (warp == S::kWarpMma) {
    // ------------------------------------------------------- MMA issuer
    // The whole warp runs the loop (warp-uniform waits and descriptors); an
    // elected lane, the same one every stage, issues the MMAs and commits.
    constexpr uint32_t idesc = idesc_f16(std::is_same<T, __nv_bfloat16>::value, kRowsW, 16);
    for (int j = 0; j < nst; ++j) {
      const int s = j % AS, sx = j % XS;
      if (!__all_sync(0xffffffffu, mbar_wait(full_a(s), (j / AS) & 1, abort_flag) &&
                                       mbar_wait(full_x(sx), (j / XS) & 1, abort_flag)))
        break;
      tc_fence_after();
      const uint32_t a_col = tmem + S::kACol0 + 64 * s;
      const uint32_t b_addr = smem_u32(xring + sx * S::kXBytes);
      const int halves = 2 * j + 1 < nkt ? 2 : 1;
      if (elect_one()) {
        for (int h = 0; h < halves; ++h) {
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            mma_f16_tmem_a(tmem, a_col + 32 * h + 8 * k,
                           sdesc_sw128(b_addr + h * S::kXAtom + k * 32), idesc,
                           (j > 0 || h > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(empty_a(s));
        mma_commit(empty_x(sx));
      }
      __syncwarp();
    }
    if (elect_one()) mma_commit(acc_full);                // also on abort: nothing left in flight
    __syncwarp();
  } else {
    // ------------------------------------------------------- dequantizers
    // Two groups of four warps take alternate stages; a thread owns one
    // weight row (its TMEM lane) and both k-tiles of the stage.
    const int gq = (warp - S::kWarpDq0) >> 2;            // dequantizer group
    const int q = warp & 3;                               // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;                          // weight row in the tile = TMEM lane
    const bool fp4_g16 = FP4 && a.gs_log2 == 4;
    int w_ready = 0, w_freed = 0, s_ready = 0, s_freed = 0;
    // Release weight chunks below w_done and scale chunks below s_done in
    // the loader's K order (weight chunk first on a tie), waiting for each
    // chunk's data first: every group releases every chunk, and the wait
    // keeps this group's arrivals on the slot's current phase.
    auto release_upto = [&](int w_done, int s_done) -> bool {
      bool okr = true;
      while (okr && (w_freed < w_done || s_freed < s_done)) {
        const int64_t kw = w_freed < w_done ? (int64_t)w_freed * 128 * 8 / BITS : INT64_MAX;
        const int64_t ks = s_freed < s_done
                               ? (int64_t)(sc0 + s_freed) * SGC * (1 << a.gs_log2) - (int64_t)kt0 * kBK
                               : INT64_MAX;
        if (kw <= ks) {
          if (w_freed >= w_ready) {
            okr = mbar_wait(full_w(w_freed % WS), (w_freed / WS) & 1, abort_flag);
            w_ready = w_freed + 1;
          }
          __syncwarp();
          if (okr && lane == 0) mbar_arrive(empty_w(w_freed % WS));
          ++w_freed;
        } else {
          if (s_freed >= s_ready) {
            okr = mbar_wait(full_s(s_freed % SS), (s_freed / SS) & 1, abort_flag);
            s_ready = s_freed + 1;
          }
          __syncwarp();
          if (okr && lane == 0) mbar_arrive(empty_s(s_freed % SS));
          ++s_freed;
        }
      }
      return okr;
    };
    bool ok = true;
    for (int j = gq; j < nst && ok; j += 2) {
      const int st_end = min(2 * j + 2, nkt) * kPB;       // stage bytes end (slice-relative)
      const int c_hi = (st_end - 1) >> 7;                 // last chunk the stage touches
      for (; w_ready <= c_hi && ok; ++w_ready)
        ok = mbar_wait(full_w(w_ready % WS), (w_ready / WS) & 1, abort_flag);
      const int sj = ((((kt0 + 2 * j) * kBK) >> a.gs_log2) / SGC) - sc0;
      for (; s_ready <= sj && ok; ++s_ready)
        ok = mbar_wait(full_s(s_ready % SS), (s_ready / SS) & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);                    // warp-uniform before the collectives
      if (!ok) break;
      const uint8_t* sslot = sring + ((s_ready - 1) % SS) * S::kSChunk;
      // chunks that end with this stage are released once read (a slot is
      // refilled only after all eight warps have released it)
      const bool last = j + 2 >= nst;
      const int w_done = last ? nwc : (((2 * j + 2) * kPB) >> 7);
      const int s_done = last ? nsc : (((((kt0 + 2 * j + 2) * kBK) >> a.gs_log2) / SGC) - sc0);
      const int s = j % AS;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(empty_a(s), ((j / AS) & 1) ^ 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int kt = kt0 + 2 * j + h;
        const bool tail = (kt + 1) * kBK > a.K;
        uint32_t o[32];
        if (2 * j + h < nkt) {
          Packed<BITS> pk;
          StageSB sb;
          load_row<BITS, WS>(pk, wring, (2 * j + h) * kPB, r);
          const int g0 = (kt * kBK) >> a.gs_log2;
          const int g1 = tail ? g0 : ((kt * kBK + 32) >> a.gs_log2);
          if constexpr (FP4) {
            const uint8_t* sp = sslot + r * 16;
            const int gs = 1 << a.gs_log2;
            auto sc = [&](int g) { return splat(TT<T>::from_f(fp4_scale_t<T>(sp[g % SGC], gs))); };
            if (fp4_g16) {
              sb.s[0] = sc(g0); sb.s[1] = sc(g0 + 1);
              sb.b[0] = tail ? sb.s[0] : sc(g0 + 2);
              sb.b[1] = tail ? sb.s[0] : sc(g0 + 3);
            } else {
              sb.s[0] = sc(g0); sb.s[1] = sc(g1); sb.b[0] = sb.b[1] = 0u;
            }
          } else {
            const uint16_t* sp = reinterpret_cast<const uint16_t*>(sslot + r * 16);
            const uint16_t* bp = reinterpret_cast<const uint16_t*>(sslot + kRowsW * 16 + r * 16);
            const uint32_t s0 = sp[g0 % SGC], s1 = sp[g1 % SGC];
            const uint32_t b0 = bp[g0 % SGC], b1 = bp[g1 % SGC];
            sb.s[0] = s0 | (s0 << 16); sb.s[1] = s1 | (s1 << 16);
            sb.b[0] = b0 | (b0 << 16); sb.b[1] = b1 | (b1 << 16);
          }
          dequant_row<T, BITS, FP4>(pk, sb, fp4_g16, tail, o);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0u;
        }
        tmem_st_32(tmem + ((uint32_t)(q * 32) << 16) + S::kACol0 + 64 * s + 32 * h, o);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(full_a(s));
      // after the hand-over: a release may wait for chunks that the other
      // group's next stage frees, which needs this stage's MMAs to run
      ok = release_upto(w_done, s_done);
    }
    // chunks past this group's last stage are released too
    if (!*abort_flag) release_upto(nwc, nsc);

    // ------------------------------------------------------- epilogue
    if (gq == 0) {
      const bool acc_ok = mbar_wait(acc_full, 0, abort_flag, 4000000000ull);
      tc_fence_after();
      uint32_t v[16];
      tmem_ld_16(tmem + ((uint32_t)(q * 32) << 16), v);
      tmem_ld_wait();
      // the accumulator is in registers: the MMA warp may free TMEM now
      tc_fence_before();
      named_barrier_arrive(1, 32 * 5);
      const bool live = acc_ok && !*abort_flag;
      const int owner = clustered ? r / rpo : split;
      if (clustered) cluster_wait();                      // every slice's barriers are initialised
      if (live && owner != split) {
        // send this row's partial to the slice that owns it
        const int slot = split < owner ? split : split - 1;
        const uint32_t dst = smem_u32(recv + (slot * rpo + (r - owner * rpo)) * a.mp);
        const uint32_t rdst = mapa_shared(dst, (uint32_t)owner);
        const uint32_t rbar = mapa_shared(recv_full, (uint32_t)owner);
#pragma unroll
        for (int t = 0; t < 16; t += 4)
          if (t < a.mp) st_async_v4(rdst + 4 * t, v[t], v[t + 1], v[t + 2], v[t + 3], rbar);
      }
      // every lane of the warp has sent before any lane waits: a waiting
      // lane must not hold back a sibling whose partial another slice awaits
      __syncwarp();
      if (live && owner == split) {
        // an owned row: add every slice's partial in slice order
        float acc[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) acc[t] = 0.f;
        bool have = true;
        if (clustered) have = mbar_wait_cluster(recv_full, 0, abort_flag, 4000000000ull);
        if (have) {
          // all partials of this row first (independent loads), then the
          // sum in slice order with this slice's own partial at its place
#pragma unroll
          for (int t = 0; t < 16; t += 4) {
            if (t < a.mp) {
              float4 p[7];
#pragma unroll
              for (int k = 0; k < 7; ++k)
                p[k] = k < a.splits - 1
                           ? *reinterpret_cast<const float4*>(recv + (k * rpo + (r - own0)) * a.mp + t)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
              // slices 0 .. split-1 (receive slots 0 .. split-1), this slice,
              // then slices split+1 .. (receive slots split ..)
              auto add = [&](float4 q4) {
                acc[t] += q4.x; acc[t + 1] += q4.y; acc[t + 2] += q4.z; acc[t + 3] += q4.w;
              };
#pragma unroll
              for (int k = 0; k < 7; ++k)
                if (k < split) add(p[k]);
              add(make_float4(__uint_as_float(v[t]), __uint_as_float(v[t + 1]),
                              __uint_as_float(v[t + 2]), __uint_as_float(v[t + 3])));
#pragma unroll
              for (int k = 0; k < 7; ++k)
                if (k >= split && k < a.splits - 1) add(p[k]);
            }
          }
          pdl_wait();                                     // before y is written
          if (n0 + r < a.N) {
            T* yp = reinterpret_cast<T*>(a.y) + n0 + r;
#pragma unroll
            for (int t = 0; t < 16; ++t)
              if (t < a.M) yp[(int64_t)t * a.N] = TT<T>::from_f(acc[t]);
          }
        }
      }
    }
  }

  if (warp == S::kWarpMma) {
    // every tcgen05 operation has completed (acc_full) and the epilogue warps
    // have read the accumulator
    named_barrier_sync(1, 32 * 5);
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
  __syncwarp();
  if (lane == 0 && *abort_flag) atomicOr(&g_aq_device_error, 1u);
}

template <typename T, int BITS, bool FP4>
cudaError_t launch_dec(const QmmMaps& maps, const DecArgs& a, int64_t n_tiles, cudaStream_t st) {
  auto kern = qmv_tc_kernel<T, BITS, FP4>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !attr_done[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DecShape::kSmem);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_done[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)n_tiles, 1, (unsigned)a.splits);
  cfg.blockDim = dim3(DecShape::kThreads, 1, 1);
  cfg.dynamicSmemBytes = DecShape::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = (unsigned)a.splits;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, maps, a);
}

template <typename T>
cudaError_t dec_by_bits(const QmmMaps& maps, const DecArgs& a, int64_t n_tiles, int bits, int mode,
                        cudaStream_t st) {
  if (mode == AQ_MODE_FP4) return launch_dec<T, 4, true>(maps, a, n_tiles, st);
  switch (bits) {
    case 2: return launch_dec<T, 2, false>(maps, a, n_tiles, st);
    case 3: return launch_dec<T, 3, false>(maps, a, n_tiles, st);
    case 4: return launch_dec<T, 4, false>(maps, a, n_tiles, st);
    case 5: return launch_dec<T, 5, false>(maps, a, n_tiles, st);
    case 6: return launch_dec<T, 6, false>(maps, a, n_tiles, st);
    case 8: return launch_dec<T, 8, false>(maps, a, n_tiles, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

// Host plan: split K so that the tiles fill two CTAs per SM, up to 8 slices
// of at least one 64-column stage; odd widths keep slices at an even number
// of stages so that every slice starts on a 16-byte boundary of the rows.
bool qmv_tc_applies(int64_t M, int64_t N, int64_t K, int bits, int gs, int mode,
                    const void* scales, const void* biases) {
  if (M < 1 || M > 16 || N < 1 || K < 1) return false;
  const int64_t row_bytes = K * bits / 8;
  const int esz = mode == AQ_MODE_FP4 ? 1 : 2;
  return row_bytes % 16 == 0 && ((K / gs) * esz) % 16 == 0 && ((uintptr_t)scales & 15) == 0 &&
         (mode == AQ_MODE_FP4 || ((uintptr_t)biases & 15) == 0);
}

cudaError_t launch_qmv_tc(const void* x, const void* w_q, const void* scales, const void* biases,
                          void* y, int64_t M, int64_t N, int64_t K, int bits, int gs, int mode,
                          int dtype, cudaStream_t st) {
  const int64_t n_tiles = (N + kRowsW - 1) / kRowsW;
  const int k_tiles = (int)((K + kBK - 1) / kBK);
  const int64_t slots = 2 * 148;
  int splits = 1;
  while (splits < 8 && n_tiles * splits * 2 <= slots && k_tiles >= splits * 2) splits *= 2;
  int kts = (k_tiles + splits - 1) / splits;
  kts += kts & 1;                                         // slices start on a 128-column stage
  splits = (k_tiles + kts - 1) / kts;
  DecArgs a;
  memset(&a, 0, sizeof(a));
  a.y = y;
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.gs_log2 = ilog2i(gs);
  a.k_tiles = k_tiles;
  a.kts = kts;
  a.splits = splits;
  a.mp = (int)((M + 3) / 4 * 4);
  a.weights_early = weight_prefetch_enabled();
  a.x_early = input_prefetch_enabled();
  QmmMaps maps;
  memset(&maps, 0, sizeof(maps));
  const CUtensorMapDataType tt =
      dtype == AQ_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cudaError_t e = make_map(&maps.x, x, tt, 2, M, K, kBK, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  QmmArgs wa;
  memset(&wa, 0, sizeof(wa));
  bool fast = false;
  e = weight_maps(maps, wa, w_q, scales, biases, N, K, bits, gs, mode, &fast);
  if (e != cudaSuccess) return e;
  if (!fast || wa.scale_copy) return cudaErrorInvalidValue;   // qmv_tc_applies excludes both
  return dtype == AQ_F16 ? dec_by_bits<__half>(maps, a, n_tiles, bits, mode, st)
                         : dec_by_bits<__nv_bfloat16>(maps, a, n_tiles, bits, mode, st);
}

cudaError_t read_device_error_qmv_tc(unsigned* out) { return read_tu_error(out); }

}  // namespace aq
