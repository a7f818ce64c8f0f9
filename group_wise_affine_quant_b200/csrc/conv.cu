// conv.cu — quantized NHWC conv2d as an implicit GEMM on the tcgen05 kernel
// of qmm_kernel.cuh ("[Feature] Quantized Convolution 2D - Possible PR?":
// quantize_weights pads each output channel's flattened (kh, kw, Cin/groups)
// filter to a multiple of group_size and quantizes it; img2col stacks the
// (kh, kw, C) patches and quantized_matmul multiplies).  Here no im2col is
// materialised: the B operand tile of BT output pixels x 64 K-columns is
// read straight from x.
//   * Stride-1 convolutions whose pixel tiles are rectangles (whole output
//     rows, or row segments) load each 16-channel atom column of a K-stage
//     as one 4-D TMA box at the filter tap's (w, h) offset; out-of-bounds
//     coordinates read zeros, which are the image padding, and K-columns past
//     kh*kw*Cg read a box past the image (zeros).
//   * When, besides, Cg is a multiple of 64, every 64-column K-stage is 64
//     channels of a single tap, and the stage is one 64-channel box with the
//     128-byte swizzle of the dense path (fewer, wider TMA requests).
//   * Other shapes gather 16-byte granules (8 channels) with cp.async,
//     zero-filling the padding.
// Output channel block g of the conv group g is weight rows [g*Ng, (g+1)*Ng)
// and output columns of y [Bn*Ho*Wo, Cout].
#include "qmm_kernel.cuh"

namespace aq {

cudaError_t launch_qconv(const void* x, const void* w_q, const void* scales, const void* biases,
                         void* y, int Bn, int H, int W, int Cin, int Cout, int kh, int kw,
                         int sh, int sw, int ph, int pw, int groups, int bits, int gs, int dtype,
                         cudaStream_t st) {
  const int Cg = Cin / groups, Ng = Cout / groups;
  const int Ho = (H + 2 * ph - kh) / sh + 1, Wo = (W + 2 * pw - kw) / sw + 1;
  const int k_real = kh * kw * Cg;
  const int Kp = (k_real + gs - 1) / gs * gs;
  const int64_t M = (int64_t)Bn * Ho * Wo;
  const int64_t k_tiles = (Kp + kBK - 1) / kBK;
  const int ntg = (Ng + kRowsW - 1) / kRowsW;
  const int sms = 148;

  // A pixel tile of bt output pixels is a rectangle of the output image when
  // it is a segment of one output row or a run of whole rows of one image.
  auto rect = [&](int bt) {
    return (bt <= Wo) ? (Wo % bt == 0) : (bt % Wo == 0 && ((int64_t)Ho * Wo) % bt == 0 && bt / Wo <= 256);
  };
  const bool tma_ok = sh == 1 && sw == 1 && Cg % 16 == 0 && Cin % 8 == 0;
  // The widest pixel tile: a K-stage's dequantization cost is the same at
  // every tile width and feeds twice the MMA work at 256 pixels as at 128, so
  // a single wave of wide tiles beats more waves (or K-split tiles) of
  // narrow ones.  Narrower only when the whole image batch fits one.
  int bt = 256;
  while (bt > 64 && M <= bt / 2) bt /= 2;
  int xmode = 2;
  if (tma_ok) {
    for (int cand = bt; cand >= 64; cand /= 2)
      if (rect(cand)) { bt = cand; xmode = 1; break; }
  }
  // Every 64-column K-stage is 64 channels of one tap when Cg % 64 == 0: one
  // 64-channel box per stage (weights on the TMA path, rows 16-byte multiples)
  const bool w_rows16 = ((int64_t)Kp * bits / 8) % 16 == 0;
  if (xmode == 1 && Cg % 64 == 0 && w_rows16) xmode = 3;
  QmmPlan p{};
  p.bt = bt;
  p.n_tiles = (int64_t)ntg * groups;
  p.m_tiles = (M + bt - 1) / bt;
  p.k_tiles = (int)k_tiles;
  plan_splits(p, bits, sms);

  QmmMaps maps;
  memset(&maps, 0, sizeof(maps));
  const CUtensorMapDataType tt =
      dtype == AQ_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cudaError_t e = cudaSuccess;
  if (xmode == 1 || xmode == 3) {
    const int bw = bt <= Wo ? bt : Wo;
    e = make_map_nhwc(&maps.x, x, tt, Bn, H, W, Cin, bw, bt / bw, xmode == 3 ? 64 : 16);
    if (e != cudaSuccess) return e;
  }
  QmmArgs a;
  memset(&a, 0, sizeof(a));
  a.wq = (const uint8_t*)w_q;
  a.scales = scales;
  a.biases = biases;
  a.y = y;
  a.x = x;
  a.M = (int)M;
  a.N = Cout;
  a.K = Kp;
  a.gs_log2 = ilog2i(gs);
  a.weights_early = weight_prefetch_enabled();
  a.x_early = input_prefetch_enabled();
  a.k_tiles = p.k_tiles;
  a.k_tiles_split = p.k_tiles_split;
  a.splits = p.splits;
  a.ldy = Cout;
  a.n_limit = Ng;
  a.ntg = ntg;
  a.Cin = Cin; a.Cg = Cg; a.H = H; a.W = W; a.Ho = Ho; a.Wo = Wo;
  a.kh = kh; a.kw = kw; a.sh = sh; a.sw = sw; a.ph = ph; a.pw = pw; a.k_real = k_real;
  bool fast = false;
  e = weight_maps(maps, a, w_q, scales, biases, Cout, Kp, bits, gs, AQ_MODE_AFFINE, &fast);
  if (e != cudaSuccess) return e;
  const bool f16 = dtype == AQ_F16;
  if (xmode == 3 && fast)
    return f16 ? by_bits_tc<__half, true, 3>(p, maps, a, bits, 0, st)
               : by_bits_tc<__nv_bfloat16, true, 3>(p, maps, a, bits, 0, st);
  if (xmode == 1 || xmode == 3) {
    if (fast) return f16 ? by_bits_tc<__half, true, 1>(p, maps, a, bits, 0, st)
                         : by_bits_tc<__nv_bfloat16, true, 1>(p, maps, a, bits, 0, st);
    return f16 ? by_bits_tc<__half, false, 1>(p, maps, a, bits, 0, st)
               : by_bits_tc<__nv_bfloat16, false, 1>(p, maps, a, bits, 0, st);
  }
  if (fast) return f16 ? by_bits_tc<__half, true, 2>(p, maps, a, bits, 0, st)
                       : by_bits_tc<__nv_bfloat16, true, 2>(p, maps, a, bits, 0, st);
  return f16 ? by_bits_tc<__half, false, 2>(p, maps, a, bits, 0, st)
             : by_bits_tc<__nv_bfloat16, false, 2>(p, maps, a, bits, 0, st);
}

cudaError_t read_device_error_conv(unsigned* out) { return read_tu_error(out); }

}  // namespace aq
