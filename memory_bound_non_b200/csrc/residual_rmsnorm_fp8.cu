// Op (a): residual add + RMSNorm + FP8 e4m3 quantisation, one pass per row.
//
// "FlashRT kernel fusion", §二 steps 1/7 and §2.1: the residual add, the RMS
// reduction and the quantisation all read the same row, so the row is read
// from HBM once, kept in registers across the reduction, and written once
// (new residual + FP8 codes).  §三: the `_noweight` variant drops the weight
// multiply because (1 + w) already lives in the next GEMM's weights.
//
// Mapping (B200): one small CTA per row (128 threads for D <= 16384, so up to
// 16 rows are in flight per SM); the row is split into 16-byte chunks of 8
// elements and thread t owns chunks t, t+T, t+2T, ... (K of them), so every
// warp-wide load or store is one contiguous, fully used 512-byte run.  The sum
// of squares is reduced warp-shuffle -> shared memory -> every thread, in a
// fixed order (bitwise deterministic), in fp64 so the normalised values come
// out correctly rounded in fp32.  For block-128 scales a 128-column block
// is 16 chunks owned by 16 consecutive lanes (a half-warp), so its amax comes
// from two warp-wide f32 reduxes; no shared memory and no second pass.  With
// a static scale, rstd / s is folded into the product, so no per-element
// division remains.
#include <cmath>

#include "frt_device.cuh"
#include "frt_host.h"

namespace frt {
namespace {

// Threads per CTA: at most 128 for K = 2, 512 for K >= 4 (128 at D = 4096)
// and for K = 1 (one chunk per thread: the small-batch shape, up to D =
// 4096).  Small CTAs keep many rows in flight per SM, which is what hides
// each row's load -> reduce -> quantise latency on large batches.
template <int K>
constexpr int max_threads() {
  return K == 2 ? 128 : 512;
}

// LN (NEXT-4, the ViT "add_layer_norm" producer): LayerNorm instead of
// RMSNorm, y = (h - mean) * rstd * w + b (bias may be null).  One pass over
// the register-held row sums h and h^2 in fp64 (every square of a 16-bit
// value is exact in fp64, and so are the sums short of an extreme exponent
// spread); var = E[h^2] - mean^2 in fp64 then loses at most a few fp64 ulps of
// the mean^2 / var ratio, far below the fp32 the output carries.  Per element
// h - mean is formed against the mean split into two floats (error ~1 ulp of
// the difference, so a large common offset costs no accuracy) on packed fp32
// pairs, and y carries a few fp32 roundings (FP8 codes are 2^-4 apart); with
// a static scale 1 / s is folded into rstd and the bias, as the RMS path
// folds it into rstd.
template <int DT, int K, bool WEIGHTED, int QM, bool LN>
__global__ void __launch_bounds__(max_threads<K>()) residual_rmsnorm_fp8_kernel(
    const uint4* __restrict__ x, const uint4* r_in, uint4* r_out, const uint4* __restrict__ w,
    const uint4* __restrict__ bias, uint2* __restrict__ q, const float* __restrict__ static_scale,
    float* __restrict__ block_scales, int C, int NB, float D, float eps) {
  using P16 = Pack16<DT>;
  const int t = threadIdx.x;
  const int T = blockDim.x;
  const int64_t row = blockIdx.x;
  const int64_t base = row * (int64_t)C;
  __shared__ double red[32];

  // Constant inputs first, before the wait for the previous kernel: the
  // scale (and 1 / s in fp64) and, on narrow rows (small-batch,
  // latency-bound calls), the weight, so neither is on the critical path.
  // Wide rows load the weight after the reduction and keep the registers
  // for occupancy.
  const int64_t n_rc = (int64_t)gridDim.x * C;  // 16-byte chunks of x, r_in, r_out (and 8-byte ones of q)
  float s_static = 0.0f;
  if ((QM == FRT_QUANT_STATIC || QM >= kQuantNvfp4Rows) && FRT_IDX_OK(0, 1)) s_static = __ldg(static_scale);
  const double inv_s64 = QM == FRT_QUANT_STATIC ? 1.0 / (double)s_static : 0.0;
  constexpr bool kEarlyWeight = WEIGHTED && K <= 2;
  uint4 wv_early[kEarlyWeight ? K : 1];
  if (kEarlyWeight) {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if (t + k * T < C && FRT_IDX_OK(t + k * T, C)) wv_early[k] = __ldg(w + t + k * T);
  }
  pdl_enter();

  // Issue every load of the row before any store (r_out may alias r_in).
  uint4 xv[K], rv[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = t + k * T;
    if (c < C && FRT_IDX_OK(base + c, n_rc)) {
      xv[k] = ld_stream(x + base + c);
      rv[k] = ld_plain(r_in + base + c);
    }
  }

  // Pass 1: h = x + r rounded once to 16 bits (the correctly rounded exact
  // sum), kept packed; fp64 sum of squares (squares of 16-bit values are
  // exact, so the sum is exact to ~2^-40), one accumulator per chunk.
  uint4 hv[K];
  double ss[K], sm[LN ? K : 1];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    ss[k] = 0.0;
    if (LN) sm[LN ? k : 0] = 0.0;
    const int c = t + k * T;
    if (c < C) {
      const uint32_t* xw = reinterpret_cast<const uint32_t*>(&xv[k]);
      const uint32_t* rw = reinterpret_cast<const uint32_t*>(&rv[k]);
      uint32_t* hw = reinterpret_cast<uint32_t*>(&hv[k]);
      // h = 1 * x + r by the packed 16-bit FMA: the exact sum rounded once,
      // half an instruction per element.
#pragma unroll
      for (int e = 0; e < 4; ++e) hw[e] = P16::fma2(P16::kOnes, xw[e], rw[e]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 hf = P16::to_float2(hw[e]);
        const double h0 = (double)hf.x, h1 = (double)hf.y;
        ss[k] = fma(h0, h0, ss[k]);
        ss[k] = fma(h1, h1, ss[k]);
        if (LN) sm[LN ? k : 0] += h0 + h1;  // exact: two 16-bit values
      }
      if (FRT_IDX_OK(base + c, n_rc)) r_out[base + c] = hv[k];
    } else {
      hv[k] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  double sst = ss[0], smt = LN ? sm[0] : 0.0;
#pragma unroll
  for (int k = 1; k < K; ++k) {
    sst += ss[k];
    if (LN) smt += sm[LN ? k : 0];
  }

  // Row total: warp butterfly, then every thread adds the warp partials in
  // the same order and forms rstd in fp64.  y = h * w * rstd is rounded once
  // to fp32 (h * w is exact for 16-bit operands), so y is the correctly
  // rounded fp32 value of the exact normalised element and the FP8 codes are
  // decided on the value an exact computation would give.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sst += __shfl_xor_sync(0xFFFFFFFFu, sst, o);
    if (LN) smt += __shfl_xor_sync(0xFFFFFFFFu, smt, o);
  }
  if ((t & 31) == 0) {
    red[t >> 5] = sst;
    if (LN) red[16 + (t >> 5)] = smt;
  }
  __syncthreads();
  double tot = 0.0, tsum = 0.0;
  const int nw = T >> 5;
  for (int i = 0; i < nw; ++i) {
    tot += red[i];
    if (LN) tsum += red[16 + i];
  }
  float mean_hi = 0.0f, mean_lo = 0.0f;
  double var = tot / (double)D;  // RMSNorm: the mean square
  if (LN) {
    const double mean = tsum / (double)D;
    var = fmax(var - mean * mean, 0.0);
    mean_hi = (float)mean;
    mean_lo = (float)(mean - (double)mean_hi);
  }
  const double rstd64 = rsqrt_f64(var + (double)eps);
  // Static FP8 on the RMS path: y / s as one product with rstd / s (fp64,
  // held as an fp32 pair), so each code is decided on one fp32 rounding of
  // h w rstd / s rather than on RN(RN(h w rstd) / s).  A ratio outside
  // [2^-100, 2^100] keeps y and the division.
  const double rs64 = rstd64 * inv_s64;
  const bool fold = QM == FRT_QUANT_STATIC && rs64 >= 0x1p-100 && rs64 <= 0x1p+100;
  const Split32 rstd(fold ? rs64 : rstd64);
  // LayerNorm: rstd (/ s when folded) and the bias factor (1 / s when folded)
  const float2 rstd2 = make_float2((float)(fold ? rs64 : rstd64), (float)(fold ? rs64 : rstd64));
  const float2 bfac2 = make_float2(fold ? (float)inv_s64 : 1.0f, fold ? (float)inv_s64 : 1.0f);
  const float2 nmhi2 = make_float2(-mean_hi, -mean_hi), nmlo2 = make_float2(-mean_lo, -mean_lo);
  const Divisor dv_static(QM == FRT_QUANT_STATIC ? s_static : 1.0f);
  const float rden = QM >= kQuantNvfp4Rows ? __frcp_rn(6.0f * s_static) : 0.0f;  // NVFP4: RN(1 / RN(6 gs))

  // Pass 2: y and its FP8 codes.
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = t + k * T;
    const bool valid = c < C;
    const uint32_t* hw = reinterpret_cast<const uint32_t*>(&hv[k]);
    float y[8];
    if (LN) {
      uint4 wv = make_uint4(0u, 0u, 0u, 0u), bv = make_uint4(0u, 0u, 0u, 0u);
      if (valid) {
        if (WEIGHTED && FRT_IDX_OK(c, C)) wv = kEarlyWeight ? wv_early[kEarlyWeight ? k : 0] : __ldg(w + c);
        if (bias != nullptr && FRT_IDX_OK(c, C)) bv = __ldg(bias + c);
      }
      const uint32_t* ww = reinterpret_cast<const uint32_t*>(&wv);
      const uint32_t* bw = reinterpret_cast<const uint32_t*>(&bv);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 hf = P16::to_float2(hw[e]);
        const float2 wf = WEIGHTED ? P16::to_float2(ww[e]) : make_float2(1.0f, 1.0f);
        // (h - mean) rstd w + b, on packed pairs; bias zeros when absent
        const float2 d = __fmul2_rn(__fadd2_rn(__fadd2_rn(hf, nmhi2), nmlo2), rstd2);
        const float2 yy = __ffma2_rn(d, wf, __fmul2_rn(P16::to_float2(bw[e]), bfac2));
        // lanes past the row end hold 0 (they take part in the block amax)
        y[2 * e] = valid ? yy.x : 0.0f;
        y[2 * e + 1] = valid ? yy.y : 0.0f;
      }
    } else if (WEIGHTED && valid) {
      const uint4 wv = kEarlyWeight ? wv_early[kEarlyWeight ? k : 0] : FRT_IDX_OK(c, C) ? __ldg(w + c)
                                                                                        : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t* ww = reinterpret_cast<const uint32_t*>(&wv);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 hf = P16::to_float2(hw[e]);
        const float2 wf = P16::to_float2(ww[e]);
        y[2 * e] = rstd.mul(hf.x * wf.x);
        y[2 * e + 1] = rstd.mul(hf.y * wf.y);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 hf = P16::to_float2(hw[e]);
        y[2 * e] = rstd.mul(hf.x);
        y[2 * e + 1] = rstd.mul(hf.y);
      }
    }
    if (QM == FRT_QUANT_BLOCK128) {
      float am = fmaxf(absmax4(y[0], y[1], y[2], y[3]), absmax4(y[4], y[5], y[6], y[7]));
      am = half_warp_max_abs(am);  // 16 lanes = the 16 chunks of one 128-column block
      const float sb = block_scale_448(am);
      if (valid && (t & 15) == 0 && FRT_IDX_OK(row * NB + (c >> 4), (int64_t)gridDim.x * NB))
        block_scales[row * NB + (c >> 4)] = sb;
      if (valid && FRT_IDX_OK(base + c, n_rc)) q[base + c] = quant8(y, Divisor(sb));
    } else if (QM >= kQuantNvfp4Rows) {
      // NVFP4: a 16-element block is chunks 2b and 2b+1, held by lanes t and
      // t ^ 1; codes leave as one 32-bit word per chunk, the scale factor from
      // the even lane.  q / block_scales carry the code and sf pointers.
      float am = fmaxf(absmax4(y[0], y[1], y[2], y[3]), absmax4(y[4], y[5], y[6], y[7]));
      am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
      float reff;
      const uint32_t sf = nvfp4_scale(am, rden, s_static, &reff);
      if (valid) {
        if (FRT_IDX_OK(base + c, n_rc)) reinterpret_cast<uint32_t*>(q)[base + c] = nvfp4_codes<8>(y, reff);
        if ((c & 1) == 0) {
          uint8_t* sfo = reinterpret_cast<uint8_t*>(block_scales);
          const int nsf = C >> 1;
          const int64_t o = QM == kQuantNvfp4Rows ? row * nsf + (c >> 1) : sf_offset_swizzled(row, c >> 1, nsf);
          // row-major [M, nsf]; swizzled: 128-row x 4-column atoms
          const int64_t n_sf = QM == kQuantNvfp4Rows ? (int64_t)gridDim.x * nsf
                                                     : (((int64_t)gridDim.x + 127) / 128) * 128 * ((nsf + 3) / 4) * 4;
          if (FRT_IDX_OK(o, n_sf)) sfo[o] = (uint8_t)sf;
        }
      }
    } else if (valid && FRT_IDX_OK(base + c, n_rc)) {
      q[base + c] = fold ? e4m3x8(y) : quant8(y, dv_static);
    }
  }
}

// Row-norm launch arguments (bias only with LN).
struct NormArgs {
  const void *x, *r_in;
  void* r_out;
  const void *w, *bias;
  uint8_t* q;
  const float* ss;
  float* bs;
  int M, C, NB, T;
  float eps;
};

template <int DT, int K, bool W, int QM, bool LN>
frt_status launch_k(const NormArgs& a, cudaStream_t st) {
  auto kern = residual_rmsnorm_fp8_kernel<DT, K, W, QM, LN>;
  return launch(kern, dim3(a.M), dim3(a.T), 0, st, static_cast<const uint4*>(a.x), static_cast<const uint4*>(a.r_in),
                static_cast<uint4*>(a.r_out), static_cast<const uint4*>(a.w), static_cast<const uint4*>(a.bias),
                reinterpret_cast<uint2*>(a.q), a.ss, a.bs, a.C, a.NB, (float)(a.C * 8), a.eps);
}

template <int DT, int K, bool W, bool LN>
frt_status launch_w(int qm, const NormArgs& a, cudaStream_t st) {
  switch (qm) {
    case FRT_QUANT_STATIC: return launch_k<DT, K, W, FRT_QUANT_STATIC, LN>(a, st);
    case FRT_QUANT_BLOCK128: return launch_k<DT, K, W, FRT_QUANT_BLOCK128, LN>(a, st);
    case kQuantNvfp4Rows: return launch_k<DT, K, W, kQuantNvfp4Rows, LN>(a, st);
    default: return launch_k<DT, K, W, kQuantNvfp4Swizzled, LN>(a, st);
  }
}

template <int DT, int K>
frt_status launch_dt_k(bool weighted, bool ln, int qm, const NormArgs& a, cudaStream_t st) {
  if (ln) return weighted ? launch_w<DT, K, true, true>(qm, a, st) : launch_w<DT, K, false, true>(qm, a, st);
  return weighted ? launch_w<DT, K, true, false>(qm, a, st) : launch_w<DT, K, false, false>(qm, a, st);
}

template <int DT>
frt_status launch_dt(int K, bool weighted, bool ln, int qm, const NormArgs& a, cudaStream_t st) {
  switch (K) {
    case 1: return launch_dt_k<DT, 1>(weighted, ln, qm, a, st);
    case 2: return launch_dt_k<DT, 2>(weighted, ln, qm, a, st);
    case 4: return launch_dt_k<DT, 4>(weighted, ln, qm, a, st);
    default: return launch_dt_k<DT, 8>(weighted, ln, qm, a, st);
  }
}

}  // namespace

// Chunks per thread (K) and threads per row (T) for M rows of C 16-byte
// chunks (D = 8C).  Large batches (bandwidth-bound, many rows per SM): K = 1
// up to D = 1024, 2 up to 2048, 4 up to 16384 (128 to 512 threads), 8 up to
// 32768.  Small batches (fewer rows than 4 per SM: latency-bound), up to D =
// 4096: one chunk per thread, which shortens each thread's serial part of the
// row reduction.
static void rmsnorm_shape(int M, int C, int* K, int* T) {
  int k = C <= 128 ? 1 : C <= 256 ? 2 : C <= 2048 ? 4 : 8;
  if (M < 4 * 148 && C <= 512) k = 1;
  const int per = (C + k - 1) / k;
  *K = k;
  *T = ((per + 31) / 32) * 32;
}

}  // namespace frt

extern "C" frt_status frt_residual_rmsnorm_fp8(const void* x, const void* residual_in, void* residual_out,
                                               const void* weight, uint8_t* out_fp8, const float* static_scale,
                                               float* block_scales, int M, int D, float eps, frt_dtype dt,
                                               frt_quant qm, cudaStream_t stream) {
  using namespace frt;
  if (M < 0 || D <= 0 || D % 8 != 0) return FRT_ERR_INVALID_ARG;
  if (!valid_dtype(dt) || !valid_quant(qm)) return FRT_ERR_INVALID_ARG;
  if (D > 32768) return FRT_ERR_UNSUPPORTED;
  if (M == 0) return FRT_OK;
  if (!x || !residual_in || !residual_out || !out_fp8) return FRT_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(residual_in, 16) || !aligned(residual_out, 16) || !aligned(out_fp8, 8))
    return FRT_ERR_INVALID_ARG;
  if (weight && !aligned(weight, 16)) return FRT_ERR_INVALID_ARG;
  if (!quant_args_ok(qm, static_scale, block_scales)) return FRT_ERR_INVALID_ARG;
  const int C = D / 8;
  const int NB = (D + 127) / 128;
  int K, T;
  rmsnorm_shape(M, C, &K, &T);
  const NormArgs a{x, residual_in, residual_out, weight, nullptr, out_fp8, static_scale, block_scales, M, C, NB, T,
                   eps};
  return dt == FRT_F16 ? launch_dt<FRT_F16>(K, weight != nullptr, false, qm, a, stream)
                       : launch_dt<FRT_BF16>(K, weight != nullptr, false, qm, a, stream);
}

extern "C" frt_status frt_residual_rmsnorm_nvfp4(const void* x, const void* residual_in, void* residual_out,
                                                 const void* weight, uint8_t* out_fp4, uint8_t* out_sf,
                                                 const float* global_scale, int M, int D, float eps, frt_dtype dt,
                                                 frt_sf_layout sf_layout, cudaStream_t stream) {
  using namespace frt;
  if (M < 0 || D <= 0 || D % 16 != 0 || !valid_dtype(dt)) return FRT_ERR_INVALID_ARG;
  if (sf_layout != FRT_SF_ROW_MAJOR && sf_layout != FRT_SF_SWIZZLED_128X4) return FRT_ERR_INVALID_ARG;
  if (D > 32768) return FRT_ERR_UNSUPPORTED;
  if (M == 0) return FRT_OK;
  if (!x || !residual_in || !residual_out) return FRT_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(residual_in, 16) || !aligned(residual_out, 16)) return FRT_ERR_INVALID_ARG;
  if (weight && !aligned(weight, 16)) return FRT_ERR_INVALID_ARG;
  if (!nvfp4_args_ok(sf_layout, global_scale, out_fp4, out_sf, 4)) return FRT_ERR_INVALID_ARG;
  const int C = D / 8;
  int K, T;
  rmsnorm_shape(M, C, &K, &T);
  const int qm = sf_layout == FRT_SF_ROW_MAJOR ? kQuantNvfp4Rows : kQuantNvfp4Swizzled;
  float* sf = reinterpret_cast<float*>(out_sf);  // the kernel's scale pointer carries the sf bytes
  const NormArgs a{x, residual_in, residual_out, weight, nullptr, out_fp4, global_scale, sf, M, C, 0, T, eps};
  return dt == FRT_F16 ? launch_dt<FRT_F16>(K, weight != nullptr, false, qm, a, stream)
                       : launch_dt<FRT_BF16>(K, weight != nullptr, false, qm, a, stream);
}

// NEXT-4: residual add + LayerNorm producers (the ViT "add_layer_norm").
namespace frt {
namespace {
frt_status layernorm_op(const void* x, const void* residual_in, void* residual_out, const void* weight,
                        const void* bias, uint8_t* out, const float* scale, float* scales_out, int M, int D,
                        float eps, frt_dtype dt, int qm, cudaStream_t stream) {
  if (M == 0) return FRT_OK;
  if (!x || !residual_in || !residual_out) return FRT_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(residual_in, 16) || !aligned(residual_out, 16)) return FRT_ERR_INVALID_ARG;
  if ((weight && !aligned(weight, 16)) || (bias && !aligned(bias, 16))) return FRT_ERR_INVALID_ARG;
  const int C = D / 8;
  int K, T;
  rmsnorm_shape(M, C, &K, &T);
  const NormArgs a{x, residual_in, residual_out, weight, bias, out, scale, scales_out, M, C, (D + 127) / 128, T,
                   eps};
  return dt == FRT_F16 ? launch_dt<FRT_F16>(K, weight != nullptr, true, qm, a, stream)
                       : launch_dt<FRT_BF16>(K, weight != nullptr, true, qm, a, stream);
}
}  // namespace
}  // namespace frt

extern "C" frt_status frt_residual_layernorm_fp8(const void* x, const void* residual_in, void* residual_out,
                                                 const void* weight, const void* bias, uint8_t* out_fp8,
                                                 const float* static_scale, float* block_scales, int M, int D,
                                                 float eps, frt_dtype dt, frt_quant qm, cudaStream_t stream) {
  using namespace frt;
  if (M < 0 || D <= 0 || D % 8 != 0 || !valid_dtype(dt) || !valid_quant(qm)) return FRT_ERR_INVALID_ARG;
  if (D > 32768) return FRT_ERR_UNSUPPORTED;
  if (M > 0 && (!out_fp8 || !aligned(out_fp8, 8) || !quant_args_ok(qm, static_scale, block_scales)))
    return FRT_ERR_INVALID_ARG;
  return layernorm_op(x, residual_in, residual_out, weight, bias, out_fp8, static_scale, block_scales, M, D, eps, dt,
                      qm, stream);
}

extern "C" frt_status frt_residual_layernorm_nvfp4(const void* x, const void* residual_in, void* residual_out,
                                                   const void* weight, const void* bias, uint8_t* out_fp4,
                                                   uint8_t* out_sf, const float* global_scale, int M, int D,
                                                   float eps, frt_dtype dt, frt_sf_layout sf_layout,
                                                   cudaStream_t stream) {
  using namespace frt;
  if (M < 0 || D <= 0 || D % 16 != 0 || !valid_dtype(dt)) return FRT_ERR_INVALID_ARG;
  if (sf_layout != FRT_SF_ROW_MAJOR && sf_layout != FRT_SF_SWIZZLED_128X4) return FRT_ERR_INVALID_ARG;
  if (D > 32768) return FRT_ERR_UNSUPPORTED;
  if (M > 0 && !nvfp4_args_ok(sf_layout, global_scale, out_fp4, out_sf, 4)) return FRT_ERR_INVALID_ARG;
  const int qm = sf_layout == FRT_SF_ROW_MAJOR ? kQuantNvfp4Rows : kQuantNvfp4Swizzled;
  return layernorm_op(x, residual_in, residual_out, weight, bias, out_fp4, global_scale,
                      reinterpret_cast<float*>(out_sf), M, D, eps, dt, qm, stream);
}
