// NEXT-1: gated residual + AdaRMSNorm modulation + FP8 e4m3, one pass per row.
//
// "FlashRT kernel fusion", §三: the Pi0.5 decoder's cross-layer kernel
// gate_res_adarms_fp8_static does gate multiply + residual add + AdaRMSNorm
// modulation + FP8 quantisation + descale in one kernel (6 ops -> 1) and runs
// 180 times per decode (18 layers x 10 flow steps).  Per row i with condition
// row c = i / rows_per_cond:
//   h = x * gate_c + residual (exact value rounded once), written back;
//   y = h * rstd * (1 + scale_c) + shift_c,  rstd = 1 / sqrt(mean(h^2) + eps);
//   FP8 of y (static scale or per-token block-128 scales), as op (a).
//
// Same mapping as op (a): one small CTA per row, 16-byte vectors, fp64 sum of
// squares, h * rstd formed as a correctly rounded fp32 value, FP8 codes of the
// correctly rounded quotient.
#include <cmath>

#include "frt_device.cuh"
#include "frt_host.h"

namespace frt {
namespace {

template <int K>
constexpr int max_threads() {
  return K >= 4 ? 512 : 128;
}

// True when s is a rounding midpoint of the 16-bit type DT.
template <int DT>
__device__ __forceinline__ bool midpoint16(float s) {
  const uint32_t u = __float_as_uint(s);
  if (DT == FRT_BF16) return (u & 0xFFFFu) == 0x8000u;
  const float a = fabsf(s);
  if (a >= 0x1p-14f) return (u & 0x1FFFu) == 0x1000u;
  const float t = a * 0x1p25f;  // fp16 subnormal midpoints: odd multiples of 2^-25
  return t == rintf(t) && (((int)t) & 1);
}

// r + p (p = g * x, exact in fp32) rounded so that one more rounding to the
// 16-bit type is the correctly rounded exact sum: the fp32 sum from TwoSum,
// moved one ulp towards the exact value only when it sits exactly on a 16-bit
// midpoint while the sum was inexact (the one case where rounding it again
// would differ).  Branch-free.
template <int DT>
__device__ __forceinline__ float gated_sum(float r, float p) {
  const float s = __fadd_rn(r, p);
  const float bb = __fsub_rn(s, r);
  const float e = __fadd_rn(__fsub_rn(r, __fsub_rn(s, bb)), __fsub_rn(p, bb));
  const uint32_t u = __float_as_uint(s);
  const uint32_t toward = ((__float_as_uint(e) ^ u) & 0x80000000u) ? u - 1u : u + 1u;
  return (e != 0.0f && midpoint16<DT>(s)) ? __uint_as_float(toward) : s;
}

template <int DT, int K, bool GATED, int QM>
__global__ void __launch_bounds__(max_threads<K>()) gate_residual_adarms_fp8_kernel(
    const uint4* __restrict__ x, const uint4* __restrict__ gate, const uint4* r_in, uint4* r_out,
    const uint4* __restrict__ scale, const uint4* __restrict__ shift, uint2* __restrict__ q,
    const float* __restrict__ static_scale, float* __restrict__ block_scales, int C, int NB, int rows_per_cond,
    float D, float eps) {
  using P16 = Pack16<DT>;
  pdl_enter();
  const int t = threadIdx.x;
  const int T = blockDim.x;
  const int64_t row = blockIdx.x;
  const int64_t base = row * (int64_t)C;
  const int64_t cbase = (row / rows_per_cond) * (int64_t)C;
  __shared__ double red[32];

  uint4 xv[K], rv[K], gv[GATED ? K : 1];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = t + k * T;
    if (c < C) {
      xv[k] = ld_stream(x + base + c);
      rv[k] = ld_plain(r_in + base + c);
      if (GATED) gv[k] = __ldg(gate + cbase + c);
    }
  }
  float s_static = 0.0f;
  if (QM == FRT_QUANT_STATIC) s_static = __ldg(static_scale);

  // Pass 1: h = gate * x + r rounded once to 16 bits (packed), fp64 sum of squares.
  uint4 hv[K];
  double ss[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    ss[k] = 0.0;
    const int c = t + k * T;
    if (c < C) {
      const uint32_t* xw = reinterpret_cast<const uint32_t*>(&xv[k]);
      const uint32_t* rw = reinterpret_cast<const uint32_t*>(&rv[k]);
      const uint32_t* gw = reinterpret_cast<const uint32_t*>(&gv[GATED ? k : 0]);
      uint32_t* hw = reinterpret_cast<uint32_t*>(&hv[k]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 xf = P16::to_float2(xw[e]);
        const float2 rf = P16::to_float2(rw[e]);
        float s0, s1;
        if (GATED) {
          const float2 gf = P16::to_float2(gw[e]);
          s0 = gated_sum<DT>(rf.x, gf.x * xf.x);  // 16-bit x 16-bit: exact in fp32
          s1 = gated_sum<DT>(rf.y, gf.y * xf.y);
        } else {
          s0 = add_for_16(xf.x, rf.x);
          s1 = add_for_16(xf.y, rf.y);
        }
        hw[e] = P16::from_float2(s0, s1);
        const float2 hf = P16::to_float2(hw[e]);
        ss[k] = fma((double)hf.x, (double)hf.x, ss[k]);
        ss[k] = fma((double)hf.y, (double)hf.y, ss[k]);
      }
      r_out[base + c] = hv[k];
    } else {
      hv[k] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  double sst = ss[0];
#pragma unroll
  for (int k = 1; k < K; ++k) sst += ss[k];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sst += __shfl_xor_sync(0xFFFFFFFFu, sst, o);
  if ((t & 31) == 0) red[t >> 5] = sst;
  __syncthreads();
  double tot = 0.0;
  const int nw = T >> 5;
  for (int i = 0; i < nw; ++i) tot += red[i];
  const Split32 rstd(rsqrt_f64(tot / (double)D + (double)eps));
  const Divisor dv_static(QM == FRT_QUANT_STATIC ? s_static : 1.0f);

  // Pass 2: y = h * rstd * (1 + scale) + shift, then FP8.
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = t + k * T;
    const bool valid = c < C;
    const uint32_t* hw = reinterpret_cast<const uint32_t*>(&hv[k]);
    uint4 scv = make_uint4(0u, 0u, 0u, 0u), shv = make_uint4(0u, 0u, 0u, 0u);  // 16-bit zeros
    if (valid && scale != nullptr) scv = __ldg(scale + cbase + c);
    if (valid && shift != nullptr) shv = __ldg(shift + cbase + c);
    const uint32_t* scw = reinterpret_cast<const uint32_t*>(&scv);
    const uint32_t* shw = reinterpret_cast<const uint32_t*>(&shv);
    float y[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 hf = P16::to_float2(hw[e]);
      const float2 sc = P16::to_float2(scw[e]);
      const float2 sh = P16::to_float2(shw[e]);
      y[2 * e] = fmaf(rstd.mul(hf.x), 1.0f + sc.x, sh.x);
      y[2 * e + 1] = fmaf(rstd.mul(hf.y), 1.0f + sc.y, sh.y);
    }
    if (QM == FRT_QUANT_BLOCK128) {
      float am = fmaxf(absmax4(y[0], y[1], y[2], y[3]), absmax4(y[4], y[5], y[6], y[7]));
      am = group_max<16>(am);
      const float sb = am > 0.0f ? __fdiv_rn(am, 448.0f) : 1.0f;
      if (valid && (t & 15) == 0) block_scales[row * NB + (c >> 4)] = sb;
      if (valid) q[base + c] = quant8(y, Divisor(sb));
    } else if (valid) {
      q[base + c] = quant8(y, dv_static);
    }
  }
}

struct Args {
  const void *x, *gate, *r_in;
  void* r_out;
  const void *scale, *shift;
  uint8_t* q;
  const float* ss;
  float* bs;
  int M, C, NB, rows_per_cond, T;
  float eps;
};

template <int DT, int K, bool G, int QM>
frt_status launch_k(const Args& a, cudaStream_t st) {
  return launch(gate_residual_adarms_fp8_kernel<DT, K, G, QM>, dim3(a.M), dim3(a.T), 0, st,
                static_cast<const uint4*>(a.x), static_cast<const uint4*>(a.gate), static_cast<const uint4*>(a.r_in),
                static_cast<uint4*>(a.r_out), static_cast<const uint4*>(a.scale), static_cast<const uint4*>(a.shift),
                reinterpret_cast<uint2*>(a.q), a.ss, a.bs, a.C, a.NB, a.rows_per_cond, (float)(a.C * 8), a.eps);
}

template <int DT, int K>
frt_status launch_dk(bool gated, frt_quant qm, const Args& a, cudaStream_t st) {
  if (gated)
    return qm == FRT_QUANT_STATIC ? launch_k<DT, K, true, FRT_QUANT_STATIC>(a, st)
                                  : launch_k<DT, K, true, FRT_QUANT_BLOCK128>(a, st);
  return qm == FRT_QUANT_STATIC ? launch_k<DT, K, false, FRT_QUANT_STATIC>(a, st)
                                : launch_k<DT, K, false, FRT_QUANT_BLOCK128>(a, st);
}

template <int DT>
frt_status launch_dt(int K, bool gated, frt_quant qm, const Args& a, cudaStream_t st) {
  switch (K) {
    case 1: return launch_dk<DT, 1>(gated, qm, a, st);
    case 2: return launch_dk<DT, 2>(gated, qm, a, st);
    case 4: return launch_dk<DT, 4>(gated, qm, a, st);
    default: return launch_dk<DT, 8>(gated, qm, a, st);
  }
}

}  // namespace
}  // namespace frt

extern "C" frt_status frt_gate_residual_adarms_fp8(const void* x, const void* gate, const void* residual_in,
                                                   void* residual_out, const void* scale, const void* shift,
                                                   uint8_t* out_fp8, const float* static_scale, float* block_scales,
                                                   int M, int D, int rows_per_cond, float eps, frt_dtype dt,
                                                   frt_quant qm, cudaStream_t stream) {
  using namespace frt;
  if (M < 0 || D <= 0 || D % 8 != 0 || rows_per_cond <= 0) return FRT_ERR_INVALID_ARG;
  if (!valid_dtype(dt) || !valid_quant(qm)) return FRT_ERR_INVALID_ARG;
  if (D > 32768) return FRT_ERR_UNSUPPORTED;
  if (M == 0) return FRT_OK;
  if (!x || !residual_in || !residual_out || !out_fp8) return FRT_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(residual_in, 16) || !aligned(residual_out, 16) || !aligned(out_fp8, 8))
    return FRT_ERR_INVALID_ARG;
  if ((gate && !aligned(gate, 16)) || (scale && !aligned(scale, 16)) || (shift && !aligned(shift, 16)))
    return FRT_ERR_INVALID_ARG;
  if (!quant_args_ok(qm, static_scale, block_scales)) return FRT_ERR_INVALID_ARG;
  const int C = D / 8;
  const int K = C <= 128 ? 1 : C <= 256 ? 2 : C <= 2048 ? 4 : 8;
  const int per = (C + K - 1) / K;
  Args a{x, gate, residual_in, residual_out, scale, shift, out_fp8, static_scale, block_scales, M, C,
         (D + 127) / 128, rows_per_cond, ((per + 31) / 32) * 32, eps};
  return dt == FRT_F16 ? launch_dt<FRT_F16>(K, gate != nullptr, qm, a, stream)
                       : launch_dt<FRT_BF16>(K, gate != nullptr, qm, a, stream);
}
