// NEXT-1: gated residual + AdaRMSNorm modulation + FP8 e4m3.
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
// Mapping (B200): op (a)'s layout -- one small CTA per row, thread t owns the
// 16-byte chunks t, t+T, ... of the row, sum of squares warp shuffle ->
// shared memory -> every thread.  Every load is issued at entry: x and the
// residual (HBM) and the gate (L2) into registers, scale and shift by
// asynchronous copies into shared memory, which holds them without registers
// until pass 2 needs them (each thread copies and reads back only its own
// chunks, so the staging needs no barrier).
//
// Arithmetic.  h is one packed 16-bit FMA per pair (fma.rn.{bf16x2,f16x2}:
// the exact g * x + r rounded once, subnormals kept), which is the oracle's
// definition itself.  Without modulation the sum of squares is fp64 and
// y = h * rstd is the correctly rounded fp32 value, as in op (a); with
// modulation y carries three fp32 roundings anyway and an fp32 sum of squares
// suffices.  Without modulation the FP8 codes are those of the correctly
// rounded quotient y / s; with it the division is a product (a static scale
// folded into rstd and the shift, block-128 scales through RN(1 / s_b)), one
// more fp32 rounding on top of y's.
#include <atomic>
#include <cmath>
#include <type_traits>

#include "frt_device.cuh"
#include "frt_host.h"

namespace frt {
namespace {

template <int K>
constexpr int max_threads() {
  return K >= 4 ? 512 : 128;
}

// 16-byte asynchronous global -> shared copy (cached in L2 only), and its
// group bookkeeping.
__device__ __forceinline__ void cp_async16(uint4* smem, const uint4* gmem) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

template <int DT, int K, bool GATED, bool MOD, int QM>
__global__ void __launch_bounds__(max_threads<K>()) gate_residual_adarms_fp8_kernel(
    const uint4* __restrict__ x, const uint4* __restrict__ gate, const uint4* r_in, uint4* r_out,
    const uint4* __restrict__ scale, const uint4* __restrict__ shift, uint2* __restrict__ q,
    const float* __restrict__ static_scale, float* __restrict__ block_scales, int C, int NB, int rows_per_cond,
    float D, float eps) {
  using P16 = Pack16<DT>;
  using Acc = typename std::conditional<MOD, float, double>::type;
  // The gate rides in registers with x and the residual; at the widest rows
  // (K = 8) registers run out and it is staged in shared memory instead.
  constexpr bool kGateSmem = K >= 8;
  // the static scale is a constant input: read before the wait for the
  // previous kernel (the gate, scale and shift rows are computed per step by
  // a preceding kernel, so they wait)
  float s_static = 0.0f;
  if (QM == FRT_QUANT_STATIC && FRT_IDX_OK(0, 1)) s_static = __ldg(static_scale);
  pdl_enter();
  const int t = threadIdx.x;
  const int T = blockDim.x;
  const int64_t row = blockIdx.x;
  const int64_t base = row * (int64_t)C;
  const int64_t cbase = (int64_t)((int)blockIdx.x / rows_per_cond) * C;
  __shared__ double red[32];
  extern __shared__ uint4 cond[];
  uint4* s_gate = cond;
  uint4* s_scale = cond + (GATED && kGateSmem ? C : 0);
  uint4* s_shift = s_scale + C;

  // extents: [M, C] 16-byte chunks of x / r / q, [ceil(M / rows_per_cond), C] of the condition rows
  const int64_t n_rc = (int64_t)gridDim.x * C;
  const int64_t n_cond = ((int64_t)gridDim.x + rows_per_cond - 1) / rows_per_cond * C;
  uint4 xv[K], rv[K], gv[GATED && !kGateSmem ? K : 1];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = t + k * T;
    if (c < C && FRT_IDX_OK(base + c, n_rc)) {
      xv[k] = ld_stream(x + base + c);
      rv[k] = ld_plain(r_in + base + c);
      if (GATED && !kGateSmem && FRT_IDX_OK(cbase + c, n_cond)) gv[k] = __ldg(gate + cbase + c);
    }
  }
  if (GATED && kGateSmem) {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if (t + k * T < C && FRT_IDX_OK(cbase + t + k * T, n_cond))
        cp_async16(s_gate + t + k * T, gate + cbase + t + k * T);
    cp_async_commit();
  }
  if (MOD) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int c = t + k * T;
      if (c < C) {
        if (scale != nullptr && FRT_IDX_OK(cbase + c, n_cond)) cp_async16(s_scale + c, scale + cbase + c);
        else s_scale[c] = make_uint4(0u, 0u, 0u, 0u);  // 16-bit zeros
        if (shift != nullptr && FRT_IDX_OK(cbase + c, n_cond)) cp_async16(s_shift + c, shift + cbase + c);
        else s_shift[c] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    cp_async_commit();
  }
  if (GATED && kGateSmem) {
    if (MOD) cp_async_wait<1>();  // the gate group; scale / shift may still be in flight
    else cp_async_wait<0>();
  }

  // Pass 1: h = gate * x + r rounded once to 16 bits (packed), written back;
  // sum of squares (squares of 16-bit values are exact in fp32).
  uint4 hv[K];
  Acc ss = 0;
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = t + k * T;
    hv[k] = make_uint4(0u, 0u, 0u, 0u);
    if (c < C) {
      const uint32_t* xw = reinterpret_cast<const uint32_t*>(&xv[k]);
      const uint32_t* rw = reinterpret_cast<const uint32_t*>(&rv[k]);
      uint4 g = make_uint4(0u, 0u, 0u, 0u);
      if (GATED) g = kGateSmem ? s_gate[c] : gv[kGateSmem ? 0 : k];
      const uint32_t* gw = reinterpret_cast<const uint32_t*>(&g);
      uint32_t* hw = reinterpret_cast<uint32_t*>(&hv[k]);
      Acc sk = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // h = g * x + r with one rounding of the exact value: the packed
        // 16-bit FMA (without a gate, 1 * x + r).
        hw[e] = P16::fma2(GATED ? gw[e] : P16::kOnes, xw[e], rw[e]);
        const float2 hf = P16::to_float2(hw[e]);
        sk = fma((Acc)hf.x, (Acc)hf.x, sk);
        sk = fma((Acc)hf.y, (Acc)hf.y, sk);
      }
      ss += sk;
      if (FRT_IDX_OK(base + c, n_rc)) r_out[base + c] = hv[k];
    }
  }

  // Row total: warp butterfly, then every thread adds the warp partials in
  // the same order (bitwise deterministic).
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
  if ((t & 31) == 0) red[t >> 5] = (double)ss;
  __syncthreads();
  double tot = 0.0;
  const int nw = T >> 5;
  for (int i = 0; i < nw; ++i) tot += red[i];
  const Split32 rstd(MOD ? 0.0 : rsqrt_f64(tot / (double)D + (double)eps));
  const float rstd32 = MOD ? rsqrtf((float)tot / D + eps) : 0.0f;
  const Divisor dv_static(QM == FRT_QUANT_STATIC ? s_static : 1.0f);
  // Modulated rows carry a few fp32 roundings anyway, so a static scale is
  // folded in (rstd / s and shift / s: y / s in one pass, no divide) when s
  // lies in [2^-100, 2^100]; block-128 scales divide through RN(1 / s_b).
  const bool mfold = MOD && QM == FRT_QUANT_STATIC && dv_static.fast;
  const float mrs = mfold ? rstd32 * dv_static.inv : rstd32;
  const float msh = mfold ? dv_static.inv : 1.0f;
  if (MOD) cp_async_wait<0>();

  // Pass 2: y and its FP8 codes.
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = t + k * T;
    const bool valid = c < C;
    const uint32_t* hw = reinterpret_cast<const uint32_t*>(&hv[k]);
    float y[8];
    if (MOD) {
      uint4 scv = make_uint4(0u, 0u, 0u, 0u), shv = make_uint4(0u, 0u, 0u, 0u);
      if (valid) {
        scv = s_scale[c];
        shv = s_shift[c];
      }
      const uint32_t* scw = reinterpret_cast<const uint32_t*>(&scv);
      const uint32_t* shw = reinterpret_cast<const uint32_t*>(&shv);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 hf = P16::to_float2(hw[e]);
        const float2 sc = P16::to_float2(scw[e]);
        const float2 sh = P16::to_float2(shw[e]);
        y[2 * e] = fmaf(hf.x * mrs, 1.0f + sc.x, sh.x * msh);
        y[2 * e + 1] = fmaf(hf.y * mrs, 1.0f + sc.y, sh.y * msh);
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
      am = half_warp_max_abs(am);
      const float sb = block_scale_448(am);
      if (valid && (t & 15) == 0 && FRT_IDX_OK(row * NB + (c >> 4), (int64_t)gridDim.x * NB))
        block_scales[row * NB + (c >> 4)] = sb;
      if (valid && FRT_IDX_OK(base + c, n_rc)) {
        if (MOD && sb >= 0x1p-100f && sb <= 0x1p+100f) {
          const float r = __frcp_rn(sb);
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = y[e] * r;
          q[base + c] = e4m3x8(v);
        } else {
          q[base + c] = quant8(y, Divisor(sb));
        }
      }
    } else if (valid && FRT_IDX_OK(base + c, n_rc)) {
      q[base + c] = mfold ? e4m3x8(y) : quant8(y, dv_static);
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

template <int DT, int K, bool G, bool MOD, int QM>
frt_status launch_k(const Args& a, cudaStream_t st) {
  static std::atomic<int> opted{0};
  auto kern = gate_residual_adarms_fp8_kernel<DT, K, G, MOD, QM>;
  const size_t smem = (size_t)((G && K >= 8 ? 1 : 0) + (MOD ? 2 : 0)) * a.C * sizeof(uint4);
  const frt_status os = opt_in_smem(kern, smem, opted);
  if (os != FRT_OK) return os;
  return launch(kern, dim3(a.M), dim3(a.T), smem, st, static_cast<const uint4*>(a.x),
                static_cast<const uint4*>(a.gate), static_cast<const uint4*>(a.r_in), static_cast<uint4*>(a.r_out),
                static_cast<const uint4*>(a.scale), static_cast<const uint4*>(a.shift), reinterpret_cast<uint2*>(a.q),
                a.ss, a.bs, a.C, a.NB, a.rows_per_cond, (float)(a.C * 8), a.eps);
}

template <int DT, int K, bool G>
frt_status launch_gk(bool mod, frt_quant qm, const Args& a, cudaStream_t st) {
  if (mod)
    return qm == FRT_QUANT_STATIC ? launch_k<DT, K, G, true, FRT_QUANT_STATIC>(a, st)
                                  : launch_k<DT, K, G, true, FRT_QUANT_BLOCK128>(a, st);
  return qm == FRT_QUANT_STATIC ? launch_k<DT, K, G, false, FRT_QUANT_STATIC>(a, st)
                                : launch_k<DT, K, G, false, FRT_QUANT_BLOCK128>(a, st);
}

template <int DT, int K>
frt_status launch_dk(bool gated, bool mod, frt_quant qm, const Args& a, cudaStream_t st) {
  return gated ? launch_gk<DT, K, true>(mod, qm, a, st) : launch_gk<DT, K, false>(mod, qm, a, st);
}

template <int DT>
frt_status launch_dt(int K, bool gated, bool mod, frt_quant qm, const Args& a, cudaStream_t st) {
  switch (K) {
    case 1: return launch_dk<DT, 1>(gated, mod, qm, a, st);
    case 2: return launch_dk<DT, 2>(gated, mod, qm, a, st);
    case 4: return launch_dk<DT, 4>(gated, mod, qm, a, st);
    default: return launch_dk<DT, 8>(gated, mod, qm, a, st);
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
  const bool mod = scale != nullptr || shift != nullptr;
  return dt == FRT_F16 ? launch_dt<FRT_F16>(K, gate != nullptr, mod, qm, a, stream)
                       : launch_dt<FRT_BF16>(K, gate != nullptr, mod, qm, a, stream);
}
