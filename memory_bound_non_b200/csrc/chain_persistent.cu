// NEXT-4: the layer chain as one persistent kernel (small batches).
//
// "FlashFormer: Whole-Model Kernels for Efficient Low-Batch Inference": at a
// few tokens the per-kernel launch and dependency latency dominates, so the
// whole sequence runs inside one kernel.  Here that sequence is the graphed
// chain: for every step and layer, op a (attention norm), op b (QKV), op a
// (FFN norm), op c (gated activation) ("FlashRT kernel fusion", §二 steps 1,
// 3, 7, 8-10; §三 for the per-step loop).
//
// Mapping (B200): one CTA of 256 threads per token row.  The chain's only
// dependency is the residual stream of each row (a -> a -> next layer's a);
// the QKV and gate/up buffers that ops b and c read are the fixed per-layer
// outputs of GEMMs that are not part of the chain, so every op of a row
// depends on that row alone and the CTA runs the row's whole chain in program
// order, with the residual row held in registers from the first op to the
// last (written back once).  No grid-wide barrier is needed; with real GEMMs
// between the ops it would be (those mix rows).  Each op uses the arithmetic
// of its per-op kernel (packed 16-bit add, fp64 row sum of squares, correctly
// rounded FP8 decisions, the same RoPE and activation expressions).
#include <atomic>
#include <cmath>

#include "frt_device.cuh"
#include "frt_host.h"

namespace frt {
namespace {

constexpr int kChainThreads = 256;
constexpr int kChainWarps = kChainThreads / 32;

// Block-wide fp64 sum (warp butterfly, then the warp partials in order); the
// trailing barrier lets the next call reuse `red`.
__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double tot = 0.0;
  for (int i = 0; i < kChainWarps; ++i) tot += red[i];
  __syncthreads();
  return tot;
}

// Op a on this CTA's row: h = x + r (into hv), RMSNorm, FP8 codes.
template <int DT, int K, int QM>
__device__ __forceinline__ void chain_norm(const uint4* __restrict__ x, const uint4* __restrict__ w, uint2* q,
                                           float* bs, const Divisor& dv, uint4 (&hv)[K], int64_t row, int C, int NB,
                                           float D, float eps, double* red) {
  using P16 = Pack16<DT>;
  const int t = threadIdx.x;
  uint4 xv[K], wv[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = t + k * kChainThreads;
    if (c < C) {
      xv[k] = ld_stream(x + row * C + c);
      if (w != nullptr) wv[k] = __ldg(w + c);
    }
  }
  double ss[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    ss[k] = 0.0;
    if (t + k * kChainThreads < C) {
      const uint32_t* xw = reinterpret_cast<const uint32_t*>(&xv[k]);
      uint32_t* hw = reinterpret_cast<uint32_t*>(&hv[k]);
#pragma unroll
      for (int e = 0; e < 4; ++e) hw[e] = P16::fma2(P16::kOnes, xw[e], hw[e]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 hf = P16::to_float2(hw[e]);
        ss[k] = fma((double)hf.x, (double)hf.x, ss[k]);
        ss[k] = fma((double)hf.y, (double)hf.y, ss[k]);
      }
    }
  }
  double sst = ss[0];
#pragma unroll
  for (int k = 1; k < K; ++k) sst += ss[k];
  const Split32 rstd(rsqrt_f64(block_sum(sst, red) / (double)D + (double)eps));
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = t + k * kChainThreads;
    const bool valid = c < C;
    const uint32_t* hw = reinterpret_cast<const uint32_t*>(&hv[k]);
    const uint32_t* ww = reinterpret_cast<const uint32_t*>(&wv[k]);
    float y[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 hf = P16::to_float2(hw[e]);
      if (w != nullptr && valid) {
        const float2 wf = P16::to_float2(ww[e]);
        y[2 * e] = rstd.mul(hf.x * wf.x);
        y[2 * e + 1] = rstd.mul(hf.y * wf.y);
      } else {
        y[2 * e] = rstd.mul(hf.x);
        y[2 * e + 1] = rstd.mul(hf.y);
      }
    }
    if (QM == FRT_QUANT_BLOCK128) {
      float am = fmaxf(absmax4(y[0], y[1], y[2], y[3]), absmax4(y[4], y[5], y[6], y[7]));
      am = group_max<16>(am);
      const float sb = am > 0.0f ? __fdiv_rn(am, 448.0f) : 1.0f;
      if (valid && (t & 15) == 0) bs[row * NB + (c >> 4)] = sb;
      if (valid) q[row * C + c] = quant8(y, Divisor(sb));
    } else if (valid) {
      q[row * C + c] = quant8(y, dv);
    }
  }
}

// Op b on this CTA's token: lane groups of GP lanes per head (P = 8 elements
// and their rotation partners per lane), T / GP heads per slot.
template <int DT, int GP>
__device__ __forceinline__ void chain_qkv(const uint16_t* __restrict__ qkv, const uint16_t* __restrict__ qw,
                                          const uint16_t* __restrict__ kw, uint16_t* q_out, uint16_t* k_cache,
                                          uint16_t* v_cache, const float* c, const float* s, int64_t row, int p,
                                          bool row_ok, int Hq, int Hkv, int hd, int G, float eps) {
  constexpr int P = 8;
  const int H = Hq + 2 * Hkv;
  const int NG = kChainThreads / GP;
  const int grp = threadIdx.x / GP;
  const int li = threadIdx.x & (GP - 1);
  const int half = hd >> 1;
  const int j0 = li * P;
  const bool lane_ok = li < G && row_ok;
  const uint16_t* rowp = qkv + row * H * hd;
  uint4 qwa = make_uint4(0, 0, 0, 0), qwb = qwa, kwa = qwa, kwb = qwa;
  if (lane_ok) {
    if (qw != nullptr) {
      qwa = *reinterpret_cast<const uint4*>(qw + j0);
      qwb = *reinterpret_cast<const uint4*>(qw + half + j0);
    }
    if (kw != nullptr) {
      kwa = *reinterpret_cast<const uint4*>(kw + j0);
      kwb = *reinterpret_cast<const uint4*>(kw + half + j0);
    }
  }
  for (int h0 = 0; h0 < H; h0 += NG) {
    const int h = h0 + grp;
    const bool on = lane_ok && h < H;
    const bool is_q = h < Hq;
    const bool is_v = h >= Hq + Hkv;
    const uint16_t* nw = is_q ? qw : kw;
    const bool do_norm = !is_v && nw != nullptr;
    uint4 va = make_uint4(0, 0, 0, 0), vb = va;
    if (on) {
      va = *reinterpret_cast<const uint4*>(rowp + (int64_t)h * hd + j0);
      vb = *reinterpret_cast<const uint4*>(rowp + (int64_t)h * hd + half + j0);
    }
    if (on && is_v) {
      uint16_t* dst = v_cache + ((int64_t)p * Hkv + (h - Hq - Hkv)) * hd;
      *reinterpret_cast<uint4*>(dst + j0) = va;
      *reinterpret_cast<uint4*>(dst + half + j0) = vb;
    }
    float a[P], b[P];
    float ss = 0.0f;
    if (on && !is_v) {
#pragma unroll
      for (int e = 0; e < P / 2; ++e) {
        const float2 ta = Pack16<DT>::to_float2(reinterpret_cast<const uint32_t*>(&va)[e]);
        const float2 tb = Pack16<DT>::to_float2(reinterpret_cast<const uint32_t*>(&vb)[e]);
        a[2 * e] = ta.x;
        a[2 * e + 1] = ta.y;
        b[2 * e] = tb.x;
        b[2 * e + 1] = tb.y;
      }
      if (do_norm) {
#pragma unroll
        for (int e = 0; e < P; ++e) ss = fmaf(b[e], b[e], fmaf(a[e], a[e], ss));
      }
    }
    ss = group_sum<GP>(ss);  // every lane of the warp takes part
    if (on && !is_v) {
      if (do_norm) {
        const float rstd = 1.0f / sqrtf(ss / (float)hd + eps);
        const uint4 wa = is_q ? qwa : kwa, wb = is_q ? qwb : kwb;
#pragma unroll
        for (int e = 0; e < P / 2; ++e) {
          const float2 fa = Pack16<DT>::to_float2(reinterpret_cast<const uint32_t*>(&wa)[e]);
          const float2 fb = Pack16<DT>::to_float2(reinterpret_cast<const uint32_t*>(&wb)[e]);
          a[2 * e] = a[2 * e] * rstd * fa.x;
          a[2 * e + 1] = a[2 * e + 1] * rstd * fa.y;
          b[2 * e] = b[2 * e] * rstd * fb.x;
          b[2 * e + 1] = b[2 * e + 1] * rstd * fb.y;
        }
      }
      uint4 o1, o2;
#pragma unroll
      for (int e = 0; e < P / 2; ++e) {
        const float x0 = fmaf(a[2 * e], c[2 * e], -(b[2 * e] * s[2 * e]));
        const float x1 = fmaf(a[2 * e + 1], c[2 * e + 1], -(b[2 * e + 1] * s[2 * e + 1]));
        const float y0 = fmaf(b[2 * e], c[2 * e], a[2 * e] * s[2 * e]);
        const float y1 = fmaf(b[2 * e + 1], c[2 * e + 1], a[2 * e + 1] * s[2 * e + 1]);
        reinterpret_cast<uint32_t*>(&o1)[e] = Pack16<DT>::from_float2(x0, x1);
        reinterpret_cast<uint32_t*>(&o2)[e] = Pack16<DT>::from_float2(y0, y1);
      }
      uint16_t* dst = is_q ? q_out + (row * Hq + h) * hd : k_cache + ((int64_t)p * Hkv + (h - Hq)) * hd;
      *reinterpret_cast<uint4*>(dst + j0) = o1;
      *reinterpret_cast<uint4*>(dst + half + j0) = o2;
    }
  }
}

// Op c on this CTA's row: each warp takes 128-output scale blocks, four at a
// time with their loads issued first (one 16-byte load = 4 (g, u) pairs).
template <int DT, int QM>
__device__ __forceinline__ void chain_act(const uint4* __restrict__ gu, uint32_t* q, float* bs, const Divisor& dv,
                                          int64_t row, int I4, int NBI, int act) {
  using P16 = Pack16<DT>;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint4* src = gu + row * I4;
  uint32_t* dst = q + row * I4;
  for (int b0 = warp * 4; b0 < NBI; b0 += kChainWarps * 4) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (b0 + u < NBI) v[u] = ld_stream(src + (b0 + u) * 32 + lane);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (b0 + u >= NBI) break;  // uniform across the warp
      float a[4];
      const uint32_t* w = reinterpret_cast<const uint32_t*>(&v[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 pr = P16::to_float2(w[e]);
        // the activation is uniform for the launch (a branch, not a template)
        const float g = act == FRT_ACT_RELU2 ? act_fn<FRT_ACT_RELU2>(pr.x)
                        : act == FRT_ACT_SILU ? act_fn<FRT_ACT_SILU>(pr.x)
                                              : act_fn<FRT_ACT_GELU_TANH>(pr.x);
        a[e] = g * pr.y;
      }
      if (QM == FRT_QUANT_BLOCK128) {
        const float am = group_max<32>(absmax4(a[0], a[1], a[2], a[3]));
        const float sb = am > 0.0f ? __fdiv_rn(am, 448.0f) : 1.0f;
        if (lane == 0) bs[row * NBI + b0 + u] = sb;
        dst[(b0 + u) * 32 + lane] = quant4(a, Divisor(sb));
      } else {
        dst[(b0 + u) * 32 + lane] = quant4(a, dv);
      }
    }
  }
}

template <int DT, int K, int QM, int GP>
__global__ void __launch_bounds__(kChainThreads, 1) chain_persistent_kernel(
    const frt_chain_layer* __restrict__ layers, int n_layers, int steps, uint4* residual,
    const float* __restrict__ cos_tab, const float* __restrict__ sin_tab, const int32_t* __restrict__ positions,
    const float* __restrict__ scales, int32_t* status, int C, int NB, int Hq, int Hkv, int hd, int G, int I4,
    int NBI, int max_pos, int capacity, float eps, int act) {
  __shared__ double red[kChainWarps];
  pdl_enter();
  const int t = threadIdx.x;
  const int64_t row = blockIdx.x;
  uint4 hv[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = t + k * kChainThreads;
    hv[k] = c < C ? residual[row * C + c] : make_uint4(0u, 0u, 0u, 0u);
  }
  const int p = __ldg(positions + row);
  const bool row_ok = p >= 0 && p < max_pos && p < capacity;
  if (!row_ok && t == 0 && status != nullptr) atomicOr(status, 1);
  // this lane's cos / sin slice of the token's position (op b)
  constexpr int P = 8;
  const int li = t & (GP - 1);
  const int half = hd >> 1;
  float cs[P], sn[P];
  if (row_ok && li < G) {
#pragma unroll
    for (int e = 0; e < P; e += 4) {
      const float4 tc = __ldg(reinterpret_cast<const float4*>(cos_tab + (int64_t)p * half + li * P + e));
      const float4 ts = __ldg(reinterpret_cast<const float4*>(sin_tab + (int64_t)p * half + li * P + e));
      cs[e] = tc.x, cs[e + 1] = tc.y, cs[e + 2] = tc.z, cs[e + 3] = tc.w;
      sn[e] = ts.x, sn[e + 1] = ts.y, sn[e + 2] = ts.z, sn[e + 3] = ts.w;
    }
  }
  const Divisor dv_attn(QM == FRT_QUANT_STATIC ? __ldg(scales) : 1.0f);
  const Divisor dv_ffn(QM == FRT_QUANT_STATIC ? __ldg(scales + 1) : 1.0f);
  const Divisor dv_act(QM == FRT_QUANT_STATIC ? __ldg(scales + 2) : 1.0f);
  const float D = (float)(C * 8);
  for (int step = 0; step < steps; ++step) {
    for (int l = 0; l < n_layers; ++l) {
      const frt_chain_layer& L = layers[l];
      chain_norm<DT, K, QM>(static_cast<const uint4*>(L.x_attn), static_cast<const uint4*>(L.w_attn),
                            reinterpret_cast<uint2*>(L.q8_attn), L.bs_attn, dv_attn, hv, row, C, NB, D, eps, red);
      chain_qkv<DT, GP>(static_cast<const uint16_t*>(L.qkv), static_cast<const uint16_t*>(L.q_norm_w),
                        static_cast<const uint16_t*>(L.k_norm_w), static_cast<uint16_t*>(L.q_out),
                        static_cast<uint16_t*>(L.k_cache), static_cast<uint16_t*>(L.v_cache), cs, sn, row, p, row_ok,
                        Hq, Hkv, hd, G, eps);
      chain_norm<DT, K, QM>(static_cast<const uint4*>(L.x_ffn), static_cast<const uint4*>(L.w_ffn),
                            reinterpret_cast<uint2*>(L.q8_ffn), L.bs_ffn, dv_ffn, hv, row, C, NB, D, eps, red);
      chain_act<DT, QM>(static_cast<const uint4*>(L.gate_up), reinterpret_cast<uint32_t*>(L.act8), L.bs_act, dv_act,
                        row, I4, NBI, act);
    }
  }
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int c = t + k * kChainThreads;
    if (c < C) residual[row * C + c] = hv[k];
  }
}

struct ChainArgs {
  const frt_chain_layer* layers;
  int n_layers, steps;
  void* residual;
  const float *cos_tab, *sin_tab;
  const int32_t* positions;
  const float* scales;
  int32_t* status;
  int M, C, NB, Hq, Hkv, hd, G, I4, NBI, max_pos, capacity;
  float eps;
  int act;
};

template <int DT, int K, int QM, int GP>
frt_status launch_chain(const ChainArgs& a, cudaStream_t st) {
  return launch(chain_persistent_kernel<DT, K, QM, GP>, dim3(a.M), dim3(kChainThreads), 0, st, a.layers, a.n_layers,
                a.steps, static_cast<uint4*>(a.residual), a.cos_tab, a.sin_tab, a.positions, a.scales, a.status, a.C,
                a.NB, a.Hq, a.Hkv, a.hd, a.G, a.I4, a.NBI, a.max_pos, a.capacity, a.eps, a.act);
}

template <int DT, int K, int QM>
frt_status chain_gp_dispatch(int GP, const ChainArgs& a, cudaStream_t st) {
  switch (GP) {
    case 1: return launch_chain<DT, K, QM, 1>(a, st);
    case 2: return launch_chain<DT, K, QM, 2>(a, st);
    case 4: return launch_chain<DT, K, QM, 4>(a, st);
    case 8: return launch_chain<DT, K, QM, 8>(a, st);
    default: return launch_chain<DT, K, QM, 16>(a, st);
  }
}

template <int DT>
frt_status chain_dispatch(int K, frt_quant qm, int GP, const ChainArgs& a, cudaStream_t st) {
  const bool blk = qm == FRT_QUANT_BLOCK128;
  switch (K) {
    case 1:
      return blk ? chain_gp_dispatch<DT, 1, FRT_QUANT_BLOCK128>(GP, a, st)
                 : chain_gp_dispatch<DT, 1, FRT_QUANT_STATIC>(GP, a, st);
    case 2:
      return blk ? chain_gp_dispatch<DT, 2, FRT_QUANT_BLOCK128>(GP, a, st)
                 : chain_gp_dispatch<DT, 2, FRT_QUANT_STATIC>(GP, a, st);
    default:
      return blk ? chain_gp_dispatch<DT, 4, FRT_QUANT_BLOCK128>(GP, a, st)
                 : chain_gp_dispatch<DT, 4, FRT_QUANT_STATIC>(GP, a, st);
  }
}

}  // namespace
}  // namespace frt

extern "C" frt_status frt_chain_persistent(const frt_chain_layer* layers, int n_layers, int steps, void* residual,
                                           const float* cos_tab, const float* sin_tab, const int32_t* positions,
                                           const float* scales, int32_t* status, int M, int D, int Hq, int Hkv, int hd,
                                           int I, int max_pos, int capacity, float eps, frt_dtype dt, frt_quant qm,
                                           frt_act act, cudaStream_t stream) {
  using namespace frt;
  if (M < 0 || n_layers < 0 || steps < 0 || D <= 0 || D % 8 != 0 || I <= 0) return FRT_ERR_INVALID_ARG;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || hd <= 0 || hd % 2 != 0 || max_pos <= 0 || capacity <= 0)
    return FRT_ERR_INVALID_ARG;
  if (!valid_dtype(dt) || !valid_quant(qm)) return FRT_ERR_INVALID_ARG;
  if (act != FRT_ACT_GELU_TANH && act != FRT_ACT_SILU && act != FRT_ACT_RELU2) return FRT_ERR_INVALID_ARG;
  // supported shapes: D <= 4 * 256 * 8, 16-byte head halves (hd % 16 == 0, hd <= 256),
  // whole 128-output blocks in the activation
  if (D > 8192 || hd % 16 != 0 || hd > 256 || I % 128 != 0) return FRT_ERR_UNSUPPORTED;
  if (M == 0 || n_layers == 0 || steps == 0) return FRT_OK;
  if (!layers || !residual || !cos_tab || !sin_tab || !positions || !scales) return FRT_ERR_INVALID_ARG;
  if (!aligned(layers, 8) || !aligned(residual, 16) || !aligned(cos_tab, 16) || !aligned(sin_tab, 16) ||
      !aligned(positions, 4) || !aligned(scales, 4) || (status && !aligned(status, 4)))
    return FRT_ERR_INVALID_ARG;
  const int C = D / 8;
  const int K = C <= 256 ? 1 : C <= 512 ? 2 : 4;
  const int G = (hd / 2) / 8;
  int GP = 1;
  while (GP < G) GP *= 2;
  const ChainArgs a{layers, n_layers, steps, residual, cos_tab, sin_tab, positions, scales, status, M, C,
                    (D + 127) / 128, Hq, Hkv, hd, G, I / 4, I / 128, max_pos, capacity, eps, (int)act};
  return dt == FRT_F16 ? chain_dispatch<FRT_F16>(K, qm, GP, a, stream) : chain_dispatch<FRT_BF16>(K, qm, GP, a, stream);
}
