// Op (b): packed-QKV split + per-head q/k RMSNorm + rotate-half RoPE + Q staging
// write + KV-cache write, one pass over the QKV GEMM output.
//
// "FlashRT kernel fusion", §2.2 first bullet: q_norm -> RoPE -> write Q staging
// and k_norm -> RoPE -> write KV cache in one kernel, V passing straight
// through (replacing ~16 small ops per layer); second bullet: the rotate_half
// pair (j, j + hd/2) is kept in one lane, so RoPE needs no warp shuffle; §二
// step 3: split + RoPE + KV write with no q/k norm.
//
// Mapping (B200): a group of GP lanes (power of two) owns one (token, head)
// unit; lane l holds elements [lP, lP+P) and their RoPE partners
// [hd/2 + lP, ...), P = 8 (16-byte vectors) when hd % 16 == 0, else P = 4
// (8-byte vectors; e.g. the unpadded head_dim 72 of the ViT).  The per-head
// sum of squares is an xor shuffle inside the group.  A CTA holds one token's
// heads (all of them when heads x GP <= 1024), so the token's position and
// cos/sin row are read once into L1 and shared by every head, and no thread
// divides by the head count.
#include <cmath>

#include "frt_device.cuh"
#include "frt_host.h"

namespace frt {
namespace {

template <int P>
struct Vec16;
template <>
struct Vec16<8> {
  using T = uint4;
};
template <>
struct Vec16<4> {
  using T = uint2;
};

template <int P>
__device__ __forceinline__ typename Vec16<P>::T ld_vec(const uint16_t* p) {
  return *reinterpret_cast<const typename Vec16<P>::T*>(p);
}

template <int DT, int P>
__device__ __forceinline__ void unpack(const typename Vec16<P>::T& v, float* f) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
  for (int e = 0; e < P / 2; ++e) {
    const float2 t = Pack16<DT>::to_float2(w[e]);
    f[2 * e] = t.x;
    f[2 * e + 1] = t.y;
  }
}

template <int DT, int P>
__device__ __forceinline__ void store_packed(uint16_t* dst, const float* f) {
  typename Vec16<P>::T v;
  uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
  for (int e = 0; e < P / 2; ++e) w[e] = Pack16<DT>::from_float2(f[2 * e], f[2 * e + 1]);
  *reinterpret_cast<typename Vec16<P>::T*>(dst) = v;
}

template <int P>
__device__ __forceinline__ void ld_f32(const float* p, float* f) {
#pragma unroll
  for (int e = 0; e < P; e += 4) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(p + e));
    f[e] = t.x;
    f[e + 1] = t.y;
    f[e + 2] = t.z;
    f[e + 3] = t.w;
  }
}

template <int DT, int P, int GP>
__global__ void __launch_bounds__(1024) qkv_norm_rope_kvcache_kernel(
    const uint16_t* __restrict__ qkv, const uint16_t* __restrict__ q_norm_w,
    const uint16_t* __restrict__ k_norm_w, const float* __restrict__ cos_tab, const float* __restrict__ sin_tab,
    const int32_t* __restrict__ positions, uint16_t* __restrict__ q_out, uint16_t* __restrict__ k_cache,
    uint16_t* __restrict__ v_cache, int32_t* status, int H, int HB, int nhb, int Hq, int Hkv, int hd, int G,
    int max_pos, int capacity, float eps) {
  pdl_enter();
  // CTA = (token, group of HB heads); GP lanes per head.
  const int tok = blockIdx.x / nhb;
  const int h = (blockIdx.x - tok * nhb) * HB + (int)(threadIdx.x / GP);
  const int li = threadIdx.x & (GP - 1);
  const bool in_range = threadIdx.x < (unsigned)(HB * GP) && h < H;

  const int p = __ldg(positions + tok);
  const bool row_ok = p >= 0 && p < max_pos && p < capacity;
  if (!row_ok && threadIdx.x == 0 && blockIdx.x == tok * nhb && status != nullptr) atomicOr(status, 1);
  const bool active = in_range && row_ok && li < G;
  const int half = hd >> 1;
  const int j0 = li * P;
  const bool is_q = h < Hq;
  const bool is_v = h >= Hq + Hkv;
  const uint16_t* nw = is_q ? q_norm_w : k_norm_w;
  const bool do_norm = !is_v && nw != nullptr;

  // Issue the QKV loads first and prefetch the token's cos/sin slice into L1
  // (no registers held), so the table's latency overlaps the QKV loads and
  // the per-head reduction; the table is read after the reduction.
  const uint16_t* src = qkv + ((int64_t)tok * H + h) * hd;
  const float* crow = cos_tab + (int64_t)p * half + j0;
  const float* srow = sin_tab + (int64_t)p * half + j0;
  typename Vec16<P>::T va, vb;
  if (active) {
    va = *reinterpret_cast<const typename Vec16<P>::T*>(src + j0);
    vb = *reinterpret_cast<const typename Vec16<P>::T*>(src + half + j0);
    if (!is_v) {
      asm volatile("prefetch.global.L1 [%0];" ::"l"(crow));
      asm volatile("prefetch.global.L1 [%0];" ::"l"(srow));
    }
  }

  if (is_v) {  // V: bit copy into the cache slot
    if (active) {
      uint16_t* dst = v_cache + ((int64_t)p * Hkv + (h - Hq - Hkv)) * hd;
      *reinterpret_cast<typename Vec16<P>::T*>(dst + j0) = va;
      *reinterpret_cast<typename Vec16<P>::T*>(dst + half + j0) = vb;
    }
  }

  float a[P], b[P];
  float ss = 0.0f;
  if (active && !is_v) {
    unpack<DT, P>(va, a);
    unpack<DT, P>(vb, b);
    if (do_norm) {
#pragma unroll
      for (int e = 0; e < P; ++e) ss = fmaf(b[e], b[e], fmaf(a[e], a[e], ss));
    }
  }
  ss = group_sum<GP>(ss);  // every lane of the warp takes part

  if (active && !is_v) {
    if (do_norm) {
      const float rstd = 1.0f / sqrtf(ss / (float)hd + eps);
      float fa[P], fb[P];
      unpack<DT, P>(ld_vec<P>(nw + j0), fa);
      unpack<DT, P>(ld_vec<P>(nw + half + j0), fb);
#pragma unroll
      for (int e = 0; e < P; ++e) {
        a[e] = a[e] * rstd * fa[e];
        b[e] = b[e] * rstd * fb[e];
      }
    }
    float c[P], s[P];
    ld_f32<P>(crow, c);
    ld_f32<P>(srow, s);
    float o1[P], o2[P];
#pragma unroll
    for (int e = 0; e < P; ++e) {
      o1[e] = fmaf(a[e], c[e], -(b[e] * s[e]));
      o2[e] = fmaf(b[e], c[e], a[e] * s[e]);
    }
    uint16_t* dst = is_q ? q_out + ((int64_t)tok * Hq + h) * hd
                         : k_cache + ((int64_t)p * Hkv + (h - Hq)) * hd;
    store_packed<DT, P>(dst + j0, o1);
    store_packed<DT, P>(dst + half + j0, o2);
  }
}

struct Args {
  const void* qkv;
  const void* qw;
  const void* kw;
  const float* cos_tab;
  const float* sin_tab;
  const int32_t* pos;
  void* q_out;
  void* kc;
  void* vc;
  int32_t* status;
  int M, H, Hq, Hkv, hd, G, max_pos, capacity;
  float eps;
};

// One CTA per (token, group of HB heads): HB = all heads when H * GP <= 1024.
template <int DT, int P, int GP>
frt_status launch_gp(const Args& a, cudaStream_t st) {
  const int HB = a.H * GP <= 1024 ? a.H : 1024 / GP;
  const int nhb = (a.H + HB - 1) / HB;
  const int threads = ((HB * GP + 31) / 32) * 32;
  const dim3 grid((unsigned)((int64_t)a.M * nhb));
  return launch(qkv_norm_rope_kvcache_kernel<DT, P, GP>, grid, dim3(threads), 0, st,
                static_cast<const uint16_t*>(a.qkv), static_cast<const uint16_t*>(a.qw),
                static_cast<const uint16_t*>(a.kw), a.cos_tab, a.sin_tab, a.pos, static_cast<uint16_t*>(a.q_out),
                static_cast<uint16_t*>(a.kc), static_cast<uint16_t*>(a.vc), a.status, a.H, HB, nhb, a.Hq, a.Hkv,
                a.hd, a.G, a.max_pos, a.capacity, a.eps);
}

template <int DT, int P>
frt_status launch_p(int GP, const Args& a, cudaStream_t st) {
  switch (GP) {
    case 1: return launch_gp<DT, P, 1>(a, st);
    case 2: return launch_gp<DT, P, 2>(a, st);
    case 4: return launch_gp<DT, P, 4>(a, st);
    case 8: return launch_gp<DT, P, 8>(a, st);
    case 16: return launch_gp<DT, P, 16>(a, st);
    default: return launch_gp<DT, P, 32>(a, st);
  }
}

template <int DT>
frt_status launch_dt(int P, int GP, const Args& a, cudaStream_t st) {
  return P == 8 ? launch_p<DT, 8>(GP, a, st) : launch_p<DT, 4>(GP, a, st);
}

}  // namespace
}  // namespace frt

extern "C" frt_status frt_qkv_norm_rope_kvcache(const void* qkv, const void* q_norm_w, const void* k_norm_w,
                                                const float* cos_tab, const float* sin_tab,
                                                const int32_t* positions, void* q_out, void* k_cache,
                                                void* v_cache, int32_t* status, int M, int Hq, int Hkv, int hd,
                                                int max_pos, int capacity, float eps, frt_dtype dt,
                                                cudaStream_t stream) {
  using namespace frt;
  if (M < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || hd <= 0 || hd % 2 != 0) return FRT_ERR_INVALID_ARG;
  if (max_pos <= 0 || capacity <= 0 || !valid_dtype(dt)) return FRT_ERR_INVALID_ARG;
  if (hd % 8 != 0 || hd > 256) return FRT_ERR_UNSUPPORTED;
  if (M == 0) return FRT_OK;
  if (!qkv || !cos_tab || !sin_tab || !positions || !q_out || !k_cache || !v_cache) return FRT_ERR_INVALID_ARG;
  const int P = (hd % 16 == 0) ? 8 : 4;
  const uintptr_t al = (P == 8) ? 16 : 8;
  if (!aligned(qkv, al) || !aligned(q_out, al) || !aligned(k_cache, al) || !aligned(v_cache, al))
    return FRT_ERR_INVALID_ARG;
  if ((q_norm_w && !aligned(q_norm_w, al)) || (k_norm_w && !aligned(k_norm_w, al))) return FRT_ERR_INVALID_ARG;
  if (!aligned(cos_tab, 16) || !aligned(sin_tab, 16) || !aligned(positions, 4)) return FRT_ERR_INVALID_ARG;
  if (status && !aligned(status, 4)) return FRT_ERR_INVALID_ARG;
  const int H = Hq + 2 * Hkv;
  const int G = (hd / 2) / P;  // active lanes per head, <= 31
  int GP = 1;
  while (GP < G) GP *= 2;
  Args a{qkv, q_norm_w, k_norm_w, cos_tab, sin_tab, positions, q_out, k_cache, v_cache, status,
         M, H, Hq, Hkv, hd, G, max_pos, capacity, eps};
  const int64_t HB = (int64_t)H * GP <= 1024 ? H : 1024 / GP;
  if ((int64_t)M * ((H + HB - 1) / HB) > 0x7FFFFFFF) return FRT_ERR_UNSUPPORTED;
  return dt == FRT_F16 ? launch_dt<FRT_F16>(P, GP, a, stream) : launch_dt<FRT_BF16>(P, GP, a, stream);
}
