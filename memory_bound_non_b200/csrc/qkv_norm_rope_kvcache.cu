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
// heads (or a block of them), so the token's position and cos/sin row are
// read once per lane and shared by every head the lane handles; on large
// batches each lane group takes up to four heads to keep more bytes in flight.
#include <atomic>
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
__device__ __forceinline__ void store_pairs(uint16_t* dst, const float2* f) {
  typename Vec16<P>::T v;
  pack_pairs<DT, P / 2>(f, reinterpret_cast<uint32_t*>(&v));
  *reinterpret_cast<typename Vec16<P>::T*>(dst) = v;
}

template <int NP>
__device__ __forceinline__ void ld_pairs_smem(const float* p, float2* f) {
#pragma unroll
  for (int e = 0; e < NP; e += 2) {
    const float4 t = *reinterpret_cast<const float4*>(p + 2 * e);
    f[e] = make_float2(t.x, t.y);
    f[e + 1] = make_float2(t.z, t.w);
  }
}

// Epilogue of the op (NEXT-2, the attention's Q preparation folded in): Q is
// multiplied by q_scale in fp32 before its one rounding and written
// token-major [M, Hq, hd] or head-major [Hq, M, hd]; with KV8 the K and V
// cache rows are e4m3 codes of k / k_scale and v / v_scale (kv_scales[0..1],
// device), the quotient correctly rounded in fp32.
struct Epilogue {
  float q_scale;
  int q_head_major;
  int M;
  const float* kv_scales;
  const uint16_t* q_bias;  // LayerNorm level (EPI 3): per-head bias rows, or null
  const uint16_t* k_bias;
};

__device__ __forceinline__ int64_t q_row(const Epilogue& ep, int tok, int h, int Hq) {
  return ep.q_head_major ? (int64_t)h * ep.M + tok : (int64_t)tok * Hq + h;
}

// P fp32 values -> P e4m3 codes of v / s stored at dst (P bytes, P-aligned).
template <int P>
__device__ __forceinline__ void store_codes(uint8_t* dst, const float* v, const Divisor& dv) {
  if (P == 8)
    *reinterpret_cast<uint2*>(dst) = quant8(v, dv);
  else
    *reinterpret_cast<uint32_t*>(dst) = quant4(v, dv);
}

// P fp32 values already divided by the scale -> P e4m3 codes at dst.
template <int P>
__device__ __forceinline__ void store_codes_raw(uint8_t* dst, const float2* v) {
  const float* f = reinterpret_cast<const float*>(v);
  if (P == 8)
    *reinterpret_cast<uint2*>(dst) = e4m3x8(f);
  else
    *reinterpret_cast<uint32_t*>(dst) = e4m3x4(f[0], f[1], f[2], f[3]);
}

// One head's LayerNorm on a lane's packed pairs (NEXT-4): the mean, then the
// centred sum of squares (each an xor shuffle over the GP lanes of the group;
// every lane of the warp takes part), then x = (x - mean) * rstd * w + bias in
// place, the head's affine rows given as packed 16-bit words (null:
// identity).  `on` gates the lane's arithmetic, not the shuffles.
template <int DT, int NP, int GP>
__device__ __forceinline__ void ln_head(float2* a, float2* b, bool on, float inv_hd, float eps,
                                        const uint32_t* wa, const uint32_t* wb, const uint32_t* ba,
                                        const uint32_t* bb) {
  float2 acc = make_float2(0.0f, 0.0f);
  if (on) {
#pragma unroll
    for (int e = 0; e < NP; ++e) acc = __fadd2_rn(__fadd2_rn(acc, a[e]), b[e]);
  }
  const float mean = group_sum<GP>(acc.x + acc.y) * inv_hd;
  float2 acc2 = make_float2(0.0f, 0.0f);
  if (on) {
    const float2 nm = make_float2(-mean, -mean);
#pragma unroll
    for (int e = 0; e < NP; ++e) {
      a[e] = __fadd2_rn(a[e], nm);
      b[e] = __fadd2_rn(b[e], nm);
      acc2 = __ffma2_rn(b[e], b[e], __ffma2_rn(a[e], a[e], acc2));
    }
  }
  const float s2 = group_sum<GP>(acc2.x + acc2.y);
  if (!on) return;
  const float r = head_rstd(s2, inv_hd, eps);
  const float2 rr = make_float2(r, r);
#pragma unroll
  for (int e = 0; e < NP; ++e) {
    const float2 w1 = wa ? Pack16<DT>::to_float2(wa[e]) : make_float2(1.0f, 1.0f);
    const float2 w2 = wb ? Pack16<DT>::to_float2(wb[e]) : make_float2(1.0f, 1.0f);
    const float2 b1 = ba ? Pack16<DT>::to_float2(ba[e]) : make_float2(0.0f, 0.0f);
    const float2 b2 = bb ? Pack16<DT>::to_float2(bb[e]) : make_float2(0.0f, 0.0f);
    a[e] = __ffma2_rn(__fmul2_rn(a[e], rr), w1, b1);
    b[e] = __ffma2_rn(__fmul2_rn(b[e], rr), w2, b2);
  }
}

// Register kernel (small batches, or pointers below 16-byte alignment).  One
// CTA per (token, block of heads).  The CTA's NG lane groups take up to HPG
// heads each: slot i of group g is head (hb * hpg + i) * NG + g, so for every
// slot consecutive groups read consecutive heads.  All slots' loads are issued
// first and a lane's cos/sin slice is loaded once for all its heads.
// Threads per CTA of the register kernel: up to 1024 with one head per lane
// group, 512 when the e4m3 epilogue needs the registers, 256 with four heads.
template <int HPG, int EPI>
constexpr int reg_kernel_threads() {
  return HPG == 1 ? (EPI == 2 ? 512 : 1024) : 256;
}

template <int DT, int P, int GP, int HPG, int EPI>
__global__ void __launch_bounds__(reg_kernel_threads<HPG, EPI>()) qkv_norm_rope_kvcache_kernel(
    const uint16_t* __restrict__ qkv, const uint16_t* __restrict__ q_norm_w,
    const uint16_t* __restrict__ k_norm_w, const float* __restrict__ cos_tab, const float* __restrict__ sin_tab,
    const int32_t* __restrict__ positions, uint16_t* __restrict__ q_out, void* __restrict__ k_cache,
    void* __restrict__ v_cache, int32_t* status, int H, int NG, int hpg, int nhb, int Hq, int Hkv, int hd,
    int G, int max_pos, int capacity, float eps, Epilogue ep) {
  using V = typename Vec16<P>::T;
  constexpr bool QEPI = EPI >= 1;
  constexpr bool KV8 = EPI == 2;
  const int tok = blockIdx.x / nhb;
  const int hb = blockIdx.x - tok * nhb;
  const int grp = (int)(threadIdx.x / GP);
  const int li = threadIdx.x & (GP - 1);
  const bool lane_ok = threadIdx.x < (unsigned)(NG * GP) && li < G;
  const int half = hd >> 1;
  const int j0 = li * P;
  // Constant inputs before the wait for the previous kernel: the position,
  // the lane's cos/sin slice at that position (two dependent loads, off the
  // critical path this way), the norm weights and the e4m3 cache scales.
  const int64_t M = gridDim.x / nhb;  // extents for the bounds-checked build
  const int p = FRT_IDX_OK(tok, M) ? __ldg(positions + tok) : -1;
  const bool row_ok = p >= 0 && p < max_pos && p < capacity;
  const bool active = lane_ok && row_ok;
  constexpr int NP = P / 2;
  float2 cs[NP], sn[NP], nsn[NP];
  if (active && FRT_SPAN_OK((int64_t)p * half + j0, P, (int64_t)max_pos * half))
    load_rope_pairs<NP>(cos_tab + (int64_t)p * half + j0, sin_tab + (int64_t)p * half + j0, cs, sn, nsn);
  V qwa, qwb, kwa, kwb;
  if (HPG == 1 && lane_ok && FRT_SPAN_OK(j0, half + P, hd)) {
    if (q_norm_w != nullptr) {
      qwa = ld_vec<P>(q_norm_w + j0);
      qwb = ld_vec<P>(q_norm_w + half + j0);
    }
    if (k_norm_w != nullptr) {
      kwa = ld_vec<P>(k_norm_w + j0);
      kwb = ld_vec<P>(k_norm_w + half + j0);
    }
  }
  const float k_inv = KV8 && FRT_IDX_OK(0, 2) ? __frcp_rn(__ldg(ep.kv_scales)) : 1.0f;  // RN(1 / k_scale)
  const float v_scale = KV8 && FRT_IDX_OK(1, 2) ? __ldg(ep.kv_scales + 1) : 1.0f;
  pdl_enter();
  const uint16_t* row = qkv + (int64_t)tok * H * hd;
  const int64_t n_qkv = M * H * hd, n_q = M * Hq * hd, n_kv = (int64_t)capacity * Hkv * hd;
  V va[HPG], vb[HPG];
#pragma unroll
  for (int i = 0; i < HPG; ++i) {
    const int h = (hb * hpg + i) * NG + grp;
    if (lane_ok && i < hpg && h < H && FRT_SPAN_OK((int64_t)tok * H * hd + (int64_t)h * hd + j0, half + P, n_qkv)) {
      va[i] = *reinterpret_cast<const V*>(row + (int64_t)h * hd + j0);
      vb[i] = *reinterpret_cast<const V*>(row + (int64_t)h * hd + half + j0);
    }
  }
  if (!row_ok && threadIdx.x == 0 && hb == 0 && status != nullptr) atomicOr(status, 1);
  const float inv_hd = 1.0f / (float)hd;
#pragma unroll
  for (int i = 0; i < HPG; ++i) {
    if (i >= hpg) break;  // uniform across the CTA
    const int h = (hb * hpg + i) * NG + grp;
    const bool on = active && h < H;
    const bool is_q = h < Hq;
    const bool is_v = h >= Hq + Hkv;
    const uint16_t* nw = is_q ? q_norm_w : k_norm_w;
    const bool do_norm = !is_v && nw != nullptr;
    if (on && is_v && FRT_SPAN_OK(((int64_t)p * Hkv + (h - Hq - Hkv)) * hd + j0, half + P, n_kv)) {
      // V: bit copy into the cache slot (or its e4m3 codes)
      const int64_t off = ((int64_t)p * Hkv + (h - Hq - Hkv)) * hd;
      if (KV8) {
        float a[P], b[P];
        unpack<DT, P>(va[i], a);
        unpack<DT, P>(vb[i], b);
        uint8_t* dst = static_cast<uint8_t*>(v_cache) + off;
        const Divisor dvs(v_scale);
        store_codes<P>(dst + j0, a, dvs);
        store_codes<P>(dst + half + j0, b, dvs);
      } else {
        uint16_t* dst = static_cast<uint16_t*>(v_cache) + off;
        *reinterpret_cast<V*>(dst + j0) = va[i];
        *reinterpret_cast<V*>(dst + half + j0) = vb[i];
      }
    }
    float2 a[NP], b[NP];
    float ss = 0.0f;
    if (on && !is_v) {
      unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&va[i]), a);
      unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&vb[i]), b);
      if (do_norm) ss = sum_squares_pairs<NP>(a, b);
    }
    ss = group_sum<GP>(ss);  // every lane of the warp takes part
    if (on && !is_v) {
      // the Q epilogue's scale and, with e4m3 caches, RN(1 / k_scale) ride on
      // the head's norm factor (a product per element otherwise)
      const float post = (QEPI && is_q) ? ep.q_scale : (KV8 && !is_q) ? k_inv : 1.0f;
      if (!do_norm && ((QEPI && is_q) || (KV8 && !is_q))) {
        mul_pairs<NP>(a, post);
        mul_pairs<NP>(b, post);
      }
      if (do_norm) {
        const float rstd = head_rstd(ss, inv_hd, eps) * post;
        float2 fa[NP], fb[NP];
        if (HPG == 1) {  // weights already in registers
          const V wa = is_q ? qwa : kwa, wb = is_q ? qwb : kwb;
          unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&wa), fa);
          unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&wb), fb);
        } else {
          V wa, wb;
          if (FRT_SPAN_OK(j0, half + P, hd)) {
            wa = ld_vec<P>(nw + j0);
            wb = ld_vec<P>(nw + half + j0);
          }
          unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&wa), fa);
          unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&wb), fb);
        }
        scale_pairs<NP>(a, rstd, fa);
        scale_pairs<NP>(b, rstd, fb);
      }
      float2 o1[NP], o2[NP];
      rope_pairs<NP>(a, b, cs, sn, nsn, o1, o2);
      if (is_q) {
        const int64_t qo = (QEPI ? q_row(ep, tok, h, Hq) : (int64_t)tok * Hq + h) * hd;
        uint16_t* dst = q_out + qo;
        if (FRT_SPAN_OK(qo + j0, half + P, n_q)) {
          store_pairs<DT, P>(dst + j0, o1);
          store_pairs<DT, P>(dst + half + j0, o2);
        }
      } else if (FRT_SPAN_OK(((int64_t)p * Hkv + (h - Hq)) * hd + j0, half + P, n_kv)) {
        const int64_t off = ((int64_t)p * Hkv + (h - Hq)) * hd;
        if (KV8) {  // already divided by k_scale
          uint8_t* dst = static_cast<uint8_t*>(k_cache) + off;
          store_codes_raw<P>(dst + j0, o1);
          store_codes_raw<P>(dst + half + j0, o2);
        } else {
          uint16_t* dst = static_cast<uint16_t*>(k_cache) + off;
          store_pairs<DT, P>(dst + j0, o1);
          store_pairs<DT, P>(dst + half + j0, o2);
        }
      }
    }
  }
}

// One token's heads, in shared memory, for the bulk-copy kernels: lane groups
// normalise and rotate the Q and K heads in place (Q scaled, head-major Q
// straight to global memory; e4m3 codes of K and V into their own rows with
// EPI 2).  The caller orders these writes before its bulk stores.
template <int DT, int P, int GP, int EPI>
__device__ __forceinline__ void process_token(uint16_t* rowbuf, const float* cbuf, const float* sbuf,
                                              const float* kvs, const uint16_t* qwbuf, const uint16_t* kwbuf, uint8_t* k8buf,
                                              uint8_t* v8buf, const uint16_t* q_norm_w, const uint16_t* k_norm_w,
                                              uint16_t* q_out, int tok, int tid, int H, int NG, int Hq, int Hkv,
                                              int hd, int G, float eps, const Epilogue& ep) {
  using V = typename Vec16<P>::T;
  constexpr bool QEPI = EPI == 1 || EPI == 2;
  constexpr bool KV8 = EPI == 2;
  constexpr bool LN = EPI == 3;
  const int half = hd >> 1;
  const int grp = tid / GP;
  const int li = tid & (GP - 1);
  const bool lane_ok = grp < NG && li < G;
  const int j0 = li * P;
  constexpr int NP = P / 2;
  const float inv_hd = 1.0f / (float)hd;
  const bool q_direct = QEPI && ep.q_head_major;  // head-major Q leaves from registers
  // Q and K heads; V heads too with KV8 (their codes), else V leaves untouched.
  const int nheads = KV8 ? H : Hq + Hkv;
  const int nslots = (nheads + NG - 1) / NG;
  for (int i = 0; i < nslots; ++i) {
    const int h = i * NG + grp;
    const bool on = lane_ok && h < nheads;
    const bool is_q = h < Hq;
    const bool is_v = h >= Hq + Hkv;
    const uint16_t* nwg = is_v ? nullptr : is_q ? q_norm_w : k_norm_w;
    const uint16_t* nws = is_q ? qwbuf : kwbuf;
    uint16_t* vec = rowbuf + h * hd;
    if (LN) {
      // per-head LayerNorm with the head's affine rows (global memory, each
      // optional), then RoPE in place
      float2 x1[NP], x2[NP];
      if (on) {
        const V va = *reinterpret_cast<const V*>(vec + j0), vb = *reinterpret_cast<const V*>(vec + half + j0);
        unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&va), x1);
        unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&vb), x2);
      }
      const int64_t off = (int64_t)(is_q ? h : h - Hq) * hd;
      const uint16_t* pw = is_q ? q_norm_w : k_norm_w;
      const uint16_t* pb = is_q ? ep.q_bias : ep.k_bias;
      V wa, wb, ba, bb;
      const int64_t n_aff = (int64_t)(is_q ? Hq : Hkv) * hd;  // per-head affine rows [Hq | Hkv, hd]
      if (on && pw != nullptr && FRT_SPAN_OK(off + j0, half + P, n_aff)) {
        wa = ld_vec<P>(pw + off + j0);
        wb = ld_vec<P>(pw + off + half + j0);
      }
      if (on && pb != nullptr && FRT_SPAN_OK(off + j0, half + P, n_aff)) {
        ba = ld_vec<P>(pb + off + j0);
        bb = ld_vec<P>(pb + off + half + j0);
      }
      ln_head<DT, NP, GP>(x1, x2, on, inv_hd, eps, pw ? reinterpret_cast<const uint32_t*>(&wa) : nullptr,
                          pw ? reinterpret_cast<const uint32_t*>(&wb) : nullptr,
                          pb ? reinterpret_cast<const uint32_t*>(&ba) : nullptr,
                          pb ? reinterpret_cast<const uint32_t*>(&bb) : nullptr);
      if (on) {
        float2 o1[NP], o2[NP];
#pragma unroll
        for (int e = 0; e < NP; e += 2) {
          float2 cs[2], sn[2], nsn[2];
          ld_pairs_smem<2>(cbuf + j0 + 2 * e, cs);
          ld_pairs_smem<2>(sbuf + j0 + 2 * e, sn);
          nsn[0] = make_float2(-sn[0].x, -sn[0].y);
          nsn[1] = make_float2(-sn[1].x, -sn[1].y);
          rope_pairs<2>(x1 + e, x2 + e, cs, sn, nsn, o1 + e, o2 + e);
        }
        store_pairs<DT, P>(vec + j0, o1);
        store_pairs<DT, P>(vec + half + j0, o2);
      }
      continue;
    }
    float2 x1[NP], x2[NP];
    float ss = 0.0f;
    if (on) {
      const V va = *reinterpret_cast<const V*>(vec + j0), vb = *reinterpret_cast<const V*>(vec + half + j0);
      unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&va), x1);
      unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&vb), x2);
      if (nwg != nullptr) ss = sum_squares_pairs<NP>(x1, x2);
    }
    ss = group_sum<GP>(ss);  // every lane of the warp takes part
    if (on && KV8 && is_v) {
      uint8_t* dst = v8buf + (h - Hq - Hkv) * hd;
      const Divisor dvs(kvs[2], kvs[3]);
      store_codes<P>(dst + j0, reinterpret_cast<const float*>(x1), dvs);
      store_codes<P>(dst + half + j0, reinterpret_cast<const float*>(x2), dvs);
    } else if (on) {
      // the Q epilogue's scale and, with e4m3 caches, RN(1 / k_scale) ride on
      // the head's norm factor (a product per element otherwise)
      const float post = (QEPI && is_q) ? ep.q_scale : (KV8 && !is_q) ? kvs[1] : 1.0f;
      if (nwg != nullptr) {
        const float rstd = head_rstd(ss, inv_hd, eps) * post;
        const V wa = *reinterpret_cast<const V*>(nws + j0), wb = *reinterpret_cast<const V*>(nws + half + j0);
        float2 fa[NP], fb[NP];
        unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&wa), fa);
        unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&wb), fb);
        scale_pairs<NP>(x1, rstd, fa);
        scale_pairs<NP>(x2, rstd, fb);
      } else if ((QEPI && is_q) || (KV8 && !is_q)) {
        mul_pairs<NP>(x1, post);
        mul_pairs<NP>(x2, post);
      }
      // this slot's cos and sin slices from shared memory (-sin negated here)
      float2 cs[NP], sn[NP], nsn[NP];
      ld_pairs_smem<NP>(cbuf + j0, cs);
      ld_pairs_smem<NP>(sbuf + j0, sn);
#pragma unroll
      for (int e = 0; e < NP; ++e) nsn[e] = make_float2(-sn[e].x, -sn[e].y);
      float2 o1[NP], o2[NP];
      rope_pairs<NP>(x1, x2, cs, sn, nsn, o1, o2);
      if (KV8 && !is_q) {  // already divided by k_scale
        uint8_t* dst = k8buf + (h - Hq) * hd;
        store_codes_raw<P>(dst + j0, o1);
        store_codes_raw<P>(dst + half + j0, o2);
      } else if (q_direct && is_q) {
        uint16_t* dst = q_out + ((int64_t)h * ep.M + tok) * hd;
        if (FRT_SPAN_OK(((int64_t)h * ep.M + tok) * hd + j0, half + P, (int64_t)Hq * ep.M * hd)) {
          store_pairs<DT, P>(dst + j0, o1);
          store_pairs<DT, P>(dst + half + j0, o2);
        }
      } else {
        store_pairs<DT, P>(vec + j0, o1);
        store_pairs<DT, P>(vec + half + j0, o2);
      }
    }
  }
}

// One token's outputs leave shared memory as bulk stores (issued by one
// thread; the caller commits and waits): token-major Q as one row (head-major
// Q went straight from registers), the K and V cache rows at slot p.
template <int EPI>
__device__ __forceinline__ void store_token(const uint16_t* rowbuf, const uint8_t* k8buf, const uint8_t* v8buf,
                                            uint16_t* q_out, void* k_cache, void* v_cache, int tok, int p, int Hq,
                                            int Hkv, int hd, int capacity, const Epilogue& ep) {
  const int64_t n_kv = (int64_t)capacity * Hkv * hd;
  if (!((EPI == 1 || EPI == 2) && ep.q_head_major) &&
      FRT_SPAN_OK((int64_t)tok * Hq * hd, Hq * hd, (int64_t)ep.M * Hq * hd))
    bulk_store(q_out + (int64_t)tok * Hq * hd, rowbuf, (unsigned)(Hq * hd * 2));
  if (!FRT_SPAN_OK((int64_t)p * Hkv * hd, Hkv * hd, n_kv)) return;
  if (EPI == 2) {
    bulk_store(static_cast<uint8_t*>(k_cache) + (int64_t)p * Hkv * hd, k8buf, (unsigned)(Hkv * hd));
    bulk_store(static_cast<uint8_t*>(v_cache) + (int64_t)p * Hkv * hd, v8buf, (unsigned)(Hkv * hd));
  } else {
    bulk_store(static_cast<uint16_t*>(k_cache) + (int64_t)p * Hkv * hd, rowbuf + Hq * hd, (unsigned)(Hkv * hd * 2));
    bulk_store(static_cast<uint16_t*>(v_cache) + (int64_t)p * Hkv * hd, rowbuf + (Hq + Hkv) * hd,
               (unsigned)(Hkv * hd * 2));
  }
}

// NEXT-4: per-head LayerNorm on Q and K + rotate-half RoPE + Q staging + KV
// write ("FlashRT kernel fusion", §2.2 second bullet: the Chameleon prefill
// kernel, LayerNorm(Q) + LayerNorm(K) + two rotate_half RoPE in one kernel
// with each rotation pair kept in one lane).  Lane groups of GP lanes take up
// to HPG heads of one token each (slot i of group g is head
// (hb * HPG + i) * NG + g); all QKV loads and the cos/sin slice are issued
// first.  Per head the mean and the centred sum of squares are two
// xor-shuffle reductions inside the group, then y = (v - mean) * rstd * w_h +
// b_h with per-head affine rows (each optional, read from L2).
template <int DT, int P, int GP, int HPG>
__global__ void __launch_bounds__(HPG == 1 ? 512 : 256) qkv_layernorm_rope_kvcache_kernel(
    const uint16_t* __restrict__ qkv, const uint16_t* __restrict__ q_w, const uint16_t* __restrict__ q_b,
    const uint16_t* __restrict__ k_w, const uint16_t* __restrict__ k_b, const float* __restrict__ cos_tab,
    const float* __restrict__ sin_tab, const int32_t* __restrict__ positions, uint16_t* __restrict__ q_out,
    uint16_t* __restrict__ k_cache, uint16_t* __restrict__ v_cache, int32_t* status, int H, int NG, int nhb, int Hq,
    int Hkv, int hd, int G, int max_pos, int capacity, float eps) {
  using V = typename Vec16<P>::T;
  const int tok = blockIdx.x / nhb;
  const int hb = blockIdx.x - tok * nhb;
  const int grp = (int)(threadIdx.x / GP);
  const int li = threadIdx.x & (GP - 1);
  const int half = hd >> 1;
  const int j0 = li * P;
  const bool lane_ok = threadIdx.x < (unsigned)(NG * GP) && li < G;
  // the position and the lane's cos/sin slice are constant inputs: read
  // before the wait for the previous kernel
  const int64_t M = gridDim.x / nhb;  // extents for the bounds-checked build
  const int p = FRT_IDX_OK(tok, M) ? __ldg(positions + tok) : -1;
  const bool row_ok = p >= 0 && p < max_pos && p < capacity;
  const bool active = lane_ok && row_ok;
  constexpr int NP = P / 2;
  float2 cs[NP], sn[NP], nsn[NP];
  if (active && FRT_SPAN_OK((int64_t)p * half + j0, P, (int64_t)max_pos * half))
    load_rope_pairs<NP>(cos_tab + (int64_t)p * half + j0, sin_tab + (int64_t)p * half + j0, cs, sn, nsn);
  pdl_enter();
  const uint16_t* row = qkv + (int64_t)tok * H * hd;
  const int64_t n_kv = (int64_t)capacity * Hkv * hd;
  V va[HPG], vb[HPG];
#pragma unroll
  for (int i = 0; i < HPG; ++i) {
    const int h = (hb * HPG + i) * NG + grp;
    if (lane_ok && h < H && FRT_SPAN_OK((int64_t)tok * H * hd + (int64_t)h * hd + j0, half + P, M * H * hd)) {
      va[i] = *reinterpret_cast<const V*>(row + (int64_t)h * hd + j0);
      vb[i] = *reinterpret_cast<const V*>(row + (int64_t)h * hd + half + j0);
    }
  }
  if (!row_ok && threadIdx.x == 0 && hb == 0 && status != nullptr) atomicOr(status, 1);
  const float inv_hd = 1.0f / (float)hd;
#pragma unroll
  for (int i = 0; i < HPG; ++i) {
    const int h = (hb * HPG + i) * NG + grp;
    const bool on = active && h < H;
    const bool is_q = h < Hq;
    const bool is_v = h >= Hq + Hkv;
    if (on && is_v && FRT_SPAN_OK(((int64_t)p * Hkv + (h - Hq - Hkv)) * hd + j0, half + P, n_kv)) {
      // V: bit copy into the cache slot
      uint16_t* dst = v_cache + ((int64_t)p * Hkv + (h - Hq - Hkv)) * hd;
      *reinterpret_cast<V*>(dst + j0) = va[i];
      *reinterpret_cast<V*>(dst + half + j0) = vb[i];
    }
    const bool qk = on && !is_v;
    float2 a[NP], b[NP];
    if (qk) {
      unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&va[i]), a);
      unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&vb[i]), b);
    }
    const int hh = is_q ? h : h - Hq;
    const uint16_t* pw = is_q ? q_w : k_w;
    const uint16_t* pb = is_q ? q_b : k_b;
    V wa, wb, ba, bb;
    const int64_t n_aff = (int64_t)(is_q ? Hq : Hkv) * hd;  // per-head affine rows
    if (qk && pw != nullptr && FRT_SPAN_OK((int64_t)hh * hd + j0, half + P, n_aff)) {
      wa = ld_vec<P>(pw + (int64_t)hh * hd + j0);
      wb = ld_vec<P>(pw + (int64_t)hh * hd + half + j0);
    }
    if (qk && pb != nullptr && FRT_SPAN_OK((int64_t)hh * hd + j0, half + P, n_aff)) {
      ba = ld_vec<P>(pb + (int64_t)hh * hd + j0);
      bb = ld_vec<P>(pb + (int64_t)hh * hd + half + j0);
    }
    ln_head<DT, NP, GP>(a, b, qk, inv_hd, eps, pw ? reinterpret_cast<const uint32_t*>(&wa) : nullptr,
                        pw ? reinterpret_cast<const uint32_t*>(&wb) : nullptr,
                        pb ? reinterpret_cast<const uint32_t*>(&ba) : nullptr,
                        pb ? reinterpret_cast<const uint32_t*>(&bb) : nullptr);
    if (qk) {
      float2 o1[NP], o2[NP];
      rope_pairs<NP>(a, b, cs, sn, nsn, o1, o2);
      const int64_t o = is_q ? ((int64_t)tok * Hq + h) * hd : ((int64_t)p * Hkv + hh) * hd;
      uint16_t* dst = (is_q ? q_out : k_cache) + o;
      if (FRT_SPAN_OK(o + j0, half + P, is_q ? M * Hq * hd : n_kv)) {
        store_pairs<DT, P>(dst + j0, o1);
        store_pairs<DT, P>(dst + half + j0, o2);
      }
    }
  }
}

// Any even head_dim (hd % 8 != 0, e.g. 66 or 100, where no vector width fits
// both halves of a head): one warp per (token, head) slot, lane l holding the
// elements j = l, l + 32, ... (< hd/2) and their rotate-half partners
// j + hd/2, read and written as single 16-bit elements (a 64-byte run per
// warp access).  The arithmetic is the vector kernels', element by element:
// the head's sum of squares (or mean and centred squares for LayerNorm) is a
// warp reduction, then norm, RoPE, the Q epilogue and the cache stores.
// EPI as the bulk-copy kernel (0 op (b), 1 Q epilogue, 2 + e4m3 caches, 3
// per-head LayerNorm with affine rows [H, hd] and biases in ep).
constexpr int kGenericMaxK = 4;  // hd / 2 <= 128 = 32 lanes x 4

template <int DT>
__device__ __forceinline__ float ld16(const uint16_t* p) {
  const uint32_t u = *p;
  return DT == FRT_BF16 ? __uint_as_float(u << 16) : __half2float(__ushort_as_half((unsigned short)u));
}
template <int DT>
__device__ __forceinline__ void st16(uint16_t* p, float v) {
  if (DT == FRT_BF16)
    *p = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  else
    *p = __half_as_ushort(__float2half_rn(v));
}

template <int DT, int EPI>
__global__ void __launch_bounds__(512) qkv_generic_kernel(
    const uint16_t* __restrict__ qkv, const uint16_t* __restrict__ q_w, const uint16_t* __restrict__ k_w,
    const float* __restrict__ cos_tab, const float* __restrict__ sin_tab, const int32_t* __restrict__ positions,
    uint16_t* __restrict__ q_out, void* __restrict__ k_cache, void* __restrict__ v_cache, int32_t* status, int H,
    int Hq, int Hkv, int hd, int max_pos, int capacity, float eps, Epilogue ep) {
  constexpr bool QEPI = EPI == 1 || EPI == 2;
  constexpr bool KV8 = EPI == 2;
  constexpr bool LN = EPI == 3;
  const int tok = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const int half = hd >> 1;
  // constant inputs before the wait for the previous kernel
  const int64_t M = gridDim.x;  // extents for the bounds-checked build
  const int p = FRT_IDX_OK(tok, M) ? __ldg(positions + tok) : -1;
  const bool row_ok = p >= 0 && p < max_pos && p < capacity;
  float cs[kGenericMaxK], sn[kGenericMaxK];
#pragma unroll
  for (int k = 0; k < kGenericMaxK; ++k) {
    const int j = lane + 32 * k;
    cs[k] = sn[k] = 0.0f;
    if (row_ok && j < half && FRT_IDX_OK((int64_t)p * half + j, (int64_t)max_pos * half)) {
      cs[k] = __ldg(cos_tab + (int64_t)p * half + j);
      sn[k] = __ldg(sin_tab + (int64_t)p * half + j);
    }
  }
  const float k_scale = KV8 && FRT_IDX_OK(0, 2) ? __ldg(ep.kv_scales) : 1.0f;
  const float v_scale = KV8 && FRT_IDX_OK(1, 2) ? __ldg(ep.kv_scales + 1) : 1.0f;
  pdl_enter();
  const int64_t n_qkv = M * H * hd, n_q = M * Hq * hd, n_kv = (int64_t)capacity * Hkv * hd;
  if (!row_ok) {
    if (threadIdx.x == 0 && status != nullptr) atomicOr(status, 1);
    return;
  }
  const float inv_hd = 1.0f / (float)hd;
  const Divisor dk(k_scale), dv(v_scale);
  const uint16_t* row = qkv + (int64_t)tok * H * hd;
  for (int h = threadIdx.x >> 5; h < H; h += blockDim.x >> 5) {  // uniform per warp
    const bool is_q = h < Hq;
    const bool is_v = h >= Hq + Hkv;
    const int hh = is_q ? h : is_v ? h - Hq - Hkv : h - Hq;  // head index within its section
    float a[kGenericMaxK], b[kGenericMaxK];
#pragma unroll
    for (int k = 0; k < kGenericMaxK; ++k) {
      const int j = lane + 32 * k;
      a[k] = b[k] = 0.0f;
      if (j < half && FRT_SPAN_OK((int64_t)tok * H * hd + (int64_t)h * hd + j, half + 1, n_qkv)) {
        a[k] = ld16<DT>(row + (int64_t)h * hd + j);
        b[k] = ld16<DT>(row + (int64_t)h * hd + half + j);
      }
    }
    const int64_t cache_off = ((int64_t)p * Hkv + hh) * hd;
    if (is_v) {
#pragma unroll
      for (int k = 0; k < kGenericMaxK; ++k) {
        const int j = lane + 32 * k;
        if (j >= half || !FRT_SPAN_OK(cache_off + j, half + 1, n_kv)) continue;
        if (KV8) {
          uint8_t* dst = static_cast<uint8_t*>(v_cache) + cache_off;
          dst[j] = (uint8_t)(e4m3x2(dv.fast ? dv.div(a[k]) : dv.div_slow(a[k]), 0.0f) & 0xFFu);
          dst[half + j] = (uint8_t)(e4m3x2(dv.fast ? dv.div(b[k]) : dv.div_slow(b[k]), 0.0f) & 0xFFu);
        } else {  // bit copy
          uint16_t* dst = static_cast<uint16_t*>(v_cache) + cache_off;
          dst[j] = row[(int64_t)h * hd + j];
          dst[half + j] = row[(int64_t)h * hd + half + j];
        }
      }
      continue;
    }
    const uint16_t* w = is_q ? q_w : k_w;
    if (LN) {
      const uint16_t* bias = is_q ? ep.q_bias : ep.k_bias;
      float acc = 0.0f;
#pragma unroll
      for (int k = 0; k < kGenericMaxK; ++k) acc += a[k] + b[k];
      const float mean = group_sum<32>(acc) * inv_hd;
      float acc2 = 0.0f;
#pragma unroll
      for (int k = 0; k < kGenericMaxK; ++k) {
        if (lane + 32 * k < half) {
          a[k] -= mean;
          b[k] -= mean;
          acc2 = fmaf(b[k], b[k], fmaf(a[k], a[k], acc2));
        }
      }
      const float r = head_rstd(group_sum<32>(acc2), inv_hd, eps);
#pragma unroll
      for (int k = 0; k < kGenericMaxK; ++k) {
        const int j = lane + 32 * k;
        if (j >= half) continue;
        const int64_t o = (int64_t)hh * hd;
        const bool aff_ok = FRT_SPAN_OK(o + j, half + 1, (int64_t)(is_q ? Hq : Hkv) * hd);  // rows [Hq | Hkv, hd]
        const float w1 = w && aff_ok ? ld16<DT>(w + o + j) : 1.0f, w2 = w && aff_ok ? ld16<DT>(w + o + half + j) : 1.0f;
        const float b1 = bias && aff_ok ? ld16<DT>(bias + o + j) : 0.0f;
        const float b2 = bias && aff_ok ? ld16<DT>(bias + o + half + j) : 0.0f;
        a[k] = fmaf(a[k] * r, w1, b1);
        b[k] = fmaf(b[k] * r, w2, b2);
      }
    } else if (w != nullptr) {
      float acc = 0.0f;
#pragma unroll
      for (int k = 0; k < kGenericMaxK; ++k) acc = fmaf(b[k], b[k], fmaf(a[k], a[k], acc));
      const float r = head_rstd(group_sum<32>(acc), inv_hd, eps);
#pragma unroll
      for (int k = 0; k < kGenericMaxK; ++k) {
        const int j = lane + 32 * k;
        if (j >= half || !FRT_SPAN_OK(j, half + 1, hd)) continue;
        a[k] = (a[k] * r) * ld16<DT>(w + j);
        b[k] = (b[k] * r) * ld16<DT>(w + half + j);
      }
    }
#pragma unroll
    for (int k = 0; k < kGenericMaxK; ++k) {
      const int j = lane + 32 * k;
      if (j >= half) continue;
      float o1 = fmaf(a[k], cs[k], b[k] * -sn[k]);
      float o2 = fmaf(b[k], cs[k], a[k] * sn[k]);
      if (is_q) {
        if (QEPI) {
          o1 *= ep.q_scale;
          o2 *= ep.q_scale;
        }
        const int64_t qo = (QEPI ? q_row(ep, tok, h, Hq) : (int64_t)tok * Hq + h) * hd;
        if (!FRT_SPAN_OK(qo + j, half + 1, n_q)) continue;
        st16<DT>(q_out + qo + j, o1);
        st16<DT>(q_out + qo + half + j, o2);
      } else if (!FRT_SPAN_OK(cache_off + j, half + 1, n_kv)) {
        continue;
      } else if (KV8) {
        uint8_t* dst = static_cast<uint8_t*>(k_cache) + cache_off;
        dst[j] = (uint8_t)(e4m3x2(dk.fast ? dk.div(o1) : dk.div_slow(o1), 0.0f) & 0xFFu);
        dst[half + j] = (uint8_t)(e4m3x2(dk.fast ? dk.div(o2) : dk.div_slow(o2), 0.0f) & 0xFFu);
      } else {
        uint16_t* dst = static_cast<uint16_t*>(k_cache) + cache_off;
        st16<DT>(dst + j, o1);
        st16<DT>(dst + half + j, o2);
      }
    }
  }
}

template <int DT>
frt_status launch_generic(int epi, const uint16_t* qkv, const uint16_t* qw, const uint16_t* kw, const float* c,
                          const float* sn, const int32_t* pos, uint16_t* qo, void* kc, void* vc, int32_t* status,
                          int M, int H, int Hq, int Hkv, int hd, int max_pos, int capacity, float eps,
                          const Epilogue& ep, cudaStream_t st) {
  const int warps = H < 16 ? H : 16;
  const dim3 grid((unsigned)M), block((unsigned)(32 * warps));
  switch (epi) {
    case 0: return launch(qkv_generic_kernel<DT, 0>, grid, block, 0, st, qkv, qw, kw, c, sn, pos, qo, kc, vc, status,
                          H, Hq, Hkv, hd, max_pos, capacity, eps, ep);
    case 1: return launch(qkv_generic_kernel<DT, 1>, grid, block, 0, st, qkv, qw, kw, c, sn, pos, qo, kc, vc, status,
                          H, Hq, Hkv, hd, max_pos, capacity, eps, ep);
    case 2: return launch(qkv_generic_kernel<DT, 2>, grid, block, 0, st, qkv, qw, kw, c, sn, pos, qo, kc, vc, status,
                          H, Hq, Hkv, hd, max_pos, capacity, eps, ep);
    default: return launch(qkv_generic_kernel<DT, 3>, grid, block, 0, st, qkv, qw, kw, c, sn, pos, qo, kc, vc,
                           status, H, Hq, Hkv, hd, max_pos, capacity, eps, ep);
  }
}

// Polls of the drain wait that follows a give-up (each poll may suspend the
// thread for a while; the bound is far beyond any real copy).  The first
// wait's bound is the process-wide limit of frt_set_wait_polls.
constexpr int kDrainPolls = 1 << 22;

// Bulk-copy kernel (large batches).  One CTA per token.  One thread moves the
// token's whole QKV row, its cos/sin rows and both norm weights into shared
// memory with 1-D bulk copies (TMA) completed on an mbarrier, so no register
// holds in-flight data and a small CTA keeps 12+ KB per token in flight.  Lane
// groups (GP lanes per head) normalise and rotate the Q and K heads in place;
// then the Q row, the K row and the untouched V row leave as three bulk
// stores.  A barrier wait that runs out of polls (max_polls) sets bit 1 of
// *status; the CTA then writes nothing, waits again (kDrainPolls) for the
// copies it issued to land, so that none is still writing into its shared
// memory when it exits, and returns.
// EPI: 0 = op (b) as is (Q token-major, unscaled; 16-bit caches), 1 = Q
// epilogue (scale, layout), 2 = Q epilogue + e4m3 caches, 3 = per-head
// LayerNorm in place of the RMSNorm (affine rows read from global memory,
// nothing staged for them).  At most 128 threads (launched with 96, or 64 at
// the LayerNorm level); the register budget (48 registers at level 0, 55-56
// at levels 1 and 2, 64 at level 3) keeps 12-16 CTAs (tokens) resident per SM:
// the kernel waits on memory, so resident tokens set its rate.  The head
// arithmetic runs on packed fp32 pairs, and the rotation reads cos and sin
// from shared memory slot by slot rather than holding them (negating sin in
// registers: a per-token pass writing -sin beside sin cost a CTA barrier per
// token, 254 -> 238 us for the e4m3 level at 65536 tokens).
template <int EPI>
constexpr int tma_min_blocks() {
  return EPI == 1 || EPI == 3 ? 8 : EPI == 2 ? 9 : 10;
}

template <int DT, int P, int GP, int EPI>
__global__ void __launch_bounds__(128, tma_min_blocks<EPI>()) qkv_norm_rope_kvcache_tma_kernel(
    const uint16_t* __restrict__ qkv, const uint16_t* __restrict__ q_norm_w,
    const uint16_t* __restrict__ k_norm_w, const float* __restrict__ cos_tab, const float* __restrict__ sin_tab,
    const int32_t* __restrict__ positions, uint16_t* __restrict__ q_out, void* __restrict__ k_cache,
    void* __restrict__ v_cache, int32_t* status, int H, int NG, int Hq, int Hkv, int hd, int G, int max_pos,
    int capacity, float eps, Epilogue ep, int max_polls) {
  pdl_enter();
  // [QKV row][cos][sin][q weight][k weight] (+ [K codes][V codes] with EPI 2)
  extern __shared__ __align__(128) uint8_t dsmem[];
  __shared__ uint64_t bar;
  __shared__ int s_pos;
  __shared__ float s_kv[4];  // e4m3 cache scales and their rounded reciprocals (EPI 2)
  const int tok = blockIdx.x;
  const int tid = threadIdx.x;
  const int half = hd >> 1;
  const unsigned row_bytes = (unsigned)(H * hd * 2);
  const unsigned tab_bytes = (unsigned)(half * 4);
  const unsigned w_bytes = (unsigned)(hd * 2);
  uint16_t* rowbuf = reinterpret_cast<uint16_t*>(dsmem);
  float* cbuf = reinterpret_cast<float*>(dsmem + row_bytes);
  float* sbuf = cbuf + half;
  uint16_t* qwbuf = reinterpret_cast<uint16_t*>(sbuf + half);
  uint16_t* kwbuf = qwbuf + hd;
  uint8_t* k8buf = reinterpret_cast<uint8_t*>(kwbuf + hd);
  uint8_t* v8buf = k8buf + Hkv * hd;

  if (tid == 0) {
    mbar_init(&bar, 2);  // two arrivals: the row (+ weights), then the table rows
    mbar_init_fence();
  }
  __syncthreads();
  if (tid == 0) {
    const bool stage_w = EPI != 3;  // LayerNorm rows are per head: read from global memory instead
    // (bounds-checked build: a row outside the QKV buffer is not copied and
    // the token is skipped like a bad position, without the status bit)
    const bool in_b = FRT_SPAN_OK((int64_t)tok * H * hd, H * hd, (int64_t)gridDim.x * H * hd);
    const unsigned first =
        in_b ? row_bytes + (stage_w && q_norm_w ? w_bytes : 0u) + (stage_w && k_norm_w ? w_bytes : 0u) : 0u;
    mbar_arrive_expect_tx(&bar, first);
    if (in_b) {
      bulk_load(rowbuf, qkv + (int64_t)tok * H * hd, row_bytes, &bar);
      if (stage_w && q_norm_w) bulk_load(qwbuf, q_norm_w, w_bytes, &bar);
      if (stage_w && k_norm_w) bulk_load(kwbuf, k_norm_w, w_bytes, &bar);
    }
    const int p = in_b ? __ldg(positions + tok) : -1;
    const bool ok = p >= 0 && p < max_pos && p < capacity &&
                    FRT_SPAN_OK((int64_t)p * half, half, (int64_t)max_pos * half);
    s_pos = ok ? p : -1;
    if (EPI == 2 && FRT_SPAN_OK(0, 2, 2)) {
      const float ks = __ldg(ep.kv_scales), vs = __ldg(ep.kv_scales + 1);
      s_kv[0] = ks;
      s_kv[1] = __frcp_rn(ks);
      s_kv[2] = vs;
      s_kv[3] = __frcp_rn(vs);
    }
    if (ok) {
      mbar_arrive_expect_tx(&bar, 2 * tab_bytes);
      bulk_load(cbuf, cos_tab + (int64_t)p * half, tab_bytes, &bar);
      bulk_load(sbuf, sin_tab + (int64_t)p * half, tab_bytes, &bar);
    } else {
      if (status != nullptr && in_b) atomicOr(status, 1);
      mbar_arrive_expect_tx(&bar, 0u);
    }
  }
  const bool landed = mbar_wait_bounded(&bar, 0, max_polls);
  if (!__syncthreads_and(landed)) {
    if (tid == 0 && status != nullptr) atomicOr(status, 2);
    // Write nothing; drain: every copy above was issued with a byte count the
    // barrier expects, so its phase completes once they have landed.  Only a
    // device whose copies never complete runs this wait out too, and then
    // the CTA exits with them outstanding.
    mbar_wait_bounded(&bar, 0, kDrainPolls);
    return;
  }
  const int p = s_pos;
  if (p < 0) return;  // position out of range: nothing is written
  // (the landed row, tables and weights are visible to every thread: the
  // barrier wait above completed for all of them)
  process_token<DT, P, GP, EPI>(rowbuf, cbuf, sbuf, s_kv, qwbuf, kwbuf, k8buf, v8buf, q_norm_w, k_norm_w, q_out, tok, tid,
                                H, NG, Hq, Hkv, hd, G, eps, ep);
  fence_proxy_async_smem();  // this thread's writes -> the bulk stores below
  __syncthreads();
  if (tid == 0) {
    store_token<EPI>(rowbuf, k8buf, v8buf, q_out, k_cache, v_cache, tok, p, Hq, Hkv, hd, capacity, ep);
    bulk_commit();
    bulk_wait_read();  // shared memory must outlive the stores' reads
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
  Epilogue ep;
};

// CTA shape for GP lanes per head.  Small batches (launch/latency-bound):
// one head per group and up to 1024 threads per token.  Large batches: up to
// four heads per group, NG = ceil(H / 4) groups (at most 256 threads), so each
// thread keeps four heads' loads in flight.
struct Shape {
  int NG, hpg, nhb, threads;
};

inline Shape qkv_shape(int M, int H, int GP, bool kv8) {
  Shape sh;
  const bool large = M >= 4 * 148;
  const int max_threads = kv8 ? 512 : 1024;
  if (large && H >= 2) {
    sh.NG = (H + 3) / 4;
    if (sh.NG * GP > 256) sh.NG = 256 / GP;
    sh.hpg = (H + sh.NG - 1) / sh.NG;
    if (sh.hpg > 4) sh.hpg = 4;
  } else {
    sh.NG = H * GP <= max_threads ? H : max_threads / GP;
    sh.hpg = 1;
  }
  sh.nhb = (H + sh.NG * sh.hpg - 1) / (sh.NG * sh.hpg);
  sh.threads = ((sh.NG * GP + 31) / 32) * 32;
  return sh;
}

// Shared memory of the bulk-copy kernel: the QKV row, cos and sin rows, two
// norm weights, and with an e4m3 cache the K and V code rows.
inline size_t tma_smem(int H, int Hkv, int hd, bool kv8) {
  return (size_t)H * hd * 2 + (size_t)hd * 2 * 2 + (size_t)hd * 2 * 2 + (kv8 ? (size_t)2 * Hkv * hd : 0);
}
constexpr size_t kTmaSmemMax = 200 * 1024;

// Threads of the bulk-copy kernel: a token's heads are taken a few slots at a
// time by fewer lane groups, so more tokens (CTAs) fit on an SM and more
// bytes are in flight; the kernel's rate follows resident tokens.  Measured
// at 65536 tokens of 32/8 heads of 128: 96 threads run op (b) 5 % faster
// than 128 (14 resident tokens instead of 10), and 64 threads suit the
// LayerNorm level (64 registers a thread).
constexpr int kTmaThreads = 96;
constexpr int kTmaThreadsLn = 64;

template <int DT, int P, int GP, int EPI>
frt_status launch_gp(const Args& a, bool tma, cudaStream_t st) {
  constexpr bool KV8 = EPI == 2;
  const uint16_t* qkv = static_cast<const uint16_t*>(a.qkv);
  const uint16_t* qw = static_cast<const uint16_t*>(a.qw);
  const uint16_t* kw = static_cast<const uint16_t*>(a.kw);
  uint16_t* qo = static_cast<uint16_t*>(a.q_out);
  if (tma) {
    static std::atomic<int> opted{0};
    auto kt = qkv_norm_rope_kvcache_tma_kernel<DT, P, GP, EPI>;
    const size_t smem = tma_smem(a.H, a.Hkv, a.hd, KV8);
    const frt_status os = opt_in_smem(kt, smem, opted);
    if (os != FRT_OK) return os;
    const int per = KV8 ? a.H : a.Hq + a.Hkv;  // lane groups needed for one slot of every processed head
    int NG = (per * GP <= kTmaThreads) ? per : kTmaThreads / GP;
    if (NG < 1) NG = 1;
    const int threads = ((NG * GP + 31) / 32) * 32;
    return launch(kt, dim3((unsigned)a.M), dim3(threads), smem, st, qkv, qw, kw, a.cos_tab, a.sin_tab, a.pos, qo,
                  a.kc, a.vc, a.status, a.H, NG, a.Hq, a.Hkv, a.hd, a.G, a.max_pos, a.capacity, a.eps, a.ep,
                  wait_polls());
  }
  const Shape sh = qkv_shape(a.M, a.H, GP, KV8);
  const dim3 grid((unsigned)((int64_t)a.M * sh.nhb));
  if (sh.hpg == 1)
    return launch(qkv_norm_rope_kvcache_kernel<DT, P, GP, 1, EPI>, grid, dim3(sh.threads), 0, st, qkv, qw, kw,
                  a.cos_tab, a.sin_tab, a.pos, qo, a.kc, a.vc, a.status, a.H, sh.NG, sh.hpg, sh.nhb, a.Hq, a.Hkv,
                  a.hd, a.G, a.max_pos, a.capacity, a.eps, a.ep);
  return launch(qkv_norm_rope_kvcache_kernel<DT, P, GP, 4, EPI>, grid, dim3(sh.threads), 0, st, qkv, qw, kw,
                a.cos_tab, a.sin_tab, a.pos, qo, a.kc, a.vc, a.status, a.H, sh.NG, sh.hpg, sh.nhb, a.Hq, a.Hkv, a.hd,
                a.G, a.max_pos, a.capacity, a.eps, a.ep);
}

template <int DT, int P, int GP>
frt_status launch_kv(int epi, const Args& a, bool tma, cudaStream_t st) {
  switch (epi) {
    case 0: return launch_gp<DT, P, GP, 0>(a, tma, st);
    case 1: return launch_gp<DT, P, GP, 1>(a, tma, st);
    default: return launch_gp<DT, P, GP, 2>(a, tma, st);
  }
}

template <int DT, int P>
frt_status launch_p(int GP, int epi, const Args& a, bool tma, cudaStream_t st) {
  switch (GP) {
    case 1: return launch_kv<DT, P, 1>(epi, a, tma, st);
    case 2: return launch_kv<DT, P, 2>(epi, a, tma, st);
    case 4: return launch_kv<DT, P, 4>(epi, a, tma, st);
    case 8: return launch_kv<DT, P, 8>(epi, a, tma, st);
    case 16: return launch_kv<DT, P, 16>(epi, a, tma, st);
    default: return launch_kv<DT, P, 32>(epi, a, tma, st);
  }
}

template <int DT>
frt_status launch_dt(int P, int GP, int epi, const Args& a, bool tma, cudaStream_t st) {
  return P == 8 ? launch_p<DT, 8>(GP, epi, a, tma, st) : launch_p<DT, 4>(GP, epi, a, tma, st);
}

// The bulk-copy kernel at its LayerNorm level (EPI 3), P = 8 rows.
template <int DT, int GP>
frt_status launch_ln_gp(const Args& a, cudaStream_t st) {
  static std::atomic<int> opted{0};
  auto kt = qkv_norm_rope_kvcache_tma_kernel<DT, 8, GP, 3>;
  const size_t smem = tma_smem(a.H, a.Hkv, a.hd, false);
  const frt_status os = opt_in_smem(kt, smem, opted);
  if (os != FRT_OK) return os;
  const int per = a.Hq + a.Hkv;
  int NG = (per * GP <= kTmaThreadsLn) ? per : kTmaThreadsLn / GP;
  if (NG < 1) NG = 1;
  const int threads = ((NG * GP + 31) / 32) * 32;
  return launch(kt, dim3((unsigned)a.M), dim3(threads), smem, st, static_cast<const uint16_t*>(a.qkv),
                static_cast<const uint16_t*>(a.qw), static_cast<const uint16_t*>(a.kw), a.cos_tab, a.sin_tab, a.pos,
                static_cast<uint16_t*>(a.q_out), a.kc, a.vc, a.status, a.H, NG, a.Hq, a.Hkv, a.hd, a.G, a.max_pos,
                a.capacity, a.eps, a.ep, wait_polls());
}

template <int DT>
frt_status launch_ln_tma(int GP, const Args& a, cudaStream_t st) {
  switch (GP) {
    case 1: return launch_ln_gp<DT, 1>(a, st);
    case 2: return launch_ln_gp<DT, 2>(a, st);
    case 4: return launch_ln_gp<DT, 4>(a, st);
    case 8: return launch_ln_gp<DT, 8>(a, st);
    case 16: return launch_ln_gp<DT, 16>(a, st);
    default: return launch_ln_gp<DT, 32>(a, st);
  }
}

// Shared validation and dispatch of both entry points.
frt_status qkv_op(const void* qkv, const void* q_norm_w, const void* k_norm_w, const float* cos_tab,
                  const float* sin_tab, const int32_t* positions, void* q_out, void* k_cache, void* v_cache,
                  int32_t* status, int M, int Hq, int Hkv, int hd, int max_pos, int capacity, float eps,
                  float q_scale, frt_q_layout q_layout, frt_kv_format kv_format, const float* kv_scales,
                  frt_dtype dt, cudaStream_t stream) {
  if (M < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || hd <= 0 || hd % 2 != 0) return FRT_ERR_INVALID_ARG;
  if (max_pos <= 0 || capacity <= 0 || !valid_dtype(dt)) return FRT_ERR_INVALID_ARG;
  if (q_layout != FRT_Q_TOKEN_MAJOR && q_layout != FRT_Q_HEAD_MAJOR) return FRT_ERR_INVALID_ARG;
  if (kv_format != FRT_KV_16BIT && kv_format != FRT_KV_E4M3) return FRT_ERR_INVALID_ARG;
  if (!std::isfinite(q_scale)) return FRT_ERR_INVALID_ARG;
  if (hd > 256) return FRT_ERR_UNSUPPORTED;
  if (M == 0) return FRT_OK;
  if (!qkv || !cos_tab || !sin_tab || !positions || !q_out || !k_cache || !v_cache) return FRT_ERR_INVALID_ARG;
  const bool kv8 = kv_format == FRT_KV_E4M3;
  if (kv8 && (!kv_scales || !aligned(kv_scales, 4))) return FRT_ERR_INVALID_ARG;
  const int epi = kv8 ? 2 : (q_scale != 1.0f || q_layout != FRT_Q_TOKEN_MAJOR) ? 1 : 0;
  if (hd % 8 != 0) {  // element-wise kernel: 16-bit pointers 2-byte aligned
    if (!aligned(qkv, 2) || !aligned(q_out, 2) || (!kv8 && (!aligned(k_cache, 2) || !aligned(v_cache, 2))) ||
        (q_norm_w && !aligned(q_norm_w, 2)) || (k_norm_w && !aligned(k_norm_w, 2)) || !aligned(cos_tab, 4) ||
        !aligned(sin_tab, 4) || !aligned(positions, 4) || (status && !aligned(status, 4)))
      return FRT_ERR_INVALID_ARG;
    const Epilogue ep{q_scale, q_layout == FRT_Q_HEAD_MAJOR ? 1 : 0, M, kv_scales, nullptr, nullptr};
    const int H = Hq + 2 * Hkv;
    const auto* qk = static_cast<const uint16_t*>(qkv);
    const auto* qw = static_cast<const uint16_t*>(q_norm_w);
    const auto* kw = static_cast<const uint16_t*>(k_norm_w);
    auto* qo = static_cast<uint16_t*>(q_out);
    return dt == FRT_F16 ? launch_generic<FRT_F16>(epi, qk, qw, kw, cos_tab, sin_tab, positions, qo, k_cache, v_cache,
                                                   status, M, H, Hq, Hkv, hd, max_pos, capacity, eps, ep, stream)
                         : launch_generic<FRT_BF16>(epi, qk, qw, kw, cos_tab, sin_tab, positions, qo, k_cache,
                                                    v_cache, status, M, H, Hq, Hkv, hd, max_pos, capacity, eps, ep,
                                                    stream);
  }
  const int P = (hd % 16 == 0) ? 8 : 4;
  const uintptr_t al = (P == 8) ? 16 : 8;
  const uintptr_t al_kv = kv8 ? (uintptr_t)P : al;  // e4m3 rows: P codes per lane store
  if (!aligned(qkv, al) || !aligned(q_out, al) || !aligned(k_cache, al_kv) || !aligned(v_cache, al_kv))
    return FRT_ERR_INVALID_ARG;
  if ((q_norm_w && !aligned(q_norm_w, al)) || (k_norm_w && !aligned(k_norm_w, al))) return FRT_ERR_INVALID_ARG;
  if (!aligned(cos_tab, 16) || !aligned(sin_tab, 16) || !aligned(positions, 4)) return FRT_ERR_INVALID_ARG;
  if (status && !aligned(status, 4)) return FRT_ERR_INVALID_ARG;
  const int H = Hq + 2 * Hkv;
  const int G = (hd / 2) / P;  // active lanes per head, <= 31
  int GP = 1;
  while (GP < G) GP *= 2;
  Args a{qkv, q_norm_w, k_norm_w, cos_tab, sin_tab, positions, q_out, k_cache, v_cache, status,
         M, H, Hq, Hkv, hd, G, max_pos, capacity, eps,
         Epilogue{q_scale, q_layout == FRT_Q_HEAD_MAJOR ? 1 : 0, M, kv_scales, nullptr, nullptr}};
  if ((int64_t)M * qkv_shape(M, H, GP, kv8).nhb > 0x7FFFFFFF) return FRT_ERR_UNSUPPORTED;
  // Bulk-copy path for large batches when every row it moves is 16-byte
  // aligned (bulk copies need 16-byte addresses and sizes) and fits in
  // shared memory; the register kernel otherwise.
  const bool tma = M >= 4 * 148 && aligned(qkv, 16) && aligned(q_out, 16) && aligned(k_cache, 16) &&
                   aligned(v_cache, 16) && (!q_norm_w || aligned(q_norm_w, 16)) &&
                   (!k_norm_w || aligned(k_norm_w, 16)) && (!kv8 || (Hkv * hd) % 16 == 0) &&
                   tma_smem(H, Hkv, hd, kv8) <= kTmaSmemMax;
  return dt == FRT_F16 ? launch_dt<FRT_F16>(P, GP, epi, a, tma, stream)
                       : launch_dt<FRT_BF16>(P, GP, epi, a, tma, stream);
}

}  // namespace
}  // namespace frt

extern "C" frt_status frt_qkv_norm_rope_kvcache(const void* qkv, const void* q_norm_w, const void* k_norm_w,
                                                const float* cos_tab, const float* sin_tab,
                                                const int32_t* positions, void* q_out, void* k_cache,
                                                void* v_cache, int32_t* status, int M, int Hq, int Hkv, int hd,
                                                int max_pos, int capacity, float eps, frt_dtype dt,
                                                cudaStream_t stream) {
  return frt::qkv_op(qkv, q_norm_w, k_norm_w, cos_tab, sin_tab, positions, q_out, k_cache, v_cache, status, M, Hq,
                     Hkv, hd, max_pos, capacity, eps, 1.0f, FRT_Q_TOKEN_MAJOR, FRT_KV_16BIT, nullptr, dt, stream);
}

extern "C" frt_status frt_qkv_norm_rope_prepq_kvcache(const void* qkv, const void* q_norm_w, const void* k_norm_w,
                                                      const float* cos_tab, const float* sin_tab,
                                                      const int32_t* positions, void* q_out, void* k_cache,
                                                      void* v_cache, int32_t* status, int M, int Hq, int Hkv,
                                                      int hd, int max_pos, int capacity, float eps, float q_scale,
                                                      frt_q_layout q_layout, frt_kv_format kv_format,
                                                      const float* kv_scales, frt_dtype dt, cudaStream_t stream) {
  return frt::qkv_op(qkv, q_norm_w, k_norm_w, cos_tab, sin_tab, positions, q_out, k_cache, v_cache, status, M, Hq,
                     Hkv, hd, max_pos, capacity, eps, q_scale, q_layout, kv_format, kv_scales, dt, stream);
}

extern "C" frt_status frt_qkv_layernorm_rope_kvcache(const void* qkv, const void* q_w, const void* q_b, const void* k_w,
                                                    const void* k_b, const float* cos_tab, const float* sin_tab,
                                                    const int32_t* positions, void* q_out, void* k_cache,
                                                    void* v_cache, int32_t* status, int M, int Hq, int Hkv, int hd,
                                                    int max_pos, int capacity, float eps, frt_dtype dt,
                                                    cudaStream_t stream) {
  using namespace frt;
  if (M < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || hd <= 0 || hd % 2 != 0) return FRT_ERR_INVALID_ARG;
  if (max_pos <= 0 || capacity <= 0 || !valid_dtype(dt)) return FRT_ERR_INVALID_ARG;
  if (hd > 256) return FRT_ERR_UNSUPPORTED;
  if (M == 0) return FRT_OK;
  if (!qkv || !cos_tab || !sin_tab || !positions || !q_out || !k_cache || !v_cache) return FRT_ERR_INVALID_ARG;
  const int H = Hq + 2 * Hkv;
  if (hd % 8 != 0) {  // element-wise kernel (see frt_qkv_norm_rope_kvcache)
    if (!aligned(qkv, 2) || !aligned(q_out, 2) || !aligned(k_cache, 2) || !aligned(v_cache, 2) ||
        !aligned(cos_tab, 4) || !aligned(sin_tab, 4) || !aligned(positions, 4) || (status && !aligned(status, 4)))
      return FRT_ERR_INVALID_ARG;
    for (const void* w : {q_w, q_b, k_w, k_b})
      if (w && !aligned(w, 2)) return FRT_ERR_INVALID_ARG;
    const Epilogue ep{1.0f, 0, M, nullptr, static_cast<const uint16_t*>(q_b), static_cast<const uint16_t*>(k_b)};
    const auto* qk = static_cast<const uint16_t*>(qkv);
    const auto* qw = static_cast<const uint16_t*>(q_w);
    const auto* kw = static_cast<const uint16_t*>(k_w);
    auto* qo = static_cast<uint16_t*>(q_out);
    return dt == FRT_F16 ? launch_generic<FRT_F16>(3, qk, qw, kw, cos_tab, sin_tab, positions, qo, k_cache, v_cache,
                                                   status, M, H, Hq, Hkv, hd, max_pos, capacity, eps, ep, stream)
                         : launch_generic<FRT_BF16>(3, qk, qw, kw, cos_tab, sin_tab, positions, qo, k_cache, v_cache,
                                                    status, M, H, Hq, Hkv, hd, max_pos, capacity, eps, ep, stream);
  }
  const int P = (hd % 16 == 0) ? 8 : 4;
  const uintptr_t al = (P == 8) ? 16 : 8;
  if (!aligned(qkv, al) || !aligned(q_out, al) || !aligned(k_cache, al) || !aligned(v_cache, al))
    return FRT_ERR_INVALID_ARG;
  for (const void* w : {q_w, q_b, k_w, k_b})
    if (w && !aligned(w, al)) return FRT_ERR_INVALID_ARG;
  if (!aligned(cos_tab, 16) || !aligned(sin_tab, 16) || !aligned(positions, 4)) return FRT_ERR_INVALID_ARG;
  if (status && !aligned(status, 4)) return FRT_ERR_INVALID_ARG;
  const int G = (hd / 2) / P;
  int GP = 1;
  while (GP < G) GP *= 2;
  // Small batches: one head per lane group, up to 512 threads per token.
  // Large batches: up to four heads per group (more bytes in flight per
  // thread), at most 256 threads.
  const bool large = M >= 4 * 148;
  int NG, HPG;
  if (large && H >= 2) {
    NG = (H + 3) / 4;
    if (NG * GP > 256) NG = 256 / GP;
    HPG = 4;
  } else {
    NG = H * GP <= 512 ? H : 512 / GP;
    HPG = 1;
  }
  const int nhb = (H + NG * HPG - 1) / (NG * HPG);
  if ((int64_t)M * nhb > 0x7FFFFFFF) return FRT_ERR_UNSUPPORTED;
  const int threads = ((NG * GP + 31) / 32) * 32;
  const dim3 grid((unsigned)((int64_t)M * nhb));
  // Large batches with 16-byte rows: the bulk-copy kernel at its LayerNorm
  // level (the token's row staged in shared memory, 10 tokens per SM).
  if (large && P == 8 && aligned(qkv, 16) && aligned(q_out, 16) && aligned(k_cache, 16) && aligned(v_cache, 16) &&
      tma_smem(H, Hkv, hd, false) <= kTmaSmemMax) {
    Args a{qkv, q_w, k_w, cos_tab, sin_tab, positions, q_out, k_cache, v_cache, status, M, H, Hq, Hkv, hd, G,
           max_pos, capacity, eps,
           Epilogue{1.0f, 0, M, nullptr, static_cast<const uint16_t*>(q_b), static_cast<const uint16_t*>(k_b)}};
    return dt == FRT_F16 ? launch_ln_tma<FRT_F16>(GP, a, stream) : launch_ln_tma<FRT_BF16>(GP, a, stream);
  }
  const uint16_t* qk = static_cast<const uint16_t*>(qkv);
  const uint16_t* w16[4] = {static_cast<const uint16_t*>(q_w), static_cast<const uint16_t*>(q_b),
                            static_cast<const uint16_t*>(k_w), static_cast<const uint16_t*>(k_b)};
  uint16_t* qo = static_cast<uint16_t*>(q_out);
  uint16_t* kc = static_cast<uint16_t*>(k_cache);
  uint16_t* vc = static_cast<uint16_t*>(v_cache);
#define FRT_LN_LAUNCH(DT_, P_, GP_)                                                                            \
  return HPG == 1 ? launch(qkv_layernorm_rope_kvcache_kernel<DT_, P_, GP_, 1>, grid, dim3(threads), 0, stream, qk, \
                           w16[0], w16[1], w16[2], w16[3], cos_tab, sin_tab, positions, qo, kc, vc, status, H, NG, \
                           nhb, Hq, Hkv, hd, G, max_pos, capacity, eps)                                            \
                  : launch(qkv_layernorm_rope_kvcache_kernel<DT_, P_, GP_, 4>, grid, dim3(threads), 0, stream, qk, \
                           w16[0], w16[1], w16[2], w16[3], cos_tab, sin_tab, positions, qo, kc, vc, status, H, NG, \
                           nhb, Hq, Hkv, hd, G, max_pos, capacity, eps)
#define FRT_LN_GP(DT_, P_)          \
  switch (GP) {                     \
    case 1: FRT_LN_LAUNCH(DT_, P_, 1);  \
    case 2: FRT_LN_LAUNCH(DT_, P_, 2);  \
    case 4: FRT_LN_LAUNCH(DT_, P_, 4);  \
    case 8: FRT_LN_LAUNCH(DT_, P_, 8);  \
    case 16: FRT_LN_LAUNCH(DT_, P_, 16); \
    default: FRT_LN_LAUNCH(DT_, P_, 32); \
  }
  if (dt == FRT_F16) {
    if (P == 8) {
      FRT_LN_GP(FRT_F16, 8)
    } else {
      FRT_LN_GP(FRT_F16, 4)
    }
  }
  if (P == 8) {
    FRT_LN_GP(FRT_BF16, 8)
  }
  FRT_LN_GP(FRT_BF16, 4)
#undef FRT_LN_GP
#undef FRT_LN_LAUNCH
}
