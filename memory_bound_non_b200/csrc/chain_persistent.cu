// NEXT-4: the layer chain as one persistent kernel (small batches).
//
// "FlashFormer: Whole-Model Kernels for Efficient Low-Batch Inference": at a
// few tokens the per-kernel launch and dependency latency dominates, so the
// whole sequence runs inside one kernel.  Here that sequence is the graphed
// chain: for every step and layer, op a (attention norm), op b (QKV), op a
// (FFN norm), op c (gated activation) ("FlashRT kernel fusion", §二 steps 1,
// 3, 7, 8-10; §三 for the per-step loop).
//
// Mapping (B200).  The chain's only dependency is the residual stream of each
// row (a -> a -> next layer's a); the QKV and gate/up buffers that ops b and c
// read are the fixed per-layer outputs of GEMMs that are not part of the
// chain, so a row's ops depend on that row alone, and ops b and c do not
// depend on the residual at all.  Each row is owned by a thread-block cluster
// of S CTAs (S <= 8, so that rows x S fills the SMs) that runs the row's whole
// chain in one launch with no grid-wide barrier and no cross-CTA exchange:
// CTA 0 runs the residual chain (both norms of every layer, the residual row
// in registers from the first op to the last), while CTAs 1..S-1 split the
// heads of op b and the 128-output blocks of op c between them and run
// alongside (with S == 1 one CTA does everything in order).  Each CTA copies
// the next layer invocation's input slices into a second shared-memory stage
// (16-byte asynchronous copies, spread evenly over all its threads) while the
// current one computes.  With real GEMMs between the ops, rows would mix and a
// grid-wide step would be needed.  Each op uses the arithmetic of its per-op
// kernel (packed 16-bit add, fp64 row sum of squares, the same FP8 decision
// arithmetic, RoPE and activation expressions), so the results equal the
// per-op launches bit for bit.  A table pointer below its field's alignment
// sets status bit 2 before anything is read or written.
//
// Staging forms measured at 10 and 41 tokens and not kept: the eight slices
// as 1-D bulk copies (TMA) issued by one thread on an mbarrier (7-9 % slower:
// one thread's eight issues sit on the critical path at the next barrier,
// wherever they are placed), and the copies issued after the barrier so they
// overlap the arithmetic (8-10 % slower: they queue beside the norms' shared
// loads and shuffles).
#include <atomic>
#include <cmath>
#include <cstddef>
#include <cooperative_groups.h>

#include "frt_device.cuh"
#include "frt_host.h"

namespace frt {
namespace {

namespace cg = cooperative_groups;

constexpr int kChainThreads = 256;
constexpr int kChainWarps = kChainThreads / 32;

// CTA-wide fp64 sum (warp butterfly, then the warp partials in order).  The
// two norms of a layer use the two halves of a 2 * kChainWarps buffer, so a
// call needs no trailing barrier: the next call on the same half comes after
// the loop's barriers.
__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double tot = 0.0;
#pragma unroll
  for (int i = 0; i < kChainWarps; ++i) tot += red[i];
  return tot;
}

// The cluster's slices of one row.
struct Slice {
  int c0, nc;  // 16-byte chunks of the D columns
  int h0, nh;  // heads
  int b0, nb;  // 128-output activation blocks
};

// Op a on the row (held by this CTA): h = x + r (into hv), RMSNorm, FP8 codes.
template <int DT, int K, int QM>
__device__ __forceinline__ void chain_norm(const uint4* xs, const uint4* ws, uint2* q, float* bs, const Divisor& dv,
                                           double inv_s64, uint4 (&hv)[K], int64_t row, const Slice& sl, int C,
                                           int NB, float D, double invD, float eps, double* red, int64_t n_rows) {
  using P16 = Pack16<DT>;
  const int t = threadIdx.x;
  uint4 xv[K], wv[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int j = t + k * kChainThreads;
    if (j < sl.nc) {
      xv[k] = xs[j];
      if (ws != nullptr) wv[k] = ws[j];
    }
  }
  double ss[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    ss[k] = 0.0;
    if (t + k * kChainThreads < sl.nc) {
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
  const double tot = block_sum(sst, red);
  // the mean square (for a power-of-two D the product with 1 / D is exact)
  const double ms = invD > 0.0 ? tot * invD : tot / (double)D;
  // static FP8: one product with rstd / s, as op a does
  const double rstd64 = rsqrt_f64(ms + (double)eps);
  const double rs64 = rstd64 * inv_s64;
  const bool fold = QM == FRT_QUANT_STATIC && rs64 >= 0x1p-100 && rs64 <= 0x1p+100;
  const Split32 rstd(fold ? rs64 : rstd64);
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int j = t + k * kChainThreads;
    const bool valid = j < sl.nc;
    const int c = sl.c0 + j;
    const uint32_t* hw = reinterpret_cast<const uint32_t*>(&hv[k]);
    const uint32_t* ww = reinterpret_cast<const uint32_t*>(&wv[k]);
    float y[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 hf = P16::to_float2(hw[e]);
      if (ws != nullptr && valid) {
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
      am = half_warp_max_abs(am);
      const float sb = block_scale_448(am);
      if (valid && (j & 15) == 0 && FRT_IDX_OK(row * NB + (c >> 4), n_rows * NB)) bs[row * NB + (c >> 4)] = sb;
      if (valid && FRT_IDX_OK(row * C + c, n_rows * C)) q[row * C + c] = quant8(y, Divisor(sb));
    } else if (valid && FRT_IDX_OK(row * C + c, n_rows * C)) {
      q[row * C + c] = fold ? e4m3x8(y) : quant8(y, dv);
    }
  }
}

// Op b on this CTA's heads: lane groups of GP lanes per head (P = 8 elements
// and their rotation partners per lane), kChainThreads / GP heads per pass.
template <int DT, int GP>
__device__ __forceinline__ void chain_qkv(const uint16_t* heads, const uint16_t* qw, const uint16_t* kw,
                                          uint16_t* q_out, uint16_t* k_cache, uint16_t* v_cache, const float2* cs,
                                          const float2* sn, const float2* nsn, int64_t row, int p, bool row_ok,
                                          const Slice& sl, int Hq, int Hkv, int hd, int G, float eps,
                                          int64_t n_rows, int capacity) {
  constexpr int P = 8;
  constexpr int NP = P / 2;
  const float inv_hd = 1.0f / (float)hd;
  const int NG = kChainThreads / GP;
  const int grp = threadIdx.x / GP;
  const int li = threadIdx.x & (GP - 1);
  const int half = hd >> 1;
  const int j0 = li * P;
  const bool lane_ok = li < G && row_ok;
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
  for (int i0 = 0; i0 < sl.nh; i0 += NG) {
    const int i = i0 + grp;  // head index within the slice
    const int h = sl.h0 + i;
    const bool on = lane_ok && i < sl.nh;
    const bool is_q = h < Hq;
    const bool is_v = h >= Hq + Hkv;
    const uint16_t* nw = is_q ? qw : kw;
    const bool do_norm = !is_v && nw != nullptr;
    uint4 va = make_uint4(0, 0, 0, 0), vb = va;
    if (on) {
      va = *reinterpret_cast<const uint4*>(heads + (int64_t)i * hd + j0);
      vb = *reinterpret_cast<const uint4*>(heads + (int64_t)i * hd + half + j0);
    }
    const int64_t n_kv = (int64_t)capacity * Hkv * hd;
    if (on && is_v && FRT_SPAN_OK(((int64_t)p * Hkv + (h - Hq - Hkv)) * hd + j0, half + P, n_kv)) {
      uint16_t* dst = v_cache + ((int64_t)p * Hkv + (h - Hq - Hkv)) * hd;
      *reinterpret_cast<uint4*>(dst + j0) = va;
      *reinterpret_cast<uint4*>(dst + half + j0) = vb;
    }
    float2 a[NP], b[NP];
    float ss = 0.0f;
    if (on && !is_v) {
      unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&va), a);
      unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&vb), b);
      if (do_norm) ss = sum_squares_pairs<NP>(a, b);
    }
    ss = group_sum<GP>(ss);  // every lane of the warp takes part
    if (on && !is_v) {
      if (do_norm) {
        const float rstd = head_rstd(ss, inv_hd, eps);
        const uint4 wa = is_q ? qwa : kwa, wb = is_q ? qwb : kwb;
        float2 fa[NP], fb[NP];
        unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&wa), fa);
        unpack_pairs<DT, NP>(reinterpret_cast<const uint32_t*>(&wb), fb);
        scale_pairs<NP>(a, rstd, fa);
        scale_pairs<NP>(b, rstd, fb);
      }
      float2 x[NP], y[NP];
      rope_pairs<NP>(a, b, cs, sn, nsn, x, y);
      uint4 o1, o2;
      pack_pairs<DT, NP>(x, reinterpret_cast<uint32_t*>(&o1));
      pack_pairs<DT, NP>(y, reinterpret_cast<uint32_t*>(&o2));
      const int64_t o = is_q ? (row * Hq + h) * hd : ((int64_t)p * Hkv + (h - Hq)) * hd;
      uint16_t* dst = (is_q ? q_out : k_cache) + o;
      if (FRT_SPAN_OK(o + j0, half + P, is_q ? n_rows * Hq * hd : n_kv)) {
        *reinterpret_cast<uint4*>(dst + j0) = o1;
        *reinterpret_cast<uint4*>(dst + half + j0) = o2;
      }
    }
  }
}

// Op c on this CTA's 128-output blocks: each warp takes blocks four at a time
// with their loads issued first (one 16-byte load = 4 (g, u) pairs).
template <int DT, int QM, int ACT>
__device__ __forceinline__ void chain_act(const uint4* gs, uint32_t* q, float* bs, const Divisor& dv, int64_t row,
                                          const Slice& sl, int I4, int NBI, int64_t n_rows) {
  const int lane = threadIdx.x & 31;
  // blocks go to the warps from the last one down and heads (chain_qkv) to
  // the threads from the first one up, so small slices of both overlap
  const int warp = kChainWarps - 1 - (threadIdx.x >> 5);
  uint32_t* dst = q + row * I4;
  for (int i0 = warp * 4; i0 < sl.nb; i0 += kChainWarps * 4) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (i0 + u < sl.nb) v[u] = gs[(i0 + u) * 32 + lane];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (i0 + u >= sl.nb) break;  // uniform across the warp
      const int b = sl.b0 + i0 + u;
      float a[4];
      const uint32_t* w = reinterpret_cast<const uint32_t*>(&v[u]);
      const float2 a01 = act_mul2<DT, ACT>(w[0], w[1]), a23 = act_mul2<DT, ACT>(w[2], w[3]);
      a[0] = a01.x;
      a[1] = a01.y;
      a[2] = a23.x;
      a[3] = a23.y;
      if (QM == FRT_QUANT_BLOCK128) {
        const float am = warp_max_abs(absmax4(a[0], a[1], a[2], a[3]));
        const float sb = block_scale_448(am);
        if (lane == 0 && FRT_IDX_OK(row * NBI + b, n_rows * NBI)) bs[row * NBI + b] = sb;
        if (FRT_IDX_OK(row * I4 + b * 32 + lane, n_rows * I4)) dst[b * 32 + lane] = quant4(a, Divisor(sb));
      } else if (FRT_IDX_OK(row * I4 + b * 32 + lane, n_rows * I4)) {
        dst[b * 32 + lane] = quant4(a, dv);
      }
    }
  }
}

// 16-byte asynchronous global -> shared copy (L2 only) and its groups.
__device__ __forceinline__ void cp_async16(uint4* smem, const void* gmem) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(smem);
  // no memory clobber: nothing reads the stage before cp_async_wait1 and the
  // barrier after it, which order the copies for the compiler
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(a), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// Offsets (16-byte chunks) of one stage of this CTA's slices: x_attn, x_ffn,
// the two norm weights, the head slice of the QKV row, the q / k norm
// weights, the block slice of the gate/up row.
struct StageMap {
  int xa, xf, wa, wf, qkv, qw, kw, gu, len;
  __host__ __device__ StageMap(int cs, int heads16, int hd16, int gu16)
      : xa(0), xf(cs), wa(2 * cs), wf(3 * cs), qkv(4 * cs), qw(4 * cs + heads16), kw(4 * cs + heads16 + hd16),
        gu(4 * cs + heads16 + 2 * hd16), len(4 * cs + heads16 + 2 * hd16 + gu16) {}
};

// A layer's eight stage sources are the first eight pointers of its table
// entry, in StageMap order.
static_assert(offsetof(frt_chain_layer, x_attn) == 0 && offsetof(frt_chain_layer, x_ffn) == 8 &&
                  offsetof(frt_chain_layer, w_attn) == 16 && offsetof(frt_chain_layer, w_ffn) == 24 &&
                  offsetof(frt_chain_layer, qkv) == 32 && offsetof(frt_chain_layer, q_norm_w) == 40 &&
                  offsetof(frt_chain_layer, k_norm_w) == 48 && offsetof(frt_chain_layer, gate_up) == 56,
              "stage sources lead the layer record");

// Words of one frt_chain_layer record, and the alignment each pointer needs:
// the eight staged inputs and the 16-byte stores (q_out, the caches) 16
// bytes, the 8-byte code stores 8, the activation codes and the scales 4.
constexpr int kLayerWords = (int)(sizeof(frt_chain_layer) / 8);
static_assert(kLayerWords == 17, "frt_chain_layer holds 17 pointers");
static_assert(offsetof(frt_chain_layer, k_cache) == 64 && offsetof(frt_chain_layer, q_out) == 80 &&
                  offsetof(frt_chain_layer, q8_attn) == 88 && offsetof(frt_chain_layer, act8) == 104,
              "frt_chain_layer field order");
__device__ __forceinline__ uint64_t layer_field_align(int field) {
  return field < 11 ? 16u : field < 13 ? 8u : 4u;
}

// Where the chunks of one stage slice come from: stage chunk i of slice s is
// chunk delta + i of that slice's source buffer (lim chunks long).
struct SliceSrc {
  int64_t delta, lim;
};

// Copies every input slice one layer invocation of this CTA reads.  The stage
// is one run of m.len chunks (slices in StageMap order); each thread takes
// every kChainThreads-th chunk, finds its slice by comparing against the slice
// starts, and copies it from that layer's source pointer (src: the layer's
// eight source pointers, null for an absent weight).
__device__ __forceinline__ void stage_layer(uint4* st, const StageMap& m, const uint64_t* src, const SliceSrc* ss) {
  for (int i = threadIdx.x; i < m.len; i += kChainThreads) {
    const int s = (i >= m.xf) + (i >= m.wa) + (i >= m.wf) + (i >= m.qkv) + (i >= m.qw) + (i >= m.kw) + (i >= m.gu);
    const uint64_t p = src[s];
    const int64_t j = ss[s].delta + i;
    if (p != 0 && FRT_IDX_OK(j, ss[s].lim)) cp_async16(st + i, reinterpret_cast<const uint4*>(p) + j);
  }
}

template <int DT, int K, int QM, int GP, int ACT>
__global__ void __launch_bounds__(kChainThreads, 1) chain_persistent_kernel(
    const frt_chain_layer* __restrict__ layers, int n_layers, int steps, uint4* residual,
    const float* __restrict__ cos_tab, const float* __restrict__ sin_tab, const int32_t* __restrict__ positions,
    const float* __restrict__ scales, int32_t* status, int C, int NB, int Hq, int Hkv, int hd, int G, int I4,
    int NBI, int max_pos, int capacity, float eps) {
  __shared__ double red[2 * kChainWarps];
  pdl_enter();
  cg::cluster_group cl = cg::this_cluster();
  const unsigned S = cl.num_blocks();
  const int r = (int)cl.block_rank();
  const int t = threadIdx.x;
  const int64_t row = blockIdx.x / S;
  const int H = Hq + 2 * Hkv;
  // roles: CTA 0 runs both norms on the whole row (the residual chain); the
  // heads and activation blocks go to CTAs 1..S-1 (all to CTA 0 when S == 1)
  const bool norm_cta = r == 0;
  const int workers = S > 1 ? (int)S - 1 : 1;
  const int w = S > 1 ? r - 1 : 0;
  Slice sl;
  sl.c0 = 0;
  sl.nc = norm_cta ? C : 0;
  const int hs = (H + workers - 1) / workers, bsl = (NBI + workers - 1) / workers;
  const bool bc_cta = S == 1 || r > 0;
  sl.h0 = bc_cta ? min(H, w * hs) : 0;
  sl.nh = bc_cta ? min(H, sl.h0 + hs) - sl.h0 : 0;
  sl.b0 = bc_cta ? min(NBI, w * bsl) : 0;
  sl.nb = bc_cta ? min(NBI, sl.b0 + bsl) - sl.b0 : 0;

  const int64_t n_rows = gridDim.x / S;  // extents for the bounds-checked build
  uint4 hv[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int j = t + k * kChainThreads;
    hv[k] = j < sl.nc && FRT_IDX_OK(row * C + sl.c0 + j, n_rows * C) ? residual[row * C + sl.c0 + j]
                                                                   : make_uint4(0u, 0u, 0u, 0u);
  }
  const int p = FRT_IDX_OK(row, n_rows) ? __ldg(positions + row) : -1;
  const bool row_ok = p >= 0 && p < max_pos && p < capacity;
  if (!row_ok && t == 0 && r == 0 && status != nullptr) atomicOr(status, 1);
  constexpr int P = 8;
  const int li = t & (GP - 1);
  const int half = hd >> 1;
  float2 cs8[P / 2], sn8[P / 2], nsn8[P / 2];
  if (row_ok && li < G && FRT_SPAN_OK((int64_t)p * half + li * P, P, (int64_t)max_pos * half))
    load_rope_pairs<P / 2>(cos_tab + (int64_t)p * half + li * P, sin_tab + (int64_t)p * half + li * P, cs8, sn8,
                           nsn8);
  const bool scales_ok = FRT_SPAN_OK(0, 3, 3);
  const Divisor dv_attn(QM == FRT_QUANT_STATIC && scales_ok ? __ldg(scales) : 1.0f);
  const Divisor dv_ffn(QM == FRT_QUANT_STATIC && scales_ok ? __ldg(scales + 1) : 1.0f);
  // static FP8: 1 / s in fp64 for the norms' folded product (0 otherwise)
  const double inv_attn = QM == FRT_QUANT_STATIC ? 1.0 / (double)dv_attn.s : 0.0;
  const double inv_ffn = QM == FRT_QUANT_STATIC ? 1.0 / (double)dv_ffn.s : 0.0;
  const Divisor dv_act(QM == FRT_QUANT_STATIC && scales_ok ? __ldg(scales + 2) : 1.0f);
  const float D = (float)(C * 8);
  const double invD = (C * 8 & (C * 8 - 1)) == 0 ? 1.0 / (double)(C * 8) : 0.0;  // exact for powers of two
  const int qkv16 = H * hd / 8, hd16 = hd / 8;
  // this CTA's stage layout: exactly the slices of its own roles (the last
  // worker's head and block slices can be shorter than hs and bsl; the host
  // sizes shared memory for the largest layout, so this one always fits).
  // Every chunk of the layout is copied, so it must not reach past a slice.
  const StageMap m(sl.nc, sl.nh * hd16, hd16, sl.nb * 32);

  // dynamic shared memory: the layer table (so no iteration waits on a global
  // load of its pointers), then the two stages
  extern __shared__ uint4 smem[];
  __shared__ SliceSrc ssrc[8];
  frt_chain_layer* tab = reinterpret_cast<frt_chain_layer*>(smem);
  uint4* stages = smem + (n_layers * (int)sizeof(frt_chain_layer) + 15) / 16;
  {
    const uint64_t* src = reinterpret_cast<const uint64_t*>(layers);
    uint64_t* dst = reinterpret_cast<uint64_t*>(tab);
    const int words = n_layers * (int)(sizeof(frt_chain_layer) / 8);
    bool misaligned = false;
    for (int i = t; i < words; i += kChainThreads)
      if (FRT_IDX_OK(i, words)) {
        const uint64_t word = __ldg(src + i);
        dst[i] = word;
        misaligned |= (word & (layer_field_align(i % kLayerWords) - 1)) != 0;
      }
    if (t < 8) {  // slice t of this CTA's stage: where its chunks come from
      int b;
      int64_t o, l;
      switch (t) {
        case 0: b = m.xa; o = row * C + sl.c0; l = n_rows * C; break;
        case 1: b = m.xf; o = row * C + sl.c0; l = n_rows * C; break;
        case 2: b = m.wa; o = sl.c0; l = C; break;
        case 3: b = m.wf; o = sl.c0; l = C; break;
        case 4: b = m.qkv; o = row * qkv16 + (int64_t)sl.h0 * hd16; l = n_rows * qkv16; break;
        case 5: b = m.qw; o = 0; l = hd16; break;
        case 6: b = m.kw; o = 0; l = hd16; break;
        default: b = m.gu; o = row * I4 + (int64_t)sl.b0 * 32; l = n_rows * I4; break;
      }
      ssrc[t].delta = o - b;
      ssrc[t].lim = l;
    }
    // a table pointer below its field's alignment: report it and touch none
    if (__syncthreads_or(misaligned)) {
      if (t == 0 && r == 0 && status != nullptr) atomicOr(status, 4);
      return;
    }
  }
  const int total = steps * n_layers;
  if (total > 0) {
    stage_layer(stages, m, reinterpret_cast<const uint64_t*>(tab), ssrc);
    cp_async_commit();
  }
  for (int it = 0; it < total; ++it) {
    const frt_chain_layer& L = tab[it % n_layers];
    if (it + 1 < total)
      stage_layer(stages + ((it + 1) & 1) * m.len, m, reinterpret_cast<const uint64_t*>(tab + (it + 1) % n_layers),
                  ssrc);
    cp_async_commit();  // possibly empty: one group per iteration
    cp_async_wait1();   // this iteration's stage has landed (only the newest group may be pending)
    __syncthreads();    // ... for every thread's copies
    const uint4* st = stages + (it & 1) * m.len;
    if (norm_cta)
      chain_norm<DT, K, QM>(st + m.xa, L.w_attn != nullptr ? st + m.wa : nullptr,
                            reinterpret_cast<uint2*>(L.q8_attn), L.bs_attn, dv_attn, inv_attn, hv, row, sl, C, NB, D,
                            invD, eps, red, n_rows);
    chain_qkv<DT, GP>(reinterpret_cast<const uint16_t*>(st + m.qkv),
                      L.q_norm_w != nullptr ? reinterpret_cast<const uint16_t*>(st + m.qw) : nullptr,
                      L.k_norm_w != nullptr ? reinterpret_cast<const uint16_t*>(st + m.kw) : nullptr,
                      static_cast<uint16_t*>(L.q_out), static_cast<uint16_t*>(L.k_cache),
                      static_cast<uint16_t*>(L.v_cache), cs8, sn8, nsn8, row, p, row_ok, sl, Hq, Hkv, hd, G, eps,
                      n_rows, capacity);
    if (norm_cta)
      chain_norm<DT, K, QM>(st + m.xf, L.w_ffn != nullptr ? st + m.wf : nullptr, reinterpret_cast<uint2*>(L.q8_ffn),
                            L.bs_ffn, dv_ffn, inv_ffn, hv, row, sl, C, NB, D, invD, eps, red + kChainWarps, n_rows);
    chain_act<DT, QM, ACT>(st + m.gu, reinterpret_cast<uint32_t*>(L.act8), L.bs_act, dv_act, row, sl, I4, NBI,
                           n_rows);
    __syncthreads();  // the slot read here is refilled (for it + 2) at the top of it + 1
  }
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int j = t + k * kChainThreads;
    if (j < sl.nc && FRT_IDX_OK(row * C + sl.c0 + j, n_rows * C)) residual[row * C + sl.c0 + j] = hv[k];
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
  int M, C, NB, Hq, Hkv, hd, G, I4, NBI, S, max_pos, capacity;
  float eps;
};

template <int DT, int K, int QM, int GP, int ACT>
frt_status launch_chain(const ChainArgs& a, size_t smem, cudaStream_t st) {
  static std::atomic<int> opted{0};
  auto kern = chain_persistent_kernel<DT, K, QM, GP, ACT>;
  const frt_status os = opt_in_smem(kern, smem, opted);
  if (os != FRT_OK) return os;
  return launch_cluster(kern, dim3((unsigned)(a.M * a.S)), dim3(kChainThreads), smem, st, (unsigned)a.S, a.layers,
                        a.n_layers, a.steps, static_cast<uint4*>(a.residual), a.cos_tab, a.sin_tab, a.positions,
                        a.scales, a.status, a.C, a.NB, a.Hq, a.Hkv, a.hd, a.G, a.I4, a.NBI, a.max_pos, a.capacity,
                        a.eps);
}

template <int DT, int K, int QM, int GP>
frt_status chain_act_dispatch(frt_act act, const ChainArgs& a, size_t smem, cudaStream_t st) {
  switch (act) {
    case FRT_ACT_GELU_TANH: return launch_chain<DT, K, QM, GP, FRT_ACT_GELU_TANH>(a, smem, st);
    case FRT_ACT_SILU: return launch_chain<DT, K, QM, GP, FRT_ACT_SILU>(a, smem, st);
    default: return launch_chain<DT, K, QM, GP, FRT_ACT_RELU2>(a, smem, st);
  }
}

template <int DT, int K, int QM>
frt_status chain_gp_dispatch(int GP, frt_act act, const ChainArgs& a, size_t smem, cudaStream_t st) {
  switch (GP) {
    case 4: return chain_act_dispatch<DT, K, QM, 4>(act, a, smem, st);
    case 8: return chain_act_dispatch<DT, K, QM, 8>(act, a, smem, st);
    default: return chain_act_dispatch<DT, K, QM, 16>(act, a, smem, st);
  }
}

template <int DT>
frt_status chain_dispatch(int K, frt_quant qm, int GP, frt_act act, const ChainArgs& a, size_t smem,
                          cudaStream_t st) {
  const bool blk = qm == FRT_QUANT_BLOCK128;
  switch (K) {
    case 1:
      return blk ? chain_gp_dispatch<DT, 1, FRT_QUANT_BLOCK128>(GP, act, a, smem, st)
                 : chain_gp_dispatch<DT, 1, FRT_QUANT_STATIC>(GP, act, a, smem, st);
    case 2:
      return blk ? chain_gp_dispatch<DT, 2, FRT_QUANT_BLOCK128>(GP, act, a, smem, st)
                 : chain_gp_dispatch<DT, 2, FRT_QUANT_STATIC>(GP, act, a, smem, st);
    default:
      return blk ? chain_gp_dispatch<DT, 4, FRT_QUANT_BLOCK128>(GP, act, a, smem, st)
                 : chain_gp_dispatch<DT, 4, FRT_QUANT_STATIC>(GP, act, a, smem, st);
  }
}

// Largest dynamic shared memory the chain uses (one CTA per SM).
constexpr size_t kChainSmemMax = 200 * 1024;


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
  // supported shapes: D <= 4 * 256 * 8, 16-byte head halves with 4..16 lanes
  // per head (hd % 16 == 0, 64 <= hd <= 256), whole 128-output activation blocks
  if (D > 8192 || hd % 16 != 0 || hd < 64 || hd > 256 || I % 128 != 0) return FRT_ERR_UNSUPPORTED;
  if (M == 0 || n_layers == 0 || steps == 0) return FRT_OK;
  if (!layers || !residual || !cos_tab || !sin_tab || !positions || !scales) return FRT_ERR_INVALID_ARG;
  if (!aligned(layers, 8) || !aligned(residual, 16) || !aligned(cos_tab, 16) || !aligned(sin_tab, 16) ||
      !aligned(positions, 4) || !aligned(scales, 4) || (status && !aligned(status, 4)))
    return FRT_ERR_INVALID_ARG;
  if ((int64_t)M * 8 > 0x7FFFFFFF) return FRT_ERR_UNSUPPORTED;
  const int C = D / 8;
  const int H = Hq + 2 * Hkv;
  const int NBI = I / 128;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                cudaSuccess) {
    (void)cudaGetLastError();
    sms = 148;
  }
  // Cluster size: as many CTAs per row as fill the SMs (at most 8): one runs
  // the norms, the rest share the heads and activation blocks.
  int S = sms / M;
  S = S < 1 ? 1 : S > 8 ? 8 : S;
  const int hd16 = hd / 8;
  if (C > 4 * kChainThreads) return FRT_ERR_UNSUPPORTED;
  const int K = C <= kChainThreads ? 1 : C <= 2 * kChainThreads ? 2 : 4;
  const int G = (hd / 2) / 8;
  int GP = 1;
  while (GP < G) GP *= 2;
  const size_t table = ((size_t)n_layers * sizeof(frt_chain_layer) + 15) / 16 * 16;
  for (;; --S) {
    const int workers = S > 1 ? S - 1 : 1;
    const int hs = (H + workers - 1) / workers;
    const int bsl = (NBI + workers - 1) / workers;
    // the larger of the two roles' stages sizes the shared memory of every CTA
    const StageMap mn(C, S > 1 ? 0 : hs * hd16, hd16, S > 1 ? 0 : bsl * 32);
    const StageMap mw(0, hs * hd16, hd16, bsl * 32);
    const size_t smem = table + (size_t)2 * (mn.len > mw.len ? mn.len : mw.len) * sizeof(uint4);
    if (smem <= kChainSmemMax || S == 1) {
      if (smem > kChainSmemMax) return FRT_ERR_UNSUPPORTED;
      const ChainArgs a{layers, n_layers, steps, residual, cos_tab, sin_tab, positions, scales, status, M, C,
                        (D + 127) / 128, Hq, Hkv, hd, G, I / 4, NBI, S, max_pos, capacity, eps};
      return dt == FRT_F16 ? chain_dispatch<FRT_F16>(K, qm, GP, act, a, smem, stream)
                           : chain_dispatch<FRT_BF16>(K, qm, GP, act, a, smem, stream);
    }
  }
}
