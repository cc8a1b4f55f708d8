// Device-side helpers shared by the fused-op kernels: 16-bit <-> fp32 packing,
// FP8 e4m3 packing, streaming vector loads and warp reductions.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "frt.h"

namespace frt {

// ---------------------------------------------------- bounds-checked build --
// Built with FRT_DEBUG_BOUNDS (the separate libfrt_debug.so, relocatable
// device code), every global access of the kernels is preceded by a check of
// its element index against the extent the kernel's own arguments and grid
// give that buffer; an index out of range skips the access and counts one
// violation in frt_bounds_violations (read and cleared on the host with
// frt_debug_bounds_violations).  In the product library the checks are the
// constant true and compile to nothing.
#ifdef FRT_DEBUG_BOUNDS
extern __device__ unsigned int frt_bounds_violations;
__device__ __forceinline__ bool in_range(int64_t i, int64_t n) {
  if (i >= 0 && i < n) return true;
  atomicAdd(&frt_bounds_violations, 1u);
  return false;
}
// index i of an n-element buffer
#define FRT_IDX_OK(i, n) ::frt::in_range((int64_t)(i), (int64_t)(n))
// elements [i, i + len) of an n-element buffer
#define FRT_SPAN_OK(i, len, n) \
  (::frt::in_range((int64_t)(i), (int64_t)(n)) && ::frt::in_range((int64_t)(i) + (int64_t)(len) - 1, (int64_t)(n)))
#else
#define FRT_IDX_OK(i, n) ((void)(i), (void)(n), true)
#define FRT_SPAN_OK(i, len, n) ((void)(i), (void)(len), (void)(n), true)
#endif

// ------------------------------------------------------------------ PDL --
// Every kernel calls this before it touches any memory that the previous
// kernel of the stream may write: wait until the grid this launch depends on
// has completed and its writes are visible (a no-op without a programmatic
// dependency), then let the next launch of the stream be scheduled early.
// Loads of constant inputs (norm weights, RoPE tables, positions, scales)
// may come before it: the next kernel is launched only once every CTA of this
// one has passed the wait, so those early loads overlap the previous kernel
// alone, which never writes them.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" :::);
}

// -------------------------------------------------------------- 16-bit --
// Two 16-bit values packed in one 32-bit word, element 0 in the low half.
template <int DT>
struct Pack16;

template <>
struct Pack16<FRT_F16> {
  static __device__ __forceinline__ float2 to_float2(uint32_t w) {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    return __half22float2(h);
  }
  static __device__ __forceinline__ uint32_t from_float2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  // a * b + c on both halves, the exact value rounded once (round to nearest
  // even, subnormals kept): IEEE fusedMultiplyAdd in binary16.
  static __device__ __forceinline__ uint32_t fma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
  }
  static constexpr uint32_t kOnes = 0x3C003C00u;  // (1.0, 1.0)
};

template <>
struct Pack16<FRT_BF16> {
  static __device__ __forceinline__ float2 to_float2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  }
  static __device__ __forceinline__ uint32_t from_float2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  // a * b + c on both halves, the exact value rounded once to bfloat16
  // (round to nearest even).
  static __device__ __forceinline__ uint32_t fma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
  }
  static constexpr uint32_t kOnes = 0x3F803F80u;  // (1.0, 1.0)
};

// 1 / sqrt(x) in fp64, to ~1e-16 relative (not correctly rounded): an fp32
// estimate refined by two Newton steps in fp64.  Every lane can afford it
// (about a dozen instructions), unlike a correctly rounded sqrt + divide.
// Arguments outside the fp32 range of the estimate take the IEEE path.
__device__ __forceinline__ double rsqrt_f64(double x) {
  if (!(x >= 0x1p-120 && x <= 0x1p+120)) return 1.0 / sqrt(x);
  double r = (double)rsqrtf((float)x);
  r = r * fma(-0.5 * x * r, r, 1.5);
  r = r * fma(-0.5 * x * r, r, 1.5);
  return r;
}

// fp32 scale factor r held as an unevaluated pair rhi + rlo (from an fp64
// value).  mul(x) = fp32 rounding of x * (rhi + rlo), computed with
// an exact product (TwoProduct via FMA): correctly rounded unless the exact
// product lies within ~2^-48 of an fp32 rounding boundary.
struct Split32 {
  float hi, lo;
  __device__ __forceinline__ Split32() : hi(0.0f), lo(0.0f) {}
  __device__ __forceinline__ explicit Split32(double r) {
    hi = __double2float_rn(r);
    lo = __double2float_rn(r - (double)hi);
  }
  __device__ __forceinline__ float mul(float x) const {
    const float p = x * hi;
    const float e = fmaf(x, hi, -p);
    return p + fmaf(x, lo, e);
  }
};

// y / s rounded to nearest in fp32, from inv = RN(1/s): one FMA residual step
// on the quotient estimate gives the correctly rounded quotient (Markstein's
// theorem) while the residual y - q*s is exactly representable, which holds
// for positive scales in [2^-100, 2^100] and |y| >= 2^-100 (for smaller |y|
// the result can be one ulp off; zeros keep their sign).  Scales outside that
// range (`fast` false) use the IEEE division for every element; callers
// branch on `fast` once, outside their element loops.
struct Divisor {
  float s, inv;
  bool fast;
  __device__ __forceinline__ explicit Divisor(float s_) : s(s_) {
    inv = __frcp_rn(s_);
    fast = s_ >= 0x1p-100f && s_ <= 0x1p+100f;
  }
  // from a reciprocal formed once elsewhere (inv_ must be RN(1/s_))
  __device__ __forceinline__ Divisor(float s_, float inv_) : s(s_), inv(inv_) {
    fast = s_ >= 0x1p-100f && s_ <= 0x1p+100f;
  }
  __device__ __forceinline__ float div(float y) const {
    const float q = y * inv;
    const float r = fmaf(-q, s, y);
    const float v = fmaf(r, inv, q);
    // s > 0, so the quotient has the sign of y (this also keeps -0)
    return __uint_as_float((__float_as_uint(v) & 0x7FFFFFFFu) | (__float_as_uint(y) & 0x80000000u));
  }
  __device__ __forceinline__ float div_slow(float y) const { return __fdiv_rn(y, s); }
};

// Block scale RN(amax / 448) of the block-128 FP8 mode (1 for an all-zero
// block): Markstein's correction with the correctly rounded reciprocal of 448,
// q = RN(amax RN(1/448)), r = amax - 448 q (exact), RN(q + r RN(1/448)), which
// is the IEEE quotient for amax >= 2^-100 (tiny blocks take the IEEE division).
constexpr float kInv448 = 1.0f / 448.0f;
__device__ __forceinline__ float block_scale_448(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  if (amax < 0x1p-100f) return __fdiv_rn(amax, 448.0f);
  const float q = amax * kInv448;
  const float r = fmaf(-q, 448.0f, amax);
  return fmaf(r, kInv448, q);
}

// Eight values -> eight e4m3 codes of y / s (low byte first).
__device__ __forceinline__ uint2 quant8(const float* y, const Divisor& dv);
// Four values -> four e4m3 codes of y / s.
__device__ __forceinline__ uint32_t quant4(const float* y, const Divisor& dv);

// ----------------------------------------------------------------- FP8 --
// Two fp32 -> two e4m3 codes (low byte = a), RNE, saturating to +-448.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  return e4m3x2(a, b) | (e4m3x2(c, d) << 16);
}

__device__ __forceinline__ uint32_t quant4(const float* y, const Divisor& dv) {
  if (dv.fast) return e4m3x4(dv.div(y[0]), dv.div(y[1]), dv.div(y[2]), dv.div(y[3]));
  return e4m3x4(dv.div_slow(y[0]), dv.div_slow(y[1]), dv.div_slow(y[2]), dv.div_slow(y[3]));
}

__device__ __forceinline__ uint2 quant8(const float* y, const Divisor& dv) {
  return make_uint2(quant4(y, dv), quant4(y + 4, dv));
}
// Eight values already divided by the scale -> eight e4m3 codes.
__device__ __forceinline__ uint2 e4m3x8(const float* v) {
  return make_uint2(e4m3x4(v[0], v[1], v[2], v[3]), e4m3x4(v[4], v[5], v[6], v[7]));
}

// ----------------------------------------------------------------- NVFP4 --
// e2m1 elements in 16-element blocks, each block scaled by an unsigned e4m3
// factor sf and the per-tensor fp32 global scale gs (y ~ e2m1 * sf * gs).
// Decisions in fp32, scaling by correctly rounded reciprocals:
//   rden = RN(1 / RN(6 gs)), sf = e4m3(RN(amax * rden)),
//   eff = RN(sf * gs), reff = RN(1 / eff), code = e2m1(RN(y * reff));
// sf == 0 gives zero codes.  gs must lie in [2^-100, 2^100].

// Two fp32 -> two e2m1 codes in one byte (a in the low nibble), RNE, saturating.
__device__ __forceinline__ uint32_t e2m1x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp4x2(make_float2(a, b), __NV_E2M1, cudaRoundNearest);
}
// Exact value of an e4m3 code (e4m3 is a subset of binary16).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
  return __half2float(__half(h));
}
// Block scale: returns the sf code and the reciprocal of eff = RN(sf * gs)
// (0 when sf is 0).
__device__ __forceinline__ uint32_t nvfp4_scale(float amax, float rden, float gs, float* reff) {
  const uint32_t sf = e4m3x2(amax * rden, 0.0f) & 0xFFu;
  const float eff = e4m3_value(sf) * gs;
  *reff = eff > 0.0f ? __frcp_rn(eff) : 0.0f;
  return sf;
}
// The same with RN(1 / eff) looked up per sf code: reff_of[sf] for all 256
// codes, filled once per CTA by nvfp4_reff_entry.
__device__ __forceinline__ float nvfp4_reff_entry(uint32_t sf, float gs) {
  const float eff = e4m3_value(sf) * gs;
  return eff > 0.0f ? __frcp_rn(eff) : 0.0f;
}
__device__ __forceinline__ uint32_t nvfp4_scale_lookup(float amax, float rden, const float* reff_of, float* reff) {
  const uint32_t sf = e4m3x2(amax * rden, 0.0f) & 0xFFu;
  *reff = reff_of[sf];
  return sf;
}
// N (4 or 8) values -> N e2m1 codes of y * reff, element 0 in the low nibble.
template <int N>
__device__ __forceinline__ uint32_t nvfp4_codes(const float* y, float reff) {
  uint32_t w = 0;
#pragma unroll
  for (int e = 0; e < N; e += 2) w |= e2m1x2(y[e] * reff, y[e + 1] * reff) << (4 * e);
  return w;
}
// Byte offset of scale factor (row r, column c) of an [M, n_cols] scale
// matrix in the 128x4-swizzled layout read by block-scaled tensor-core GEMMs:
// 512-byte atoms of 128 rows x 4 columns, row-major over (r / 128, c / 4);
// inside an atom, row 32 i + k and column l sit at byte 16 k + 4 i + l.
__device__ __forceinline__ int64_t sf_offset_swizzled(int64_t r, int c, int n_cols) {
  const int64_t atom = (r >> 7) * (int64_t)((n_cols + 3) >> 2) + (c >> 2);
  const int rr = (int)(r & 127);
  return atom * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (c & 3);
}

// ------------------------------------------------------------ memory ops --
// Read-once input: bypass L1 allocation.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ld_stream(const uint2* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
// Plain coherent 16-byte load (used where the buffer may also be written by
// the same kernel, e.g. an in-place residual).
__device__ __forceinline__ uint4 ld_plain(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

// ------------------------------------------------------ bulk copies (TMA) --
// 1-D bulk copies between global and shared memory (cp.async.bulk), completed
// through an mbarrier.  Addresses must be 16-byte aligned and sizes multiples
// of 16 bytes.
__device__ __forceinline__ unsigned smem_addr(const void* p) { return (unsigned)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
// Makes the initialised barrier visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned phase) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(phase)
      : "memory");
  return ok != 0;
}
// Waits for `phase` of the barrier with a bound on the number of polls.
// Returns false if the bound ran out (the caller reports it and gives up).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned phase, int max_polls) {
  for (int i = 0; i < max_polls; ++i)
    if (mbar_try_wait(bar, phase)) return true;
  return false;
}
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gmem_src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void bulk_store(void* gmem_dst, const void* smem_src, unsigned bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst),
               "r"(smem_addr(smem_src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Blocks until the committed bulk stores have finished reading shared memory
// (the stores themselves complete before the grid does).
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Orders this thread's generic-proxy shared-memory writes before later
// bulk-copy (async-proxy) reads of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------- activations --
// act(g) in fp32 on packed pairs of gates.  GELU-tanh uses
// 0.5 (1 + tanh(z)) = 1 / (1 + exp(-2 z)), z = sqrt(2/pi) (g + 0.044715 g^3),
// and SiLU is g / (1 + exp(-g)).  exp(x) is formed as 2^(x log2 e): the
// product with log2 e is folded into the polynomial's constants and 2^t is
// the special-function unit's ex2 (relative error about 2^-22), the quotient
// g / (1 + e) a multiply by its rcp (about one ulp); both far below the
// half-step of an FP8 or e2m1 code.  t is capped at 115 (2^115 ~ e^80) so the
// denominator stays finite; the result is ~0 there either way.  The other
// steps are fp32 multiplies / FMAs two at a time (mul/fma .f32x2), each half
// rounded as the scalar operation.
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kGeluC0 = (float)(-2.0 * 0.7978845608028654 * 1.4426950408889634);
constexpr float kGeluC1 = (float)(-2.0 * 0.7978845608028654 * 0.044715 * 1.4426950408889634);
constexpr float kExp2Cap = 115.0f;

__device__ __forceinline__ float ex2_approx(float t) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(t));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// g / (1 + 2^t) per half, t capped
__device__ __forceinline__ float2 div_one_plus_exp2(float2 g, float2 t) {
  const float2 e = make_float2(ex2_approx(fminf(t.x, kExp2Cap)), ex2_approx(fminf(t.y, kExp2Cap)));
  const float2 d = __fadd2_rn(e, make_float2(1.0f, 1.0f));
  return __fmul2_rn(g, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

template <int ACT>
__device__ __forceinline__ float2 act2(float2 g) {
  if (ACT == FRT_ACT_RELU2) {
    const float2 r = make_float2(fmaxf(g.x, 0.0f), fmaxf(g.y, 0.0f));
    return __fmul2_rn(r, r);
  } else if (ACT == FRT_ACT_SILU) {
    return div_one_plus_exp2(g, __fmul2_rn(g, make_float2(-kLog2e, -kLog2e)));
  } else {
    const float2 p = __ffma2_rn(__fmul2_rn(g, g), make_float2(kGeluC1, kGeluC1), make_float2(kGeluC0, kGeluC0));
    return div_one_plus_exp2(g, __fmul2_rn(g, p));
  }
}

// act(g) * u for the (gate, up) pairs held in two packed 16-bit words.
template <int DT, int ACT>
__device__ __forceinline__ float2 act_mul2(uint32_t w0, uint32_t w1) {
  const float2 p0 = Pack16<DT>::to_float2(w0), p1 = Pack16<DT>::to_float2(w1);
  return __fmul2_rn(act2<ACT>(make_float2(p0.x, p1.x)), make_float2(p0.y, p1.y));
}

// --------------------------------------------------------- reductions --
template <int WIDTH>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = WIDTH / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// max |v| over the 32 lanes of the warp in one instruction (sm_100's f32
// redux; NaN inputs are ignored, as fmaxf does).  Every lane must call it.
__device__ __forceinline__ float warp_max_abs(float v) {
  float r;
  asm volatile("redux.sync.max.abs.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// max |v| over each 16-lane half of the warp: two warp-wide f32 reductions,
// each seeing only one half's values (the other half contributes 0).
// Every lane must call it.
__device__ __forceinline__ float half_warp_max_abs(float v) {
  const bool upper = (threadIdx.x & 16) != 0;
  const float lo = warp_max_abs(upper ? 0.0f : v);
  const float hi = warp_max_abs(upper ? v : 0.0f);
  return upper ? hi : lo;
}

__device__ __forceinline__ float absmax4(float a, float b, float c, float d) {
  return fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(c), fabsf(d)));
}

// ------------------------------------------------- q/k head arithmetic --
// One lane's share of a head: NP packed fp32 pairs of the first half (a,
// elements j0 .. j0 + 2NP - 1) and of the second half (b, the rotate-half
// partners j0 + hd/2 ...).  Blackwell issues two fp32 multiplies or FMAs per
// instruction (mul/fma .f32x2); each half of a pair is rounded to nearest
// exactly as the scalar operation, so only the order of the sum of squares
// (two interleaved partial sums) depends on the packing.
template <int DT, int NP>
__device__ __forceinline__ void unpack_pairs(const uint32_t* w, float2* f) {
#pragma unroll
  for (int e = 0; e < NP; ++e) f[e] = Pack16<DT>::to_float2(w[e]);
}

template <int DT, int NP>
__device__ __forceinline__ void pack_pairs(const float2* f, uint32_t* w) {
#pragma unroll
  for (int e = 0; e < NP; ++e) w[e] = Pack16<DT>::from_float2(f[e].x, f[e].y);
}

template <int NP>
__device__ __forceinline__ float sum_squares_pairs(const float2* a, const float2* b) {
  float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int e = 0; e < NP; ++e) {
    acc = __ffma2_rn(a[e], a[e], acc);
    acc = __ffma2_rn(b[e], b[e], acc);
  }
  return acc.x + acc.y;
}

// RMSNorm scale of a head, 1 / sqrt(ss * inv_n + eps) with inv_n = RN(1/n)
// (exact for power-of-two n): the hardware reciprocal square root, relative
// error about 2^-22, far below the half-ulp of the 16-bit outputs.
__device__ __forceinline__ float head_rstd(float ss, float inv_n, float eps) {
  return rsqrtf(fmaf(ss, inv_n, eps));
}

// x <- (x * r) * w per element (the product with r rounded first).
template <int NP>
__device__ __forceinline__ void scale_pairs(float2* x, float r, const float2* w) {
  const float2 rr = make_float2(r, r);
#pragma unroll
  for (int e = 0; e < NP; ++e) x[e] = __fmul2_rn(__fmul2_rn(x[e], rr), w[e]);
}

// Rotate-half RoPE: o1 = a cos - b sin, o2 = b cos + a sin, each one FMA on
// the rounded sine product; nsn holds -sin so that no operand needs negating.
template <int NP>
__device__ __forceinline__ void rope_pairs(const float2* a, const float2* b, const float2* cs, const float2* sn,
                                           const float2* nsn, float2* o1, float2* o2) {
#pragma unroll
  for (int e = 0; e < NP; ++e) {
    o1[e] = __ffma2_rn(a[e], cs[e], __fmul2_rn(b[e], nsn[e]));
    o2[e] = __ffma2_rn(b[e], cs[e], __fmul2_rn(a[e], sn[e]));
  }
}

template <int NP>
__device__ __forceinline__ void mul_pairs(float2* x, float r) {
  const float2 rr = make_float2(r, r);
#pragma unroll
  for (int e = 0; e < NP; ++e) x[e] = __fmul2_rn(x[e], rr);
}

// A lane's cos/sin slice (2 NP fp32 each, 16-byte aligned) as packed pairs,
// with the negated sine.
template <int NP>
__device__ __forceinline__ void load_rope_pairs(const float* c, const float* s, float2* cs, float2* sn,
                                                float2* nsn) {
#pragma unroll
  for (int e = 0; e < NP; e += 2) {
    const float4 tc = *reinterpret_cast<const float4*>(c + 2 * e);
    const float4 ts = *reinterpret_cast<const float4*>(s + 2 * e);
    cs[e] = make_float2(tc.x, tc.y);
    cs[e + 1] = make_float2(tc.z, tc.w);
    sn[e] = make_float2(ts.x, ts.y);
    sn[e + 1] = make_float2(ts.z, ts.w);
    nsn[e] = make_float2(-ts.x, -ts.y);
    nsn[e + 1] = make_float2(-ts.z, -ts.w);
  }
}

}  // namespace frt
