// Device-side helpers shared by the fused-op kernels: 16-bit <-> fp32 packing,
// FP8 e4m3 packing, streaming vector loads and warp reductions.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "frt.h"

namespace frt {

// ------------------------------------------------------------------ PDL --
// Every kernel starts with these two: wait until the grid this launch depends
// on has completed and its writes are visible (a no-op without a programmatic
// dependency), then let the next launch of the stream be scheduled early.
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
};

// Sum of two floats rounded to odd: the nearest of the two fp32 neighbours of
// the exact sum whose last significand bit is 1 (or the exact sum when it is
// representable).  Rounding this value once more to a format with at least two
// fewer significand bits gives the correctly rounded (RNE) exact sum, so
// RN16(add_round_odd(x, r)) == RN16(x + r) with no double-rounding error.
// The error term comes from Knuth's TwoSum.
__device__ __forceinline__ float add_round_odd(float a, float b) {
  const float s = __fadd_rn(a, b);
  const float bb = __fsub_rn(s, a);
  const float err = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
  uint32_t u = __float_as_uint(s);
  if (err != 0.0f && (u & 1u) == 0u) {
    // step one ulp towards the exact value: away from zero when err has the
    // sign of s, towards zero otherwise
    u += ((__float_as_uint(err) ^ u) & 0x80000000u) ? 0xFFFFFFFFu : 1u;
  }
  return __uint_as_float(u);
}

// Knuth's TwoSum: a + b == s + e exactly (fp32, round to nearest).
__device__ __forceinline__ void two_sum(float a, float b, float& s, float& e) {
  s = __fadd_rn(a, b);
  const float bb = __fsub_rn(s, a);
  e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
}

// Compensated (hi, lo) accumulator: hi + lo tracks the exact sum of the
// added terms to ~2^-48 relative.  Adding pairs is commutative bit for bit
// (TwoSum's error term is the unique exact error), so an xor-butterfly gives
// every lane the same pair.
struct Sum2 {
  float hi, lo;
  __device__ __forceinline__ void add(float x) {
    float s, e;
    two_sum(hi, x, s, e);
    hi = s;
    lo = __fadd_rn(lo, e);
  }
  __device__ __forceinline__ void add(const Sum2& o) {
    float s, e;
    two_sum(hi, o.hi, s, e);
    hi = s;
    lo = __fadd_rn(__fadd_rn(lo, o.lo), e);
  }
};

template <int WIDTH>
__device__ __forceinline__ Sum2 group_sum2(Sum2 v) {
#pragma unroll
  for (int o = WIDTH / 2; o > 0; o >>= 1) {
    Sum2 w;
    w.hi = __shfl_xor_sync(0xFFFFFFFFu, v.hi, o);
    w.lo = __shfl_xor_sync(0xFFFFFFFFu, v.lo, o);
    v.add(w);
  }
  return v;
}

// fp32 scale factor r held as an unevaluated pair rhi + rlo (from an fp64
// value).  mul_exact(x, r) = fp32 rounding of x * (rhi + rlo), computed with
// an exact product (TwoProduct via FMA): correctly rounded unless the exact
// product lies within ~2^-48 of an fp32 rounding boundary.
struct Split32 {
  float hi, lo;
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
// theorem) while the quotient and the residual stay in the normal range.
// Outside that range (tiny or huge scales, |y| < 2^-90, zeros) the IEEE
// division is used instead.
struct Divisor {
  float s, inv;
  bool fast;
  __device__ __forceinline__ explicit Divisor(float s_) : s(s_) {
    inv = __frcp_rn(s_);
    const float a = fabsf(s_);
    fast = a >= 0x1p-100f && a <= 0x1p+100f;
  }
  __device__ __forceinline__ float div(float y) const {
    if (!fast || !(fabsf(y) >= 0x1p-90f)) return __fdiv_rn(y, s);  // also zeros: keeps -0
    const float q = y * inv;
    const float r = fmaf(-q, s, y);
    return fmaf(r, inv, q);
  }
};

// ----------------------------------------------------------------- FP8 --
// Two fp32 -> two e4m3 codes (low byte = a), RNE, saturating to +-448.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  return e4m3x2(a, b) | (e4m3x2(c, d) << 16);
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

// --------------------------------------------------------- reductions --
template <int WIDTH>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = WIDTH / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
template <int WIDTH>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
  for (int o = WIDTH / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ float absmax4(float a, float b, float c, float d) {
  return fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(c), fabsf(d)));
}

}  // namespace frt
