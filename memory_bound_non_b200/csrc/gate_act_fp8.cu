// Op (c): gated activation on an interleaved gate/up buffer + FP8 e4m3.
//
// "Falcon-Perception inference optimisation", third technique: gate and up
// come out of one GEMM interleaved as [g0,u0,g1,u1,...]; one kernel reads each
// adjacent pair, forms act(g) * u and writes once, so the [M, 2I] transient is
// read once and the output is half its width.  "FlashRT kernel fusion", §二
// steps 8-10 and "sm89 prefill FFN megakernel", Phase 2 add the FP8 quant
// (static, or per-token block-128 scales) to the same pass.
//
// Mapping (B200): a 16-byte load holds 4 (g, u) pairs -> 4 outputs -> one
// 32-bit store of 4 codes, so one warp-wide load covers exactly one 128-column
// scale block (512 contiguous input bytes, 128 output bytes) and the block's
// amax is one warp-wide f32 redux.  Each warp owns U consecutive blocks of the
// flattened (row, block) index space and issues all U loads before computing,
// which keeps enough bytes in flight per SM to saturate HBM.
#include <cmath>

#include "frt_device.cuh"
#include "frt_host.h"

namespace frt {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// Scale blocks per warp: 4 on large batches (each warp keeps four loads in
// flight), 1 on small ones (latency-bound: as many warps as blocks).
constexpr int kU = 4;
constexpr int64_t kSmallBlocks = 148 * kWarps * 4;  // at most 4 CTAs per SM with one block per warp
static_assert(kThreads == 256, "the NVFP4 reciprocal table takes one sf code per thread");

// Six CTAs (48 warps) per SM need at most 40 registers a thread; the
// block-128 and row-major NVFP4 forms would take 43-44 unasked and drop to
// five (the swizzled NVFP4 form would spill at 40 and keeps five).
template <int QM, bool FULL>
constexpr int gate_min_blocks() {
  return (QM == FRT_QUANT_BLOCK128 || QM == kQuantNvfp4Rows) && FULL ? 6 : 1;
}

template <int DT, int ACT, int QM, bool FULL, int U>
__global__ void __launch_bounds__(kThreads, gate_min_blocks<QM, FULL>()) gate_act_fp8_kernel(const uint4* __restrict__ gu,
                                                                 uint32_t* __restrict__ q,
                                                                 const float* __restrict__ static_scale,
                                                                 float* __restrict__ block_scales,
                                                                 int64_t total_blocks, int NB, int C4) {
  // Constant inputs before the wait for the previous kernel: static FP8 the
  // scale; NVFP4 the global scale gs, RN(1 / RN(6 gs)) and RN(1 / RN(sf * gs))
  // for each of the 256 sf codes (one per thread).
  const float gs = QM >= kQuantNvfp4Rows && FRT_IDX_OK(0, 1) ? __ldg(static_scale) : 0.0f;
  const float rden = QM >= kQuantNvfp4Rows ? __frcp_rn(6.0f * gs) : 0.0f;
  const Divisor dv_static(QM == FRT_QUANT_STATIC && FRT_IDX_OK(0, 1) ? __ldg(static_scale) : 1.0f);
  __shared__ float reff_of[QM >= kQuantNvfp4Rows ? kThreads : 1];
  if (QM >= kQuantNvfp4Rows) reff_of[threadIdx.x] = nvfp4_reff_entry(threadIdx.x, gs);
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t gb0 = warp * U;
  // extents: M = total_blocks / NB rows of C4 16-byte input chunks (and as
  // many 4-byte output words); block scales [M, NB]
  const int64_t n_chunks = total_blocks / NB * C4;

  // Load phase: chunk `lane` of each of the U blocks (4 outputs = 16 bytes).
  // FULL (I % 128 == 0): every block is 32 whole chunks, so the flat chunk
  // index is just 32 * block + lane; otherwise rows end in a partial block
  // and the (row, block) position is tracked.
  uint4 v[U];
  int64_t idx[U];
  bool valid[U];
  if (FULL) {
    const int64_t i0 = gb0 * 32 + lane;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      valid[u] = gb0 + u < total_blocks;
      idx[u] = i0 + 32 * u;  // same index for the input (uint4) and output (uint32) views
      if (valid[u] && FRT_IDX_OK(idx[u], n_chunks)) v[u] = ld_stream(gu + idx[u]);
    }
  } else {
    int64_t row = gb0 / NB;
    int b = (int)(gb0 - row * NB);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int chunk = b * 32 + lane;  // chunk index within the row (4 outputs each)
      valid[u] = gb0 + u < total_blocks && chunk < C4;
      idx[u] = row * C4 + chunk;
      if (valid[u] && FRT_IDX_OK(idx[u], n_chunks)) v[u] = ld_stream(gu + idx[u]);
      if (++b == NB) {
        b = 0;
        ++row;
      }
    }
  }

  if (QM >= kQuantNvfp4Rows) __syncthreads();  // the reciprocal table is complete

#pragma unroll
  for (int u = 0; u < U; ++u) {
    float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (valid[u]) {
      const uint32_t* w = reinterpret_cast<const uint32_t*>(&v[u]);  // (gate, up) pairs
      const float2 a01 = act_mul2<DT, ACT>(w[0], w[1]), a23 = act_mul2<DT, ACT>(w[2], w[3]);
      a[0] = a01.x;
      a[1] = a01.y;
      a[2] = a23.x;
      a[3] = a23.y;
    }
    // code = e4m3(a / s) with the quotient correctly rounded in fp32
    if (QM == FRT_QUANT_BLOCK128) {
      const float am = warp_max_abs(absmax4(a[0], a[1], a[2], a[3]));
      const float sb = block_scale_448(am);
      const int64_t gb = gb0 + u;
      if (lane == 0 && gb < total_blocks && FRT_IDX_OK(gb, total_blocks))
        block_scales[gb] = sb;  // [M, NB] row-major == flat block index
      if (valid[u] && FRT_IDX_OK(idx[u], n_chunks)) q[idx[u]] = quant4(a, Divisor(sb));
    } else if (QM >= kQuantNvfp4Rows) {
      // NVFP4: a 16-output block is 4 consecutive lanes; codes leave as 16 bits
      // per lane, the scale factor from the block's first lane.  q /
      // block_scales carry the code and sf pointers.
      float am = absmax4(a[0], a[1], a[2], a[3]);
      am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
      am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 2));
      float reff;
      const uint32_t sf = nvfp4_scale_lookup(am, rden, reff_of, &reff);
      if (valid[u]) {
        if (FRT_IDX_OK(idx[u], n_chunks)) reinterpret_cast<uint16_t*>(q)[idx[u]] = (uint16_t)nvfp4_codes<4>(a, reff);
        if ((lane & 3) == 0) {
          uint8_t* sfo = reinterpret_cast<uint8_t*>(block_scales);
          if (QM == kQuantNvfp4Rows) {
            // flat output index / 16 == row * (I/16) + column block
            if (FRT_IDX_OK(idx[u] >> 2, n_chunks >> 2)) sfo[idx[u] >> 2] = (uint8_t)sf;
          } else {
            const int64_t row = idx[u] / C4;
            const int64_t o = sf_offset_swizzled(row, (int)((idx[u] - row * C4) >> 2), C4 >> 2);
            if (FRT_IDX_OK(o, (total_blocks / NB + 127) / 128 * 128 * (((C4 >> 2) + 3) / 4) * 4)) sfo[o] = (uint8_t)sf;
          }
        }
      }
    } else if (valid[u] && FRT_IDX_OK(idx[u], n_chunks)) {
      q[idx[u]] = quant4(a, dv_static);
    }
  }
}

template <int DT, int ACT, int QM, int U>
frt_status launch_u(bool full, const uint4* in, uint32_t* out, const float* ss, float* bs, int64_t total, int NB,
                    int C4, cudaStream_t st) {
  const int64_t warps = (total + U - 1) / U;
  const dim3 grid((unsigned)((warps + kWarps - 1) / kWarps));
  return full ? launch(gate_act_fp8_kernel<DT, ACT, QM, true, U>, grid, dim3(kThreads), 0, st, in, out, ss, bs,
                       total, NB, C4)
              : launch(gate_act_fp8_kernel<DT, ACT, QM, false, U>, grid, dim3(kThreads), 0, st, in, out, ss, bs,
                       total, NB, C4);
}

template <int DT, int ACT, int QM>
frt_status launch_q(bool full, const uint4* in, uint32_t* out, const float* ss, float* bs, int64_t total, int NB,
                    int C4, cudaStream_t st) {
  return total <= kSmallBlocks ? launch_u<DT, ACT, QM, 1>(full, in, out, ss, bs, total, NB, C4, st)
                               : launch_u<DT, ACT, QM, kU>(full, in, out, ss, bs, total, NB, C4, st);
}

template <int DT, int ACT>
frt_status launch_act(int qm, const void* gu, uint8_t* q, const float* ss, float* bs, int64_t total, int NB, int C4,
                      cudaStream_t st) {
  const uint4* in = static_cast<const uint4*>(gu);
  uint32_t* out = reinterpret_cast<uint32_t*>(q);
  const bool full = C4 == NB * 32;
  switch (qm) {
    case FRT_QUANT_STATIC: return launch_q<DT, ACT, FRT_QUANT_STATIC>(full, in, out, ss, bs, total, NB, C4, st);
    case FRT_QUANT_BLOCK128: return launch_q<DT, ACT, FRT_QUANT_BLOCK128>(full, in, out, ss, bs, total, NB, C4, st);
    case kQuantNvfp4Rows: return launch_q<DT, ACT, kQuantNvfp4Rows>(full, in, out, ss, bs, total, NB, C4, st);
    default: return launch_q<DT, ACT, kQuantNvfp4Swizzled>(full, in, out, ss, bs, total, NB, C4, st);
  }
}

template <int DT>
frt_status launch_dt(frt_act act, int qm, const void* gu, uint8_t* q, const float* ss, float* bs,
                     int64_t total, int NB, int C4, cudaStream_t st) {
  switch (act) {
    case FRT_ACT_GELU_TANH: return launch_act<DT, FRT_ACT_GELU_TANH>(qm, gu, q, ss, bs, total, NB, C4, st);
    case FRT_ACT_SILU: return launch_act<DT, FRT_ACT_SILU>(qm, gu, q, ss, bs, total, NB, C4, st);
    default: return launch_act<DT, FRT_ACT_RELU2>(qm, gu, q, ss, bs, total, NB, C4, st);
  }
}

}  // namespace
}  // namespace frt

extern "C" frt_status frt_gate_act_fp8(const void* gate_up, uint8_t* out_fp8, const float* static_scale,
                                       float* block_scales, int M, int I, frt_act act, frt_dtype dt, frt_quant qm,
                                       cudaStream_t stream) {
  using namespace frt;
  if (M < 0 || I <= 0 || I % 4 != 0) return FRT_ERR_INVALID_ARG;
  if (!valid_dtype(dt) || !valid_quant(qm)) return FRT_ERR_INVALID_ARG;
  if (act != FRT_ACT_GELU_TANH && act != FRT_ACT_SILU && act != FRT_ACT_RELU2) return FRT_ERR_INVALID_ARG;
  if (M == 0) return FRT_OK;
  if (!gate_up || !out_fp8 || !aligned(gate_up, 16) || !aligned(out_fp8, 4)) return FRT_ERR_INVALID_ARG;
  if (!quant_args_ok(qm, static_scale, block_scales)) return FRT_ERR_INVALID_ARG;
  const int NB = (I + 127) / 128;
  const int C4 = I / 4;
  const int64_t total = (int64_t)M * NB;
  const int64_t grid = (total + (int64_t)kU * kWarps - 1) / ((int64_t)kU * kWarps);
  if (grid > 0x7FFFFFFF) return FRT_ERR_UNSUPPORTED;
  if (dt == FRT_F16)
    return launch_dt<FRT_F16>(act, qm, gate_up, out_fp8, static_scale, block_scales, total, NB, C4, stream);
  return launch_dt<FRT_BF16>(act, qm, gate_up, out_fp8, static_scale, block_scales, total, NB, C4, stream);
}

extern "C" frt_status frt_gate_act_nvfp4(const void* gate_up, uint8_t* out_fp4, uint8_t* out_sf,
                                         const float* global_scale, int M, int I, frt_act act, frt_dtype dt,
                                         frt_sf_layout sf_layout, cudaStream_t stream) {
  using namespace frt;
  if (M < 0 || I <= 0 || I % 16 != 0 || !valid_dtype(dt)) return FRT_ERR_INVALID_ARG;
  if (act != FRT_ACT_GELU_TANH && act != FRT_ACT_SILU && act != FRT_ACT_RELU2) return FRT_ERR_INVALID_ARG;
  if (sf_layout != FRT_SF_ROW_MAJOR && sf_layout != FRT_SF_SWIZZLED_128X4) return FRT_ERR_INVALID_ARG;
  if (M == 0) return FRT_OK;
  if (!gate_up || !aligned(gate_up, 16)) return FRT_ERR_INVALID_ARG;
  if (!nvfp4_args_ok(sf_layout, global_scale, out_fp4, out_sf, 2)) return FRT_ERR_INVALID_ARG;
  const int NB = (I + 127) / 128;
  const int C4 = I / 4;
  const int64_t total = (int64_t)M * NB;
  const int64_t grid = (total + (int64_t)kU * kWarps - 1) / ((int64_t)kU * kWarps);
  if (grid > 0x7FFFFFFF) return FRT_ERR_UNSUPPORTED;
  const int qm = sf_layout == FRT_SF_ROW_MAJOR ? kQuantNvfp4Rows : kQuantNvfp4Swizzled;
  float* sf = reinterpret_cast<float*>(out_sf);  // the kernel's scale pointer carries the sf bytes
  if (dt == FRT_F16)
    return launch_dt<FRT_F16>(act, qm, gate_up, out_fp4, global_scale, sf, total, NB, C4, stream);
  return launch_dt<FRT_BF16>(act, qm, gate_up, out_fp4, global_scale, sf, total, NB, C4, stream);
}
