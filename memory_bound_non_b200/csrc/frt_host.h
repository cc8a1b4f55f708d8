// Host-side helpers for argument validation and launch status.
#pragma once

#include <cstdint>

#include <atomic>
#include <cuda_runtime.h>

#include <cuda_runtime_api.h>

#include "frt.h"

namespace frt {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline bool valid_dtype(frt_dtype dt) { return dt == FRT_F16 || dt == FRT_BF16; }
inline bool valid_quant(frt_quant q) { return q == FRT_QUANT_STATIC || q == FRT_QUANT_BLOCK128; }

// Status of the launch just issued on this thread.
inline frt_status launch_status() { return cudaGetLastError() == cudaSuccess ? FRT_OK : FRT_ERR_CUDA; }

// Process-wide switch for programmatic dependent launch (frt_set_pdl).
bool pdl_enabled();

// Process-wide bound on the polls of a kernel's bulk-copy barrier wait
// (frt_set_wait_polls).
int wait_polls();

// Launch `kernel` on `stream`, with programmatic stream serialisation when
// PDL is on: the kernel may then be scheduled while the previous kernel of the
// stream still runs, and waits for it (griddepcontrol.wait) before its first
// memory access.
template <typename... KArgs, typename... Args>
inline frt_status launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                         Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return FRT_ERR_CUDA;
  }
  return launch_status();
}

// As launch(), with the grid grouped into thread-block clusters of
// `cluster_x` CTAs along x (co-scheduled; they share distributed shared memory).
template <typename... KArgs, typename... Args>
inline frt_status launch_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                 unsigned cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return FRT_ERR_CUDA;
  }
  return launch_status();
}

// Output modes of the quantising kernels beyond the ABI's FP8 modes: NVFP4
// with row-major or 128x4-swizzled scale factors (internal template values).
constexpr int kQuantNvfp4Rows = 2;
constexpr int kQuantNvfp4Swizzled = 3;

// Checks shared by the two FP8-producing ops: the pointer the quant mode needs.
inline bool quant_args_ok(frt_quant qm, const float* static_scale, const float* block_scales) {
  if (qm == FRT_QUANT_STATIC) return static_scale != nullptr && aligned(static_scale, 4);
  return block_scales != nullptr && aligned(block_scales, 4);
}

// Raises a kernel's dynamic shared memory limit to `bytes` once (the largest
// size seen so far is kept in `opted`); needed above the 48 KB default.
template <typename Kern>
frt_status opt_in_smem(Kern kern, size_t bytes, std::atomic<int>& opted) {
  if ((int)bytes > opted.load(std::memory_order_relaxed)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess) {
      (void)cudaGetLastError();
      return FRT_ERR_CUDA;
    }
    int cur = opted.load(std::memory_order_relaxed);
    while ((int)bytes > cur && !opted.compare_exchange_weak(cur, (int)bytes)) {
    }
  }
  return FRT_OK;
}

// Validation shared by the NVFP4 producers: scale-factor layout, the global
// scale pointer, and the packed-code and scale-factor outputs.
inline bool nvfp4_args_ok(frt_sf_layout layout, const float* global_scale, const void* out_fp4, const void* out_sf,
                          uintptr_t code_align) {
  if (layout != FRT_SF_ROW_MAJOR && layout != FRT_SF_SWIZZLED_128X4) return false;
  return global_scale != nullptr && aligned(global_scale, 4) && out_fp4 != nullptr && out_sf != nullptr &&
         aligned(out_fp4, code_align);
}

}  // namespace frt
