// Launch-floor probe and status strings.
#include "frt_host.h"

#include <atomic>

#include "frt_device.cuh"

namespace frt {
namespace {
__global__ void noop_kernel() { pdl_enter(); }

// One CTA per row: the row's 16-byte chunks from src to dst (src may equal
// dst: each chunk is read before it is written, by the same thread).
__global__ void copy_rows_kernel(const uint4* src, uint4* dst, int C) {
  pdl_enter();
  const int64_t base = (int64_t)blockIdx.x * C;
  for (int c = threadIdx.x; c < C; c += blockDim.x)
    if (FRT_IDX_OK(base + c, (int64_t)gridDim.x * C)) dst[base + c] = ld_plain(src + base + c);
}
std::atomic<int> g_pdl{1};
std::atomic<int> g_wait_polls{FRT_DEFAULT_WAIT_POLLS};
}  // namespace

bool pdl_enabled() { return g_pdl.load(std::memory_order_relaxed) != 0; }
int wait_polls() { return g_wait_polls.load(std::memory_order_relaxed); }

}  // namespace frt

extern "C" frt_status frt_noop(int grid, int block, cudaStream_t stream) {
  if (grid < 1 || block < 1 || block > 1024) return FRT_ERR_INVALID_ARG;
  return frt::launch(frt::noop_kernel, dim3(grid), dim3(block), 0, stream);
}

extern "C" frt_status frt_copy_rows(const void* src, void* dst, int rows, int row_bytes, cudaStream_t stream) {
  if (rows < 0 || row_bytes <= 0 || row_bytes % 16 != 0 || row_bytes > (1 << 30)) return FRT_ERR_INVALID_ARG;
  if (rows == 0) return FRT_OK;
  if (!src || !dst || !frt::aligned(src, 16) || !frt::aligned(dst, 16)) return FRT_ERR_INVALID_ARG;
  const int C = row_bytes / 16;
  const int threads = C >= 1024 ? 1024 : (C + 31) / 32 * 32;
  return frt::launch(frt::copy_rows_kernel, dim3(rows), dim3(threads), 0, stream, static_cast<const uint4*>(src),
                     static_cast<uint4*>(dst), C);
}

extern "C" void frt_set_pdl(int enable) { frt::g_pdl.store(enable ? 1 : 0, std::memory_order_relaxed); }

extern "C" int frt_get_pdl(void) { return frt::g_pdl.load(std::memory_order_relaxed); }

extern "C" frt_status frt_set_wait_polls(int polls) {
  if (polls < 0) return FRT_ERR_INVALID_ARG;
  frt::g_wait_polls.store(polls, std::memory_order_relaxed);
  return FRT_OK;
}

extern "C" int frt_get_wait_polls(void) { return frt::g_wait_polls.load(std::memory_order_relaxed); }

extern "C" const char* frt_status_string(frt_status status) {
  switch (status) {
    case FRT_OK: return "FRT_OK";
    case FRT_ERR_INVALID_ARG: return "FRT_ERR_INVALID_ARG: bad size, pointer, alignment or enum";
    case FRT_ERR_UNSUPPORTED: return "FRT_ERR_UNSUPPORTED: shape outside what this build covers";
    case FRT_ERR_CUDA: return "FRT_ERR_CUDA: the kernel launch failed";
    default: return "unknown frt_status";
  }
}

#ifdef FRT_DEBUG_BOUNDS
#include "frt_debug.h"

// Violation count of the bounds-checked build (see frt_device.cuh).
namespace frt {
__device__ unsigned int frt_bounds_violations = 0;
}  // namespace frt

extern "C" frt_status frt_debug_bounds_violations(unsigned int* count) {
  if (count == nullptr) return FRT_ERR_INVALID_ARG;
  unsigned int zero = 0;
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpyFromSymbol(count, frt::frt_bounds_violations, sizeof(unsigned int)) != cudaSuccess ||
      cudaMemcpyToSymbol(frt::frt_bounds_violations, &zero, sizeof(unsigned int)) != cudaSuccess) {
    (void)cudaGetLastError();
    return FRT_ERR_CUDA;
  }
  return FRT_OK;
}
#endif
