// Launch-floor probe and status strings.
#include "frt_host.h"

#include <atomic>

#include "frt_device.cuh"

namespace frt {
namespace {
__global__ void noop_kernel() { pdl_enter(); }
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
