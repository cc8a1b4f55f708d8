// Launch-floor probe and status strings.
#include "frt_host.h"

namespace frt {
namespace {
__global__ void noop_kernel() {}
}  // namespace
}  // namespace frt

extern "C" frt_status frt_noop(int grid, int block, cudaStream_t stream) {
  if (grid < 1 || block < 1 || block > 1024) return FRT_ERR_INVALID_ARG;
  frt::noop_kernel<<<grid, block, 0, stream>>>();
  return frt::launch_status();
}

extern "C" const char* frt_status_string(frt_status status) {
  switch (status) {
    case FRT_OK: return "FRT_OK";
    case FRT_ERR_INVALID_ARG: return "FRT_ERR_INVALID_ARG: bad size, pointer, alignment or enum";
    case FRT_ERR_UNSUPPORTED: return "FRT_ERR_UNSUPPORTED: shape outside what this build covers";
    case FRT_ERR_CUDA: return "FRT_ERR_CUDA: the kernel launch failed";
    default: return "unknown frt_status";
  }
}
