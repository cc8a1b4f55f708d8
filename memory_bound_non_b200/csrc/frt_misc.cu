// Launch-floor probe and status strings.
#include "frt_host.h"

#include <atomic>
#include <mutex>
#include <unordered_map>

#include "frt_device.cuh"

namespace frt {
namespace {
__global__ void noop_kernel() { pdl_enter(); }
std::atomic<int> g_pdl{1};
}  // namespace

bool pdl_enabled() { return g_pdl.load(std::memory_order_relaxed) != 0; }

int persistent_grid(const void* kernel, int threads, size_t smem) {
  static std::mutex mu;
  static std::unordered_map<uint64_t, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const uint64_t key = reinterpret_cast<uintptr_t>(kernel) ^ ((uint64_t)threads << 40) ^ ((uint64_t)dev << 56);
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  int sms = 0, per_sm = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  const int g = sms * (per_sm > 0 ? per_sm : 1);
  std::lock_guard<std::mutex> lk(mu);
  cache[key] = g;
  return g;
}
}  // namespace frt

extern "C" frt_status frt_noop(int grid, int block, cudaStream_t stream) {
  if (grid < 1 || block < 1 || block > 1024) return FRT_ERR_INVALID_ARG;
  return frt::launch(frt::noop_kernel, dim3(grid), dim3(block), 0, stream);
}

extern "C" void frt_set_pdl(int enable) { frt::g_pdl.store(enable ? 1 : 0, std::memory_order_relaxed); }

extern "C" int frt_get_pdl(void) { return frt::g_pdl.load(std::memory_order_relaxed); }

extern "C" const char* frt_status_string(frt_status status) {
  switch (status) {
    case FRT_OK: return "FRT_OK";
    case FRT_ERR_INVALID_ARG: return "FRT_ERR_INVALID_ARG: bad size, pointer, alignment or enum";
    case FRT_ERR_UNSUPPORTED: return "FRT_ERR_UNSUPPORTED: shape outside what this build covers";
    case FRT_ERR_CUDA: return "FRT_ERR_CUDA: the kernel launch failed";
    default: return "unknown frt_status";
  }
}
