// Host-side launch helpers shared by the kernels of libnmoe.
#include <cudaTypedefs.h>

#include <mutex>
#include <vector>

#include "nmoe_internal.cuh"

namespace nmoe {

namespace {
struct SmemEntry {
  const void* kernel;
  int device;
  size_t bytes;
};
std::mutex g_smem_mu;
std::vector<SmemEntry> g_smem;
}  // namespace

cudaError_t set_smem_limit(const void* kernel, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_smem_mu);
  for (auto& s : g_smem)
    if (s.kernel == kernel && s.device == dev && s.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  for (auto& s : g_smem)
    if (s.kernel == kernel && s.device == dev) {
      s.bytes = bytes;
      return cudaSuccess;
    }
  g_smem.push_back({kernel, dev, bytes});
  return cudaSuccess;
}

void* tensor_map_encoder() {
  // looked up once; a function-local static is initialised exactly once, even when
  // several host threads make their first call at the same time
  static void* const fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();  // the failed query is not the caller's error
      f = nullptr;
    }
    return f;
  }();
  return fn;
}

}  // namespace nmoe
